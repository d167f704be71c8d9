"""GPU parity on the method's degenerate inputs: the CUDA scan and decode step
(through the C ABI) against the fp64 oracle, element by element.

These are the limits the oracle is pinned on (page "Mamba 논문 리뷰", §3.2:
Delta decides how much of the state is kept; §2.2: the discretised
recurrence), run through the kernels:

  * x = 0 on whole steps (padding tokens), alone, in runs of 60+ steps inside
    a segment and across segment boundaries, and as a leading / trailing pad;
  * Delta = 0 with softplus off: the state is kept, y = C h0 + D x;
  * delta + bias = 60: memoryless (exp(Delta A) underflows), h_t = Delta B x;
  * A = 0: the state is h0 plus a running sum of Delta B x;
  * |h0| ~ 1e4;

with one segment and with five, in fp32 io (bound 1e-5) and bf16 io (1e-2).
The kernel keeps its state scaled by s_t ~ Delta_t x_t with a 2^-64 floor:
these inputs drive s_t to that floor and the per-step rescaling factor
s_{t-1} / s_t to its extremes."""
import numpy as np
import pytest

import oracle
import ssm_inputs as gen
from tests.gpu_util import TOL, dev, gpu_scan, host, oracle_scan, rel_err

pytestmark = pytest.mark.gpu

BATCH, L, DIM, N = 2, 400, 320, 16


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    for k in ("SSM_SCAN_SEGMENTS", "SSM_SCAN_DISABLE_TMA", "SSM_SCAN_CTAS_PER_SM",
              "SSM_SCAN_WAIT_LIMIT_NS", "SSM_SCAN_TEST_STALL"):
        monkeypatch.delenv(k, raising=False)
    yield


def _to_io(a, io):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return gen.f32_to_bf16_bits(a) if io == "bf16" else a


def _as_f32(a, io):
    return gen.bf16_bits_to_f32(a) if io == "bf16" else np.asarray(a, dtype=np.float32)


def _zero_steps(inp, io, steps):
    x = _as_f32(inp["x"], io).copy()
    x[:, steps, :] = 0.0
    inp["x"] = _to_io(x, io)


def _check(inp, io, softplus=True, what=""):
    y, hl = gpu_scan(inp, softplus=softplus)
    yr, hr = oracle_scan(inp, io, softplus=softplus)
    yg, hg = host(y), host(hl)
    ey, eh = rel_err(yg, yr), rel_err(hg, hr)
    print(f"{what}: rel err y {ey:.3e}  h_last {eh:.3e}")
    assert np.all(np.isfinite(yg)) and np.all(np.isfinite(hg)), what
    assert ey <= TOL[io], f"{what}: y rel err {ey:.3e} > {TOL[io]}"
    assert eh <= TOL[io], f"{what}: h_last rel err {eh:.3e} > {TOL[io]}"
    return yg, hg


IOS = ["f32", "bf16"]
SEGS = ["1", "5"]


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_zero_x_padding_runs(monkeypatch, io, segments):
    """Zero inputs: a leading pad, single zero steps, a 70-step run in the
    middle (across a segment boundary with five segments of 80 steps) and a
    trailing pad."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 501, with_h0=True)
    steps = list(range(0, 12)) + [30, 32, 33, 97] + list(range(150, 220)) + list(range(340, L))
    _zero_steps(inp, io, steps)
    _check(inp, io, what=f"zero-x runs {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_all_zero_x_keeps_decaying_h0(monkeypatch, io, segments):
    """x = 0 everywhere: no input enters, h_t = exp(A sum Delta) h0 and
    y = C h (the skip term is zero)."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 502, with_h0=True)
    _zero_steps(inp, io, list(range(L)))
    _check(inp, io, what=f"all-zero x {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_delta_zero_keeps_state(monkeypatch, io, segments):
    """softplus off and delta + bias = 0: exp(0 A) = 1 and the input term is
    zero, so h_last = h0 and y_t = (C_t h0 + D x_t) SiLU(z_t)."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 503, with_h0=True)
    inp["delta"] = _to_io(np.zeros((BATCH, L, DIM), np.float32), io)
    inp["delta_bias"] = None
    yg, hg = _check(inp, io, softplus=False, what=f"Delta = 0 {io} seg={segments}")
    # the state is kept exactly by the definition; the GPU's within rounding
    assert rel_err(hg, inp["h0"]) <= TOL[io]


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_delta_zero_on_some_steps(monkeypatch, io, segments):
    """softplus off with Delta = 0 on every third step and in a 60-step run,
    positive elsewhere: the state passes those steps unchanged."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 504, with_h0=True)
    rng = np.random.default_rng(504)
    d = rng.uniform(0.01, 0.3, (BATCH, L, DIM)).astype(np.float32)
    d[:, ::3, :] = 0.0
    d[:, 200:260, :] = 0.0
    inp["delta"] = _to_io(d, io)
    inp["delta_bias"] = None
    _check(inp, io, softplus=False, what=f"Delta = 0 on some steps {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_huge_delta_is_memoryless(monkeypatch, io, segments):
    """delta + bias = 60 (above the softplus cut, so Delta = 60): every decay
    exp(-60 (n+1)) vanishes and h_t = Delta B_t x_t, with zero-x steps mixed
    in (then the state is zero)."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 505, with_h0=True)
    inp["delta"] = _to_io(np.full((BATCH, L, DIM), 60.0, np.float32), io)
    inp["delta_bias"] = np.zeros(DIM, np.float32)
    _zero_steps(inp, io, [5, 6, 7, 100, 250, L - 1])
    yg, hg = _check(inp, io, what=f"Delta = 60 {io} seg={segments}")
    # memoryless: h_last = 60 B_{L-1} x_{L-1}, and x_{L-1} = 0 here
    assert np.max(np.abs(hg)) <= 1e-20


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_huge_delta_on_some_steps(monkeypatch, io, segments):
    """Memoryless steps (Delta = 60) between ordinary ones: each resets the
    state to its own input term."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 506, with_h0=True)
    d = _as_f32(inp["delta"], io).copy()
    d[:, ::7, :] = 60.0
    d[:, 300:330, :] = 60.0
    inp["delta"] = _to_io(d, io)
    _check(inp, io, what=f"Delta = 60 on some steps {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_A_zero_is_a_running_sum(monkeypatch, io, segments):
    """A = 0: every decay is 1 and h_t = h0 + sum_{s<=t} Delta_s B_s x_s
    (the linear-attention recurrence), with zero-x steps mixed in."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 507, with_h0=True)
    inp["A"] = np.zeros((DIM, N), np.float32)
    _zero_steps(inp, io, list(range(40, 110)))
    _check(inp, io, what=f"A = 0 {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_large_h0(monkeypatch, io, segments):
    """|h0| ~ 1e4 with ordinary inputs, and with a run of zero-x steps at the
    start (the scaled state then holds h0 / 2^-64)."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 508, with_h0=True)
    inp["h0"] = (inp["h0"] * 1e4).astype(np.float32)
    _check(inp, io, what=f"|h0| ~ 1e4 {io} seg={segments}")
    _zero_steps(inp, io, list(range(0, 64)))
    _check(inp, io, what=f"|h0| ~ 1e4, zero-x start {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
def test_edge_values_default_plan(io):
    """All the degenerate inputs at once, in the split the library picks by
    itself, on a batch of rows wide enough for several channel tiles."""
    inp = gen.make_scan_inputs(3, 700, 768, N, io, 509, with_h0=True)
    x = _as_f32(inp["x"], io).copy()
    x[:, 100:180, :] = 0.0
    x[:, ::11, :] = 0.0
    inp["x"] = _to_io(x, io)
    d = _as_f32(inp["delta"], io).copy()
    d[:, 400:420, :] = 60.0
    inp["delta"] = _to_io(d, io)
    inp["A"][::5] = 0.0  # some channels without decay
    inp["h0"] = (inp["h0"] * 1e3).astype(np.float32)
    _check(inp, io, what=f"mixed edge values {io}")


# --------------------------------------------------------- decode step ----
def _decode_run(io, steps, edit, seed, A=None, h0_scale=1.0, softplus=True):
    """`steps` decode steps on the GPU and in the oracle; `edit(step, inp)`
    changes a step's inputs before both use them."""
    from selective_state_space_39_b200 import ssm_state_update
    batch, dim = 3, 260
    const = gen.decode_constants(dim, N, seed)
    if A is not None:
        const["A"] = A(dim)
    bias = None if not softplus else const["delta_bias"]
    rng = np.random.default_rng(seed)
    h0 = (rng.standard_normal((batch, dim, N)) * h0_scale).astype(np.float32)
    state = dev(h0).clone()
    ref = h0.astype(np.float64)
    for step in range(steps):
        inp = gen.make_decode_inputs(batch, dim, N, io, seed, step)
        edit(step, inp)
        y = ssm_state_update(state, dev(inp["x"]), dev(inp["delta"]), dev(const["A"]),
                             dev(inp["B"]), dev(inp["C"]), D=dev(const["D"]), z=dev(inp["z"]),
                             delta_bias=dev(bias), softplus=softplus)
        yr = oracle.state_update(ref, inp["x"], inp["delta"], const["A"], inp["B"], inp["C"],
                                 D=const["D"], z=inp["z"], delta_bias=bias, softplus=softplus,
                                 io=io)
        assert rel_err(host(y), yr) <= TOL[io], f"step {step}"
    assert np.all(np.isfinite(host(state)))
    assert rel_err(host(state), ref) <= TOL[io]
    return host(state), h0


@pytest.mark.parametrize("io", IOS)
def test_decode_zero_x_and_huge_delta(io):
    def edit(step, inp):
        if step % 3 == 0:
            inp["x"] = _to_io(np.zeros(inp["x"].shape, np.float32), io)
        if step % 5 == 0:
            inp["delta"] = _to_io(np.full(inp["delta"].shape, 60.0, np.float32), io)
    _decode_run(io, 30, edit, 601)


@pytest.mark.parametrize("io", IOS)
def test_decode_delta_zero_keeps_state(io):
    def edit(step, inp):
        inp["delta"] = _to_io(np.zeros(inp["delta"].shape, np.float32), io)
    state, h0 = _decode_run(io, 12, edit, 602, softplus=False)
    assert rel_err(state, h0) <= TOL[io]


@pytest.mark.parametrize("io", IOS)
def test_decode_A_zero_and_large_state(io):
    _decode_run(io, 25, lambda step, inp: None, 603,
                A=lambda dim: np.zeros((dim, N), np.float32), h0_scale=1e4)


# ------------------------------------------- A without structure (one exp per state) ----
@pytest.mark.parametrize("io", IOS)
@pytest.mark.parametrize("segments", SEGS)
def test_learned_A_edge_values(monkeypatch, io, segments):
    """A as after training (no (n+1) A_0 structure: the path with one exp per
    state), with zero-x runs, memoryless steps (Delta = 60), and single states
    without decay (A_dn = 0 for some n)."""
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 510, with_h0=True)
    A = gen.a_matrix_learned(DIM, N, 510).copy()
    A[::3, 5] = 0.0
    A[1::7, 0] = 0.0
    inp["A"] = A
    _zero_steps(inp, io, list(range(20, 95)) + [200, 201, L - 1])
    d = _as_f32(inp["delta"], io).copy()
    d[:, 150:160, :] = 60.0
    d[:, 300, :] = 60.0
    inp["delta"] = _to_io(d, io)
    _check(inp, io, what=f"learned A edge values {io} seg={segments}")


@pytest.mark.parametrize("io", IOS)
def test_learned_A_delta_zero_keeps_state(io):
    """Delta = 0 (softplus off) with A without structure: h_last = h0."""
    inp = gen.make_scan_inputs(BATCH, L, DIM, N, io, 511, with_h0=True)
    inp["A"] = gen.a_matrix_learned(DIM, N, 511)
    inp["delta"] = _to_io(np.zeros((BATCH, L, DIM), np.float32), io)
    inp["delta_bias"] = None
    _, hg = _check(inp, io, softplus=False, what=f"learned A, Delta = 0 {io}")
    assert rel_err(hg, inp["h0"]) <= TOL[io]

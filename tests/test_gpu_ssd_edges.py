"""GPU parity of the tensor-core SSD scan on the method's degenerate cases,
against the fp64 oracle (bf16 io, bound 1e-2 relative to max|ref|):

* Delta large (softplus(60) = 60): every step forgets the state, so y_t is
  C_t (Delta_t B_t x_t) + D x_t; in the kernel every factor e^{cum_t - cum_s}
  below the diagonal underflows to zero;
* Delta = 0 (softplus off, dt = 0): the state is kept, y_t = C_t h0 + D x_t;
* x = 0 on a run of steps across a chunk boundary (padding tokens);
* heads of very different decay side by side in one CTA's pair.

Lengths of 300 steps: two 128-step chunks and a ragged one. The SSD decode
step is run through the same limits, carried over 16 steps."""
import numpy as np
import pytest

import ssm_inputs as gen
from tests.test_gpu_ssd import TOL, check

pytestmark = pytest.mark.gpu

L, H, P, N = 300, 4, 64, 128


def _inputs(seed):
    return gen.make_ssd_inputs(2, L, H, P, N, "bf16", seed, with_h0=True)


def _bf16(a):
    return gen.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


@pytest.fixture(autouse=True)
def _tc(monkeypatch):
    monkeypatch.delenv("SSM_SSD_LEGACY", raising=False)
    yield


def test_ssd_large_delta_forgets_the_state():
    inp = _inputs(701)
    inp["dt"] = _bf16(np.full(inp["dt"].shape, 60.0))
    inp["dt_bias"] = np.zeros(H, dtype=np.float32)
    check(inp, "Delta = 60")


def test_ssd_zero_delta_keeps_the_state():
    inp = _inputs(702)
    inp["dt"] = _bf16(np.zeros(inp["dt"].shape))
    check(inp, "Delta = 0", softplus=False, keep=("D", "h0"))


def test_ssd_zero_input_run_across_a_chunk_boundary():
    inp = _inputs(703)
    x = gen.bf16_bits_to_f32(inp["x"]).copy()
    x[:, 100:200] = 0.0
    inp["x"] = _bf16(x)
    check(inp, "x = 0 on steps 100-199")


def test_ssd_fast_and_slow_heads_in_one_pair():
    inp = _inputs(704)
    dt = gen.bf16_bits_to_f32(inp["dt"]).copy()
    dt[:, :, 0::2] = 8.0    # softplus(8 + bias) ~ 4: decay e^{-4..-64} per step
    dt[:, :, 1::2] = -12.0  # Delta ~ 6e-6: the state barely moves
    inp["dt"] = _bf16(dt)
    check(inp, "fast and slow heads")


def test_ssd_large_state_small_input():
    inp = _inputs(705)
    inp["h0"] = (inp["h0"] * 1e4).astype(np.float32)
    check(inp, "|h0| ~ 1e4")
    assert TOL == 1e-2


# ------------------------------------------------------------ decode step ----
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_ssd_decode_degenerate_steps(io):
    """Carried decode steps against the oracle's, element by element (fp32 io
    1e-5, bf16 1e-2): ordinary steps, then dt = 60 (the state is replaced by
    the step's input term), x = 0 (the state only decays), and dt = -30
    (Delta ~ 1e-13: the state is kept), in turn."""
    import oracle
    import torch
    from selective_state_space_39_b200 import ssm_ssd_state_update
    from tests.gpu_util import dev, host, rel_err
    from tests.test_gpu_ssd import DTOL, decode_inputs

    batch, heads, p, n = 3, 4, 64, 128
    const = gen.ssd_constants(heads, 900)
    rng = np.random.default_rng(900)
    state = torch.from_numpy(rng.standard_normal((batch, heads, p, n)).astype(np.float32)).cuda()
    ref = host(state).copy()
    to_io = (lambda a: _bf16(a)) if io == "bf16" else (lambda a: np.asarray(a, np.float32))
    for step in range(16):
        inp = decode_inputs(batch, heads, p, n, io, 900, step)
        kind = step % 4
        if kind == 1:
            inp["dt"] = to_io(np.full(inp["dt"].shape, 60.0))
        elif kind == 2:
            inp["x"] = to_io(np.zeros(inp["x"].shape))
        elif kind == 3:
            inp["dt"] = to_io(np.full(inp["dt"].shape, -30.0))
        y = ssm_ssd_state_update(state, dev(inp["x"]), dev(inp["dt"]), dev(const["A"]),
                                 dev(inp["B"]), dev(inp["C"]), D=dev(const["D"]),
                                 dt_bias=dev(const["dt_bias"]))
        yr = oracle.ssd_state_update(ref, inp["x"], inp["dt"], const["A"], inp["B"], inp["C"],
                                     D=const["D"], dt_bias=const["dt_bias"], io=io)
        assert torch.isfinite(y.float()).all()
        assert rel_err(host(y), yr) <= DTOL[io], f"step {step} (kind {kind})"
    assert rel_err(host(state), ref) <= DTOL[io]

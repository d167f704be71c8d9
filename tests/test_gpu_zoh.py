"""GPU parity of the exact zero-order-hold scan and decode step
(ssm_scan_fwd_zoh, ssm_state_update_zoh, through the C ABI) against the fp64
oracle with its ZOH input term (exp(Delta A) - 1) / A * B.

Bound: the forward's, max|y - y_ref| / max|y_ref| <= 1e-5 for fp32 io and
1e-2 for bf16 io, the same for h_last."""
import numpy as np
import pytest

import ssm_inputs as gen
from tests.gpu_util import TOL, dev, host, rel_err, sample_channels

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    for k in ("SSM_SCAN_SEGMENTS", "SSM_SCAN_DISABLE_TMA"):
        monkeypatch.delenv(k, raising=False)
    yield


def gpu_zoh(inp):
    from selective_state_space_39_b200 import ssm_scan_fwd
    return ssm_scan_fwd(dev(inp["x"]), dev(inp["delta"]), dev(inp["A"]), dev(inp["B"]),
                        dev(inp["C"]), D=dev(inp.get("D")), z=dev(inp.get("z")),
                        delta_bias=dev(inp.get("delta_bias")), h0=dev(inp.get("h0")), zoh=True)


def oracle_zoh(inp, io, channels=None):
    import oracle
    return oracle.selective_scan(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                 D=inp.get("D"), z=inp.get("z"), delta_bias=inp.get("delta_bias"),
                                 h0=inp.get("h0"), io=io, channels=channels,
                                 nthreads=gen.default_threads(), zoh=True)


def check(y, hl, yr, hr, io, what):
    ey, eh = rel_err(y, yr), rel_err(hl, hr)
    print(f"{what}: rel err y {ey:.3e} h_last {eh:.3e}")
    assert np.all(np.isfinite(y)) and ey <= TOL[io] and eh <= TOL[io], what


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N", [2, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("segments", [None, "3"])
@pytest.mark.parametrize("tma", [True, False])
def test_zoh_shapes(monkeypatch, io, N, segments, tma):
    if segments:
        monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    if not tma:
        monkeypatch.setenv("SSM_SCAN_DISABLE_TMA", "1")
    inp = gen.make_scan_inputs(2, 77, 264, N, io, 21, with_h0=True)
    y, hl = gpu_zoh(inp)
    yr, hr = oracle_zoh(inp, io)
    check(host(y), host(hl), yr, hr, io, f"zoh {io} N={N} seg={segments} tma={tma}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_zoh_generic_A_and_zero_A(io):
    """A that is not (n+1) A[d,0], including entries equal to 0 (where the
    ZOH term is Delta B), takes the per-state path."""
    inp = gen.make_scan_inputs(2, 50, 136, 16, io, 23, with_h0=True)
    rng = np.random.default_rng(7)
    A = (-rng.uniform(0.05, 2.0, inp["A"].shape)).astype(np.float32)
    A[3, :] = 0.0
    A[5, 2] = 0.0
    inp["A"] = A
    y, hl = gpu_zoh(inp)
    yr, hr = oracle_zoh(inp, io)
    check(host(y), host(hl), yr, hr, io, f"zoh generic A {io}")


def test_zoh_small_steps_stay_accurate():
    """Delta A near 0 (bias giving Delta ~ 1e-4): the ZOH factor is formed
    without cancellation, so fp32 io keeps the 1e-5 bound."""
    inp = gen.make_scan_inputs(2, 200, 128, 16, "f32", 25)
    inp["delta_bias"] = np.full(128, -9.2, dtype=np.float32)  # softplus ~ 1e-4
    y, hl = gpu_zoh(inp)
    yr, hr = oracle_zoh(inp, "f32")
    check(host(y), host(hl), yr, hr, "f32", "zoh small Delta")


def test_zoh_mamba130m_layer_sampled():
    w = gen.SCAN_WORKLOADS["mamba130m_layer_b8_l2048_d1536"]
    inp = gen.workload_inputs(w)
    y, hl = gpu_zoh(inp)
    chans = sample_channels(w.batch, w.dim, 12)
    yr, hr = oracle_zoh(inp, w.io, channels=chans)
    yg, hg = host(y), host(hl)
    ys = np.stack([yg[b, :, d] for b, d in chans])
    hs = np.stack([hg[b, d] for b, d in chans])
    check(ys, hs, yr, hr, w.io, "zoh 8x2048x1536")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_zoh_decode_matches_oracle(io):
    import oracle
    from selective_state_space_39_b200 import ssm_state_update
    c = gen.make_scan_inputs(3, 6, 200, 16, io, 27, with_h0=True)
    state = dev(c["h0"]).clone()
    ref = c["h0"].astype(np.float64).copy()
    for t in range(6):
        s = {k: np.ascontiguousarray(c[k][:, t]) for k in ("x", "delta", "z", "B", "C")}
        yt = ssm_state_update(state, dev(s["x"]), dev(s["delta"]), dev(c["A"]), dev(s["B"]),
                              dev(s["C"]), D=dev(c["D"]), z=dev(s["z"]),
                              delta_bias=dev(c["delta_bias"]), zoh=True)
        yr = oracle.state_update(ref, s["x"], s["delta"], c["A"], s["B"], s["C"], D=c["D"],
                                 z=s["z"], delta_bias=c["delta_bias"], io=io, zoh=True)
        e = rel_err(host(yt), yr)
        assert e <= TOL[io], f"zoh decode {io} step {t}: {e:.3e}"
    assert rel_err(host(state), ref) <= TOL[io]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("segments", [None, "4"])
def test_zoh_degenerate_inputs(monkeypatch, io, segments):
    """The exact-ZOH scan on x = 0 runs across segments (the state only
    decays), memoryless steps (delta + bias = 60: exp(Delta A) vanishes and the
    input term is -B x / A), and |h0| ~ 1e3."""
    if segments:
        monkeypatch.setenv("SSM_SCAN_SEGMENTS", segments)
    inp = gen.make_scan_inputs(2, 240, 264, 16, io, 31, with_h0=True)
    f32 = (lambda a: gen.bf16_bits_to_f32(a)) if io == "bf16" else (lambda a: a)
    back = (lambda a: gen.f32_to_bf16_bits(a)) if io == "bf16" else (lambda a: a)
    x = f32(inp["x"]).astype(np.float32).copy()
    x[:, 40:130, :] = 0.0
    inp["x"] = back(x)
    d = f32(inp["delta"]).astype(np.float32).copy()
    d[:, 180:190, :] = 60.0
    d[:, ::17, :] = 60.0
    inp["delta"] = back(d)
    inp["h0"] = (inp["h0"] * 1e3).astype(np.float32)
    y, hl = gpu_zoh(inp)
    yr, hr = oracle_zoh(inp, io)
    check(host(y), host(hl), yr, hr, io, f"zoh degenerate {io} seg={segments}")

"""GPU parity of the backward pass: ssm_scan_bwd (through the C ABI) against
the fp64 oracle's adjoint loop, gradient by gradient.

Bound per gradient: max|g - g_ref| / max|g_ref| <= 1e-4 for fp32 io and
2e-2 for bf16 io (the dx, ddelta, dz outputs are rounded to bf16, 2^-9
relative, and the bf16 path uses MUFU approximations). fp32 io is looser
than the forward's 1e-5 because the gradients are sums over every step of
products of up to four rounded factors (dA sums batch x seqlen terms)."""
import numpy as np
import pytest
import torch

import ssm_inputs as gen
from tests.gpu_util import dev, host, rel_err, sample_channels

pytestmark = pytest.mark.gpu

TOL_BWD = {"f32": 1e-4, "bf16": 2e-2}
NAMES = ("dx", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dh0")


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    monkeypatch.delenv("SSM_SCAN_BWD_SEGMENTS", raising=False)
    yield


def gpu_bwd(inp, grads, softplus=True, **kw):
    from selective_state_space_39_b200 import ssm_scan_bwd
    return ssm_scan_bwd(dev(inp["x"]), dev(inp["delta"]), dev(inp["A"]), dev(inp["B"]),
                        dev(inp["C"]), dev(grads["dy"]), D=dev(inp.get("D")), z=dev(inp.get("z")),
                        delta_bias=dev(inp.get("delta_bias")), softplus=softplus,
                        h0=dev(inp.get("h0")), dh_last=dev(grads.get("dh_last")), **kw)


def oracle_bwd(inp, grads, io, softplus=True, channels=None, nthreads=None):
    import oracle
    return oracle.selective_scan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                     grads["dy"], D=inp.get("D"), z=inp.get("z"),
                                     delta_bias=inp.get("delta_bias"), softplus=softplus,
                                     h0=inp.get("h0"), dh_last=grads.get("dh_last"), io=io,
                                     channels=channels,
                                     nthreads=nthreads or gen.default_threads())


def check_all(g, ref, io, what, names=NAMES):
    for k in names:
        if ref.get(k) is None:
            assert g.get(k) is None, f"{what}: {k} should be None"
            continue
        got = host(g[k])
        assert np.all(np.isfinite(got)), f"{what}: {k} not finite"
        e = rel_err(got, ref[k])
        print(f"{what}: {k} rel err {e:.3e}")
        assert e <= TOL_BWD[io], f"{what}: {k} rel err {e:.3e} > {TOL_BWD[io]}"


def small_case(io, N, batch=2, L=45, dim=150, seed=11, **kw):
    inp = gen.make_scan_inputs(batch, L, dim, N, io, seed, **kw)
    grads = gen.make_grad_inputs(batch, L, dim, N, io, seed)
    return inp, grads


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N", [2, 4, 8, 16])
@pytest.mark.parametrize("segments", [None, "1", "3", "7"])
def test_bwd_ragged_shapes(monkeypatch, io, N, segments):
    """L = 45 (not a multiple of the 4-step tile), dim = 150 (not a multiple
    of the 128-channel CTA), h0 and dh_last given, gate and skip on."""
    if segments:
        monkeypatch.setenv("SSM_SCAN_BWD_SEGMENTS", segments)
    inp, grads = small_case(io, N, with_h0=True)
    g = gpu_bwd(inp, grads)
    check_all(g, oracle_bwd(inp, grads, io), io, f"{io} N={N} seg={segments}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_bwd_generic_A(io):
    """A that is not (n+1) A[d,0] takes the one-exp-per-state path."""
    inp, grads = small_case(io, 16, L=33, dim=130, with_h0=True)
    rng = np.random.default_rng(5)
    inp["A"] = (-rng.uniform(0.05, 2.0, inp["A"].shape)).astype(np.float32)
    g = gpu_bwd(inp, grads)
    check_all(g, oracle_bwd(inp, grads, io), io, f"{io} generic A")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("flags", ["no_gate", "no_skip", "no_bias", "no_softplus",
                                   "no_h0_no_dh_last"])
def test_bwd_optional_terms(io, flags):
    kw = dict(gate=flags != "no_gate", skip=flags != "no_skip", with_h0=flags != "no_h0_no_dh_last")
    inp = gen.make_scan_inputs(2, 21, 140, 16, io, 17, **kw)
    grads = gen.make_grad_inputs(2, 21, 140, 16, io, 17, with_dh_last=flags != "no_h0_no_dh_last")
    softplus = flags != "no_softplus"
    if flags == "no_bias":
        inp["delta_bias"] = None
    if not softplus:  # keep Delta > 0 without softplus: |delta| + 0.01, bias >= 0
        f = gen.as_float(inp["delta"], io)
        v = np.abs(f) + np.float32(0.01)
        inp["delta"] = gen.f32_to_bf16_bits(v) if io == "bf16" else v.astype(np.float32)
        inp["delta_bias"] = np.abs(inp["delta_bias"]) * np.float32(0.1)
    g = gpu_bwd(inp, grads, softplus=softplus)
    check_all(g, oracle_bwd(inp, grads, io, softplus=softplus), io, f"{io} {flags}")


def test_bwd_softplus_cutoff():
    """Channels whose delta + bias lies above the softplus cut (20) use the
    identity and its derivative 1."""
    inp, grads = small_case("f32", 16, L=17, dim=128)
    inp["delta_bias"][:64] = 21.0
    inp["A"][:64] *= np.float32(0.01)  # keep exp(Delta A) away from 0
    g = gpu_bwd(inp, grads)
    check_all(g, oracle_bwd(inp, grads, "f32"), "f32", "softplus cutoff")


def test_bwd_mamba130m_layer_full():
    """The 8 x 2048 x 1536 bf16 layer: every gradient of every channel."""
    w = gen.SCAN_WORKLOADS["mamba130m_layer_b8_l2048_d1536"]
    inp = gen.workload_inputs(w)
    grads = gen.make_grad_inputs(w.batch, w.seqlen, w.dim, w.dstate, w.io, w.seed)
    g = gpu_bwd(inp, grads)
    torch.cuda.synchronize()
    check_all(g, oracle_bwd(inp, grads, w.io), w.io, "mamba130m layer")


def test_bwd_long_sampled():
    """262144 steps, batch 1: per-channel gradients (dx, ddelta, dz, dh0) and
    the per-channel sums dA, dD, ddelta_bias on sampled channels."""
    w = gen.SCAN_WORKLOADS["long_b1_l262144_d1536"]
    inp = gen.workload_inputs(w)
    grads = gen.make_grad_inputs(w.batch, w.seqlen, w.dim, w.dstate, w.io, w.seed)
    g = gpu_bwd(inp, grads)
    torch.cuda.synchronize()
    chans = sample_channels(w.batch, w.dim, 10)
    # each oracle thread keeps its own (seqlen, dstate) sums: few threads here
    ref = oracle_bwd(inp, grads, w.io, channels=chans, nthreads=8)
    ds = [d for _, d in chans]
    got = {
        "dx": np.stack([host(g["dx"][b, :, d]) for b, d in chans]),
        "ddelta": np.stack([host(g["ddelta"][b, :, d]) for b, d in chans]),
        "dz": np.stack([host(g["dz"][b, :, d]) for b, d in chans]),
        "dh0": np.stack([host(g["dh0"][b, d]) for b, d in chans]),
        "dA": host(g["dA"])[ds], "dD": host(g["dD"])[ds],
        "ddelta_bias": host(g["ddelta_bias"])[ds],
    }
    ref_s = dict(ref)
    for k in ("dA", "dD", "ddelta_bias"):
        ref_s[k] = ref[k][ds]
    for k, v in got.items():
        assert np.all(np.isfinite(v)), k
        e = rel_err(v, ref_s[k])
        print(f"long: {k} rel err {e:.3e}")
        assert e <= TOL_BWD[w.io], f"long: {k} rel err {e:.3e}"


def test_bwd_deterministic():
    """Sums run in a fixed order: two calls agree bit for bit."""
    inp, grads = small_case("bf16", 16, batch=3, L=130, dim=300, with_h0=True)
    g1 = gpu_bwd(inp, grads)
    g2 = gpu_bwd(inp, grads)
    for k in NAMES:
        assert torch.equal(g1[k], g2[k]), k


def test_bwd_seqlen_zero():
    """No steps: dh0 = dh_last and every parameter gradient is zero."""
    inp, grads = small_case("f32", 16, L=0, dim=64, with_h0=True)
    g = gpu_bwd(inp, grads)
    assert torch.equal(g["dh0"].cpu(), torch.from_numpy(grads["dh_last"]))
    for k in ("dA", "dD", "ddelta_bias"):
        assert not g[k].any(), k


def test_bwd_workspace_too_small():
    from selective_state_space_39_b200 import SsmError
    inp, grads = small_case("f32", 16, L=16, dim=64)
    with pytest.raises(SsmError):
        gpu_bwd(inp, grads, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))

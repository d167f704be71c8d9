"""GPU parity of the multi-head SSD scan (Mamba-2, tensor-core chunked form,
through the C ABI) against the fp64 oracle's sequential per-head loop.

Bound: max|g - g_ref| / max|g_ref| <= 1e-2 for y and h_last: bf16 io, with
the chunk's products taken on bf16 tensor-core operands (the decay-weighted
G, the weighted x and a bf16 copy of the fp32 state for the readout are each
rounded to 2^-9 relative) and fp32 accumulation."""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as gen
from tests.gpu_util import dev, host, rel_err

pytestmark = pytest.mark.gpu

TOL = 1e-2


def run(inp, softplus=True, last=True, keep=("D", "dt_bias", "h0")):
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd
    opt = {k: (dev(inp[k]) if k in keep else None) for k in ("D", "dt_bias", "h0")}
    return ssm_ssd_scan_fwd(dev(inp["x"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["B"]),
                            dev(inp["C"]), softplus=softplus, return_last_state=last, **opt)


def reference(inp, softplus=True, keep=("D", "dt_bias", "h0"), pairs=None):
    opt = {k: (inp[k] if k in keep else None) for k in ("D", "dt_bias", "h0")}
    return oracle.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], softplus=softplus,
                           io="bf16", pairs=pairs, **opt)


def check(inp, what, **kw):
    y, hl = run(inp, **{k: v for k, v in kw.items() if k != "pairs"})
    yr, hr = reference(inp, **kw)
    assert torch.isfinite(y.float()).all() and torch.isfinite(hl).all()
    ey, eh = rel_err(host(y), yr), rel_err(host(hl), hr)
    print(f"{what}: y rel err {ey:.3e}, h_last rel err {eh:.3e}")
    assert ey <= TOL and eh <= TOL, what


@pytest.mark.parametrize("N", [64, 128, 256])
@pytest.mark.parametrize("shape", [(2, 100, 3), (1, 32, 2), (1, 5, 1), (3, 97, 4)],
                         ids=["ragged", "one_chunk", "short", "odd"])
@pytest.mark.parametrize("h0", [True, False])
def test_ssd_shapes(N, shape, h0):
    """Chunk-ragged lengths (100 = 3 chunks + 4 steps), exactly one chunk,
    fewer steps than a chunk, with and without an initial state."""
    batch, L, H = shape
    inp = gen.make_ssd_inputs(batch, L, H, 64, N, "bf16", 50 + N + L, with_h0=h0)
    check(inp, f"N={N} {shape} h0={h0}")


@pytest.mark.parametrize("softplus", [True, False])
@pytest.mark.parametrize("keep", [(), ("D",), ("dt_bias", "h0")], ids=["none", "D", "bias_h0"])
def test_ssd_optional_terms(softplus, keep):
    inp = gen.make_ssd_inputs(2, 70, 3, 64, 128, "bf16", 77, with_h0=True)
    if not softplus:  # raw steps used as they are: keep them (and the bias) positive, small
        inp["dt"] = gen.f32_to_bf16_bits(np.abs(gen.bf16_bits_to_f32(inp["dt"])) * 0.1)
        inp["dt_bias"] = np.full(3, 0.02, dtype=np.float32)
    check(inp, f"softplus={softplus} keep={keep}", softplus=softplus, keep=keep)


def test_ssd_pages_example_layer():
    """The pages' Mamba-2 layer input (1 x 1024, d_model 2048: 64 heads of 64,
    d_state 128), every output and the end state."""
    w = gen.SSD_WORKLOADS["ssd_mamba2_b1_l1024_h64_p64_n128"]
    check(gen.ssd_workload_inputs(w), w.name)


def test_ssd_full_size_sampled_heads():
    """4 x 4096, 64 heads, d_state 128, with h0: the benchmark's launch, the
    oracle on sampled (batch, head) pairs (first, last and interior heads)."""
    w = gen.SSD_WORKLOADS["ssd_mamba2_b4_l4096_h64_p64_n128"]
    inp = gen.ssd_workload_inputs(w)
    pairs = [(0, 0), (0, 63), (1, 17), (2, 32), (3, 0), (3, 63)]
    y, hl = run(inp)
    yr, hr = reference(inp, pairs=pairs)
    yh, hh = host(y), host(hl)
    for k, (b, h) in enumerate(pairs):
        ey, eh = rel_err(yh[b, :, h], yr[k]), rel_err(hh[b, h], hr[k])
        assert ey <= TOL and eh <= TOL, f"pair {(b, h)}: y {ey:.3e} h {eh:.3e}"
    assert torch.isfinite(y.float()).all()


def test_ssd_empty_sequence_passes_the_state_through():
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd
    inp = gen.make_ssd_inputs(2, 0, 3, 64, 64, "bf16", 5, with_h0=True)
    y, hl = ssm_ssd_scan_fwd(dev(inp["x"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["B"]),
                             dev(inp["C"]), h0=dev(inp["h0"]), return_last_state=True)
    assert y.shape == (2, 0, 3, 64)
    assert torch.equal(hl.cpu(), torch.from_numpy(inp["h0"]))


def test_ssd_deterministic():
    inp = gen.make_ssd_inputs(2, 300, 8, 64, 128, "bf16", 9, with_h0=True)
    y1, h1 = run(inp)
    y2, h2 = run(inp)
    assert torch.equal(y1, y2) and torch.equal(h1, h2)


def test_ssd_split_sequence_carries_the_state():
    """Two calls (first 96 steps, then the rest from the returned state) match
    one call over the whole sequence."""
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd
    inp = gen.make_ssd_inputs(1, 200, 2, 64, 128, "bf16", 21, with_h0=True)
    d = {k: dev(v) for k, v in inp.items()}
    y, hl = ssm_ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                             dt_bias=d["dt_bias"], h0=d["h0"], return_last_state=True)
    cut = lambda t, a, b: t[:, a:b].contiguous()  # noqa: E731
    y1, h1 = ssm_ssd_scan_fwd(cut(d["x"], 0, 96), cut(d["dt"], 0, 96), d["A"],
                              cut(d["B"], 0, 96), cut(d["C"], 0, 96), D=d["D"],
                              dt_bias=d["dt_bias"], h0=d["h0"], return_last_state=True)
    y2, h2 = ssm_ssd_scan_fwd(cut(d["x"], 96, 200), cut(d["dt"], 96, 200), d["A"],
                              cut(d["B"], 96, 200), cut(d["C"], 96, 200), D=d["D"],
                              dt_bias=d["dt_bias"], h0=h1, return_last_state=True)
    assert torch.equal(torch.cat([y1, y2], dim=1), y) and torch.equal(h2, hl)

"""GPU parity of the multi-head SSD scan (Mamba-2, tensor-core chunked form,
through the C ABI) and of its decode step against the fp64 oracle's
sequential per-head loop.

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


@pytest.mark.parametrize("legacy", [False, True])
def test_ssd_split_sequence_carries_the_state(monkeypatch, legacy):
    """Two calls (the first steps, then the rest from the returned state)
    against one call over the whole sequence. Split at a multiple of the
    kernels' chunk lengths (128 steps for the tcgen05 kernel, 32 for the
    warp-level one) the chunks and their arithmetic are the same, so the
    results are bit for bit equal; split anywhere else (96) the chunks group
    the steps differently, and both calls together still match the oracle's
    sequential loop within the bound."""
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd
    if legacy:
        monkeypatch.setenv("SSM_SSD_LEGACY", "1")
    else:
        monkeypatch.delenv("SSM_SSD_LEGACY", raising=False)
    inp = gen.make_ssd_inputs(1, 300, 2, 64, 128, "bf16", 21, with_h0=True)
    d = {k: dev(v) for k, v in inp.items()}
    y, hl = ssm_ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                             dt_bias=d["dt_bias"], h0=d["h0"], return_last_state=True)
    yr, hr = reference(inp)
    cut = lambda t, a, b: t[:, a:b].contiguous()  # noqa: E731
    for k in (128, 96):
        y1, h1 = ssm_ssd_scan_fwd(cut(d["x"], 0, k), cut(d["dt"], 0, k), d["A"],
                                  cut(d["B"], 0, k), cut(d["C"], 0, k), D=d["D"],
                                  dt_bias=d["dt_bias"], h0=d["h0"], return_last_state=True)
        y2, h2 = ssm_ssd_scan_fwd(cut(d["x"], k, 300), cut(d["dt"], k, 300), d["A"],
                                  cut(d["B"], k, 300), cut(d["C"], k, 300), D=d["D"],
                                  dt_bias=d["dt_bias"], h0=h1, return_last_state=True)
        ys = torch.cat([y1, y2], dim=1)
        if k == 128 or legacy:
            assert torch.equal(ys, y) and torch.equal(h2, hl), f"split at {k}"
        assert rel_err(host(ys), yr) <= TOL and rel_err(host(h2), hr) <= TOL, f"split at {k}"


# ---- decode step (fp32 state in HBM; fp32 arithmetic: 1e-5 for fp32 io, 1e-2 bf16)
DTOL = {"f32": 1e-5, "bf16": 1e-2}


def decode_inputs(batch, H, P, N, io, seed, step):
    return gen.make_ssd_decode_inputs(batch, H, P, N, io, seed, step)


@pytest.mark.parametrize("N", [32, 64, 128, 256])
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("optional", [True, False])
def test_ssd_decode_shapes(N, io, optional):
    """Odd head counts and widths (3 x 5 heads of 7), 10 carried steps."""
    from selective_state_space_39_b200 import ssm_ssd_state_update
    batch, H, P = 3, 5, 7
    seed = N + (3 if optional else 0)
    const = gen.ssd_constants(H, seed)
    rng = np.random.default_rng(seed)
    state = torch.from_numpy(rng.standard_normal((batch, H, P, N)).astype(np.float32)).cuda()
    ref = host(state).copy()
    kw = dict(D=const["D"], dt_bias=const["dt_bias"]) if optional else {}
    for step in range(10):
        inp = decode_inputs(batch, H, P, N, io, seed, step)
        y = ssm_ssd_state_update(state, dev(inp["x"]), dev(inp["dt"]), dev(const["A"]),
                                 dev(inp["B"]), dev(inp["C"]),
                                 **{k: dev(v) for k, v in kw.items()})
        yr = oracle.ssd_state_update(ref, inp["x"], inp["dt"], const["A"], inp["B"], inp["C"],
                                     io=io, **kw)
        assert rel_err(host(y), yr) <= DTOL[io], f"step {step}"
    assert rel_err(host(state), ref) <= DTOL[io]


def test_ssd_decode_workload_sampled():
    """64 sequences x 64 heads x 64, d_state 128, bf16, 1000 carried steps; the
    oracle runs the same steps on sampled sequences and heads."""
    from selective_state_space_39_b200 import ssm_ssd_state_update
    w = gen.SSD_DECODE_WORKLOADS["ssd_decode_b64_h64_p64_n128_x1000"]
    const = gen.ssd_constants(w.nheads, w.seed)
    A, D, bias = dev(const["A"]), dev(const["D"]), dev(const["dt_bias"])
    state = torch.zeros((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                        device="cuda")
    bs, hs = np.array([0, 1, 31, 63]), np.array([0, 5, 32, 63])
    ref = np.zeros((len(bs), len(hs), w.headdim, w.dstate))
    sub = lambda a: np.ascontiguousarray(a[bs][:, hs])  # noqa: E731
    ys, yrs = [], []
    for step in range(w.steps):
        inp = decode_inputs(w.batch, w.nheads, w.headdim, w.dstate, w.io, w.seed, step)
        y = ssm_ssd_state_update(state, dev(inp["x"]), dev(inp["dt"]), A, dev(inp["B"]),
                                 dev(inp["C"]), D=D, dt_bias=bias)
        if step % 50 == 49 or step < 3:
            ys.append(host(y)[bs][:, hs])
        yr = oracle.ssd_state_update(ref, sub(inp["x"]), sub(inp["dt"]),
                                     np.ascontiguousarray(const["A"][hs]),
                                     np.ascontiguousarray(inp["B"][bs]),
                                     np.ascontiguousarray(inp["C"][bs]), D=const["D"][hs],
                                     dt_bias=const["dt_bias"][hs], io=w.io)
        if step % 50 == 49 or step < 3:
            yrs.append(yr)
    ey = rel_err(np.stack(ys), np.stack(yrs))
    eh = rel_err(host(state)[bs][:, hs], ref)
    print(f"ssd decode 1000 steps: rel err y {ey:.3e} state {eh:.3e}")
    assert torch.isfinite(state).all()
    assert ey <= DTOL["bf16"] and eh <= DTOL["bf16"]


def test_ssd_decode_steps_equal_the_scan():
    """L decode steps on the GPU match the GPU's chunked SSD scan over the same
    tokens (bf16; the scan's tensor-core operands set the bound)."""
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd, ssm_ssd_state_update
    inp = gen.make_ssd_inputs(2, 70, 3, 64, 128, "bf16", 23, with_h0=True)
    d = {k: dev(v) for k, v in inp.items()}
    y, hl = ssm_ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                             dt_bias=d["dt_bias"], h0=d["h0"], return_last_state=True)
    state = d["h0"].clone()
    yd = []
    for t in range(70):
        col = lambda k: dev(np.ascontiguousarray(inp[k][:, t]))  # noqa: E731
        yd.append(ssm_ssd_state_update(state, col("x"), col("dt"), d["A"], col("B"), col("C"),
                                       D=d["D"], dt_bias=d["dt_bias"]))
    assert rel_err(host(torch.stack(yd, dim=1)), host(y)) <= TOL
    assert rel_err(host(state), host(hl)) <= TOL



def test_ssd_empty_batch_and_heads():
    """batch = 0 or heads = 0: nothing to compute, the calls succeed."""
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd, ssm_ssd_state_update
    for batch, H in ((0, 3), (2, 0)):
        inp = gen.make_ssd_inputs(batch, 16, H, 64, 64, "bf16", 3)
        y = ssm_ssd_scan_fwd(dev(inp["x"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["B"]),
                             dev(inp["C"]))
        assert y.shape == (batch, 16, H, 64)
        d = gen.make_ssd_decode_inputs(batch, H, 64, 64, "bf16", 3, 0)
        state = torch.zeros((batch, H, 64, 64), dtype=torch.float32, device="cuda")
        yd = ssm_ssd_state_update(state, dev(d["x"]), dev(d["dt"]), dev(inp["A"]), dev(d["B"]),
                                  dev(d["C"]))
        assert yd.shape == (batch, H, 64)


# ------------------------------------------- the tcgen05 path (state in TMEM)
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("L", [1, 127, 128, 129, 300])
def test_ssd_tcgen05_matches_oracle_and_legacy(monkeypatch, N, L):
    """Even head counts with dstate 64 / 128 take the tcgen05 kernel (128-step
    chunks, state in tensor memory); SSM_SSD_LEGACY=1 the warp-level MMA one.
    Lengths around the chunk size: one step, a ragged single chunk, exactly
    one chunk, one step past it, and two chunks plus a ragged one."""
    inp = gen.make_ssd_inputs(2, L, 4, 64, N, "bf16", 300 + N + L, with_h0=True)
    yr, hr = reference(inp)
    monkeypatch.delenv("SSM_SSD_LEGACY", raising=False)
    y, hl = run(inp)
    monkeypatch.setenv("SSM_SSD_LEGACY", "1")
    y2, hl2 = run(inp)
    for what, (a, b) in {"tcgen05": (y, hl), "legacy": (y2, hl2)}.items():
        ey, eh = rel_err(host(a), yr), rel_err(host(b), hr)
        print(f"{what} N={N} L={L}: y {ey:.3e} h_last {eh:.3e}")
        assert torch.isfinite(a.float()).all() and torch.isfinite(b).all()
        assert ey <= TOL and eh <= TOL, f"{what} N={N} L={L}"


def test_ssd_tcgen05_in_place_state_and_no_h_last(monkeypatch):
    """h_last may be h0 itself (each CTA reads its heads' state before it
    writes them); without h_last only y is written."""
    monkeypatch.delenv("SSM_SSD_LEGACY", raising=False)
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd
    inp = gen.make_ssd_inputs(2, 200, 6, 64, 128, "bf16", 311, with_h0=True)
    yr, hr = reference(inp)
    h = dev(inp["h0"]).clone()
    y, hl = ssm_ssd_scan_fwd(dev(inp["x"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["B"]),
                             dev(inp["C"]), D=dev(inp["D"]), dt_bias=dev(inp["dt_bias"]), h0=h,
                             h_last=h, return_last_state=True)
    assert hl.data_ptr() == h.data_ptr()
    assert rel_err(host(y), yr) <= TOL and rel_err(host(hl), hr) <= TOL
    y3 = run(inp, last=False)
    assert rel_err(host(y3), yr) <= TOL


def test_ssd_tcgen05_timeout_is_reported(monkeypatch):
    """One CTA waits for 16 bytes that no copy delivers (test hook): its
    bounded wait runs out, it frees its tensor memory, ssm_ssd_scan_status
    reports the timeout once, and the next call is correct."""
    from selective_state_space_39_b200 import ssm_ssd_scan_status
    monkeypatch.delenv("SSM_SSD_LEGACY", raising=False)
    inp = gen.make_ssd_inputs(1, 256, 4, 64, 128, "bf16", 313, with_h0=True)
    assert ssm_ssd_scan_status() == 0
    monkeypatch.setenv("SSM_SSD_TEST_STALL", "1")
    monkeypatch.setenv("SSM_SCAN_WAIT_LIMIT_NS", "20000000")  # 20 ms
    run(inp)
    assert ssm_ssd_scan_status() == -5
    assert ssm_ssd_scan_status() == 0  # the flag is cleared
    monkeypatch.delenv("SSM_SSD_TEST_STALL")
    monkeypatch.delenv("SSM_SCAN_WAIT_LIMIT_NS")
    y, hl = run(inp)
    assert ssm_ssd_scan_status() == 0
    yr, hr = reference(inp)
    assert rel_err(host(y), yr) <= TOL and rel_err(host(hl), hr) <= TOL

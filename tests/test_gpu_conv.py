"""GPU parity of the block's causal depthwise conv1d + SiLU (forward and
backward, through the C ABI) against the fp64 oracle.

Bound: max|g - g_ref| / max|g_ref| <= 1e-5 for fp32 io (1e-4 for dw and
dbias, sums over batch x seqlen terms) and 1e-2 for bf16 io (outputs rounded
to bf16, 2^-9 relative; MUFU tanh for the sigmoid)."""
import numpy as np
import pytest
import torch

import ssm_inputs as gen
from tests.gpu_util import dev, host, rel_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 1e-2}
TOL_SUM = {"f32": 1e-4, "bf16": 1e-2}


def run_fwd(c, silu=True, bias=True):
    from selective_state_space_39_b200 import ssm_conv1d_silu_fwd
    return ssm_conv1d_silu_fwd(dev(c["x"]), dev(c["w"]), dev(c["bias"]) if bias else None,
                               silu=silu)


def run_bwd(c, silu=True, bias=True):
    from selective_state_space_39_b200 import ssm_conv1d_silu_bwd
    return ssm_conv1d_silu_bwd(dev(c["x"]), dev(c["w"]), dev(c["dout"]),
                               dev(c["bias"]) if bias else None, silu=silu)


def check(c, io, silu=True, bias=True, what=""):
    import oracle
    b = c["bias"] if bias else None
    out = run_fwd(c, silu, bias)
    ref = oracle.conv1d_silu(c["x"], c["w"], b, silu=silu, io=io)
    e = rel_err(host(out), ref)
    print(f"{what}: out rel err {e:.3e}")
    assert np.all(np.isfinite(host(out))) and e <= TOL[io], f"{what}: out {e:.3e}"
    g = run_bwd(c, silu, bias)
    dx, dw, db = oracle.conv1d_silu_bwd(c["x"], c["w"], c["dout"], b, silu=silu, io=io)
    for name, got, want, tol in (("dx", g["dx"], dx, TOL[io]), ("dw", g["dw"], dw, TOL_SUM[io]),
                                 ("dbias", g["dbias"], db, TOL_SUM[io])):
        e = rel_err(host(got), want)
        print(f"{what}: {name} rel err {e:.3e}")
        assert e <= tol, f"{what}: {name} rel err {e:.3e} > {tol}"


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("width", [2, 3, 4])
@pytest.mark.parametrize("shape", [(2, 70, 256), (2, 45, 150), (1, 5, 24), (3, 96, 1032)],
                         ids=["vec", "ragged", "short", "odd_blocks"])
def test_conv_shapes(io, width, shape):
    """Vector path (dim a multiple of 4), element path (dim 150), a sequence
    shorter than the 4-step window, and a chunk count that is not a multiple
    of anything (L = 96, dim 1032 = 258 vectors)."""
    c = gen.make_conv_inputs(*shape, width, io, 3)
    check(c, io, what=f"{io} w={width} {shape}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("silu,bias", [(False, True), (True, False), (False, False)])
def test_conv_optional_terms(io, silu, bias):
    c = gen.make_conv_inputs(2, 40, 64, 4, io, 5)
    check(c, io, silu=silu, bias=bias, what=f"{io} silu={silu} bias={bias}")


def test_conv_mamba130m_layer_full():
    """The 8 x 2048 x 1536 bf16 layer's conv, every output and gradient."""
    c = gen.make_conv_inputs(8, 2048, 1536, 4, "bf16", 1)
    check(c, "bf16", what="8x2048x1536")


def test_conv_vector_and_element_paths_agree():
    """The 8-byte vector path and the one-element path compute the same
    numbers bit for bit (same per-element arithmetic, same summation order)."""
    from selective_state_space_39_b200 import ssm_conv1d_silu_bwd, ssm_conv1d_silu_fwd
    c = gen.make_conv_inputs(2, 100, 256, 4, "bf16", 9)
    x, w, b, g = dev(c["x"]), dev(c["w"]), dev(c["bias"]), dev(c["dout"])
    out_v = ssm_conv1d_silu_fwd(x, w, b)
    gv = ssm_conv1d_silu_bwd(x, w, g, b)
    # an offset view breaks the 8-byte alignment: the element path runs
    xs = torch.empty(x.numel() + 1, dtype=x.dtype, device=x.device)[1:].view(x.shape)
    gs = torch.empty(g.numel() + 1, dtype=g.dtype, device=g.device)[1:].view(g.shape)
    xs.copy_(x)
    gs.copy_(g)
    out_s = ssm_conv1d_silu_fwd(xs, w, b)
    gsr = ssm_conv1d_silu_bwd(xs, w, gs, b)
    assert torch.equal(out_v, out_s)
    for k in ("dx", "dw", "dbias"):
        assert torch.equal(gv[k], gsr[k]), k


def test_conv_bwd_deterministic():
    c = gen.make_conv_inputs(4, 300, 512, 4, "bf16", 11)
    g1, g2 = run_bwd(c), run_bwd(c)
    for k in ("dx", "dw", "dbias"):
        assert torch.equal(g1[k], g2[k]), k


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("width", [2, 3, 4])
def test_conv_update_steps_match_oracle(io, width):
    """Decode steps of the conv (rolling state) against the oracle's steps,
    and against the GPU's own conv over the same tokens."""
    import oracle
    from selective_state_space_39_b200 import ssm_conv1d_silu_fwd, ssm_conv1d_silu_update
    c = gen.make_conv_inputs(3, 9, 130, width, io, 13)
    st = torch.zeros((3, 130, width - 1), dtype=dev(c["x"]).dtype, device="cuda")
    ref = np.zeros((3, 130, width - 1))
    full = host(ssm_conv1d_silu_fwd(dev(c["x"]), dev(c["w"]), dev(c["bias"])))
    for t in range(9):
        xt = np.ascontiguousarray(c["x"][:, t])
        out = host(ssm_conv1d_silu_update(st, dev(xt), dev(c["w"]), dev(c["bias"])))
        want = oracle.conv1d_silu_update(ref, xt, c["w"], c["bias"], io=io)
        assert rel_err(out, want) <= TOL[io], f"step {t}"
        assert rel_err(out, full[:, t]) <= TOL[io], f"step {t} vs the conv"


def test_conv_empty_sequence():
    """L = 0: the forward writes nothing, the backward returns zero dw and
    dbias (sums over no steps)."""
    from selective_state_space_39_b200 import ssm_conv1d_silu_bwd, ssm_conv1d_silu_fwd
    c = gen.make_conv_inputs(2, 0, 64, 4, "bf16", 21)
    out = ssm_conv1d_silu_fwd(dev(c["x"]), dev(c["w"]), dev(c["bias"]))
    assert out.shape == (2, 0, 64)
    g = ssm_conv1d_silu_bwd(dev(c["x"]), dev(c["w"]), dev(c["dout"]), dev(c["bias"]))
    assert g["dx"].shape == (2, 0, 64)
    assert torch.count_nonzero(g["dw"]) == 0 and torch.count_nonzero(g["dbias"]) == 0


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 2, 3])
@pytest.mark.parametrize("dim", [256, 150])
def test_conv_sequence_shorter_than_the_taps(io, L, dim):
    """L < width (4): every output sees the zero left padding; the weight
    gradient of the taps that never meet a token is zero. Vector and element
    paths."""
    c = gen.make_conv_inputs(2, L, dim, 4, io, 40 + L)
    check(c, io, what=f"{io} L={L} dim={dim}")


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_conv_zero_input_run(io):
    """x = 0 on a run of steps longer than the window (padding tokens): the
    outputs there are SiLU(bias) exactly, and the gradients flow around it."""
    c = gen.make_conv_inputs(2, 300, 256, 4, io, 47)
    x = (gen.bf16_bits_to_f32(c["x"]) if io == "bf16" else c["x"]).copy()
    x[:, 100:180] = 0.0
    c["x"] = gen.f32_to_bf16_bits(x) if io == "bf16" else x.astype(np.float32)
    check(c, io, what=f"{io} zero run")

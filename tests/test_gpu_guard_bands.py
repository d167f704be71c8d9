"""Guard bands: every output (and every state updated in place) is a view
into a larger buffer whose margins hold a sentinel; after the call the
margins must be untouched and the interior must match the oracle. This is
the bounds check used in place of a memory checker."""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as gen
from tests.gpu_util import TOL, dev, host, rel_err

pytestmark = pytest.mark.gpu

PAD = 4096      # elements on each side (keeps 16-byte alignment)
SENTINEL = 7.0


def padded(shape, dtype, fill=None):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * PAD,), SENTINEL, dtype=dtype, device="cuda")
    view = buf[PAD:PAD + n].view(*shape)
    if fill is not None:
        view.copy_(fill)
    return buf, view


def margins_intact(buf):
    torch.cuda.synchronize()
    return bool(torch.all(buf[:PAD] == SENTINEL)) and bool(torch.all(buf[-PAD:] == SENTINEL))


def test_decode_step_stays_in_bounds():
    from selective_state_space_39_b200 import ssm_state_update
    batch, dim, N = 5, 390, 16
    const = gen.decode_constants(dim, N, 3)
    inp = gen.make_decode_inputs(batch, dim, N, "bf16", 3, 0)
    rng = np.random.default_rng(3)
    s0 = rng.standard_normal((batch, dim, N)).astype(np.float32)
    sbuf, state = padded((batch, dim, N), torch.float32, torch.from_numpy(s0))
    ybuf, y = padded((batch, dim), torch.bfloat16)
    ssm_state_update(state, dev(inp["x"]), dev(inp["delta"]), dev(const["A"]), dev(inp["B"]),
                     dev(inp["C"]), D=dev(const["D"]), z=dev(inp["z"]),
                     delta_bias=dev(const["delta_bias"]), y=y)
    assert margins_intact(sbuf) and margins_intact(ybuf)
    ref = s0.astype(np.float64)
    yr = oracle.state_update(ref, inp["x"], inp["delta"], const["A"], inp["B"], inp["C"],
                             D=const["D"], z=inp["z"], delta_bias=const["delta_bias"], io="bf16")
    assert rel_err(host(y), yr) <= TOL["bf16"] and rel_err(host(state), ref) <= TOL["bf16"]


@pytest.mark.parametrize("dim", [1032, 150], ids=["vector", "element"])
def test_conv_stays_in_bounds(dim):
    from selective_state_space_39_b200 import ssm_conv1d_silu_fwd, ssm_conv1d_silu_update
    c = gen.make_conv_inputs(2, 45, dim, 4, "bf16", 5)
    obuf, out = padded((2, 45, dim), torch.bfloat16)
    ssm_conv1d_silu_fwd(dev(c["x"]), dev(c["w"]), dev(c["bias"]), out=out)
    assert margins_intact(obuf)
    assert rel_err(host(out), oracle.conv1d_silu(c["x"], c["w"], c["bias"], io="bf16")) <= 1e-2
    # decode step: rolling state and output
    sbuf, st = padded((2, dim, 3), torch.bfloat16, torch.zeros(2, dim, 3))
    ubuf, u = padded((2, dim), torch.bfloat16)
    x0 = np.ascontiguousarray(c["x"][:, 0])
    ssm_conv1d_silu_update(st, dev(x0), dev(c["w"]), dev(c["bias"]), out=u)
    assert margins_intact(sbuf) and margins_intact(ubuf)
    want = oracle.conv1d_silu_update(np.zeros((2, dim, 3)), x0, c["w"], c["bias"], io="bf16")
    assert rel_err(host(u), want) <= 1e-2


def test_ssd_scan_stays_in_bounds():
    from selective_state_space_39_b200 import ssm_ssd_scan_fwd
    inp = gen.make_ssd_inputs(2, 77, 3, 64, 128, "bf16", 11, with_h0=True)
    ybuf, y = padded((2, 77, 3, 64), torch.bfloat16)
    _, hl = ssm_ssd_scan_fwd(dev(inp["x"]), dev(inp["dt"]), dev(inp["A"]), dev(inp["B"]),
                             dev(inp["C"]), D=dev(inp["D"]), dt_bias=dev(inp["dt_bias"]),
                             h0=dev(inp["h0"]), return_last_state=True, y=y)
    assert margins_intact(ybuf)
    yr, hr = oracle.ssd_scan(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                             dt_bias=inp["dt_bias"], h0=inp["h0"], io="bf16")
    assert rel_err(host(y), yr) <= 1e-2 and rel_err(host(hl), hr) <= 1e-2


def test_ssd_decode_step_stays_in_bounds():
    from selective_state_space_39_b200 import ssm_ssd_state_update
    batch, H, P, N = 3, 5, 7, 64
    const = gen.ssd_constants(H, 13)
    inp = gen.make_ssd_decode_inputs(batch, H, P, N, "f32", 13, 0)
    rng = np.random.default_rng(13)
    s0 = rng.standard_normal((batch, H, P, N)).astype(np.float32)
    sbuf, state = padded((batch, H, P, N), torch.float32, torch.from_numpy(s0))
    ybuf, y = padded((batch, H, P), torch.float32)
    ssm_ssd_state_update(state, dev(inp["x"]), dev(inp["dt"]), dev(const["A"]), dev(inp["B"]),
                         dev(inp["C"]), D=dev(const["D"]), dt_bias=dev(const["dt_bias"]), y=y)
    assert margins_intact(sbuf) and margins_intact(ybuf)
    ref = s0.astype(np.float64)
    yr = oracle.ssd_state_update(ref, inp["x"], inp["dt"], const["A"], inp["B"], inp["C"],
                                 D=const["D"], dt_bias=const["dt_bias"], io="f32")
    assert rel_err(host(y), yr) <= TOL["f32"] and rel_err(host(state), ref) <= TOL["f32"]

"""ssm_scan_fwd_noalloc, the entry point for callers that cannot allocate
device memory (it takes its scratch from an array the library reserves on
each GPU). Checked through the C ABI against ssm_scan_fwd, which uses a
caller-provided workspace, on two calls in a row that share the reserved
scratch. This file is collected last on purpose."""
import pytest
import torch

import ssm_inputs as gen
from tests.gpu_util import TOL, dev, host, rel_err

pytestmark = pytest.mark.gpu


def _both(inp, io):
    from selective_state_space_39_b200 import ssm_scan_fwd, ssm_scan_fwd_noalloc
    args = (dev(inp["x"]), dev(inp["delta"]), dev(inp["A"]), dev(inp["B"]), dev(inp["C"]))
    kw = dict(D=dev(inp["D"]), z=dev(inp["z"]), delta_bias=dev(inp["delta_bias"]),
              h0=dev(inp["h0"]))
    y_ref, h_ref = ssm_scan_fwd(*args, **kw)
    y, h = ssm_scan_fwd_noalloc(*args, **kw)
    torch.cuda.synchronize()
    return y, h, y_ref, h_ref


def test_noalloc_matches_workspace_entry_on_consecutive_calls(monkeypatch):
    monkeypatch.delenv("SSM_SCAN_SEGMENTS", raising=False)
    monkeypatch.delenv("SSM_SCAN_CTAS_PER_SM", raising=False)
    first = gen.make_scan_inputs(3, 700, 1024, 16, "bf16", 101, with_h0=True)
    second = gen.make_scan_inputs(2, 1500, 768, 16, "bf16", 202, with_h0=False)
    for inp, io in ((first, "bf16"), (second, "bf16")):
        y, h, y_ref, h_ref = _both(inp, io)
        assert rel_err(host(y), host(y_ref)) <= TOL[io]
        assert rel_err(host(h), host(h_ref)) <= TOL[io]


def test_noalloc_multisegment_fp32_twice(monkeypatch):
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", "5")
    inp = gen.make_scan_inputs(2, 333, 300, 16, "f32", 303, with_h0=True)
    for _ in range(2):
        y, h, y_ref, h_ref = _both(inp, "f32")
        assert rel_err(host(y), host(y_ref)) <= TOL["f32"]
        assert rel_err(host(h), host(h_ref)) <= TOL["f32"]


def test_noalloc_rejects_problems_beyond_its_scratch(monkeypatch):
    from selective_state_space_39_b200 import SsmError, scan_workspace_bytes, ssm_scan_fwd_noalloc
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", "64")
    batch, L, dim, N = 8, 4096, 2048, 16
    assert scan_workspace_bytes(batch, L, dim, N, torch.bfloat16) > (8 << 20)
    x = torch.zeros((batch, L, dim), dtype=torch.bfloat16, device="cuda")
    bc = torch.zeros((batch, L, N), dtype=torch.bfloat16, device="cuda")
    A = -torch.ones((dim, N), dtype=torch.float32, device="cuda")
    with pytest.raises(SsmError, match="scratch"):
        ssm_scan_fwd_noalloc(x, x, A, bc, bc)

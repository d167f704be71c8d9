"""Failure detection on the GPU without a fault: a bounded wait inside the
scan kernel is made to run out (one CTA waits for 16 bytes that no copy
delivers), the kernel reports a timeout through the workspace status, and
the context stays usable for the next call."""
import pytest
import torch

import ssm_inputs as gen
from tests.gpu_util import TOL, gpu_scan, host, oracle_scan, rel_err

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(monkeypatch):
    from selective_state_space_39_b200 import scan_workspace_bytes, ssm_scan_status
    inp = gen.make_scan_inputs(2, 200, 512, 16, "bf16", 41, with_h0=True)
    dims = (2, 200, 512, 16)
    ws = torch.empty(scan_workspace_bytes(*dims, torch.bfloat16), dtype=torch.uint8, device="cuda")
    monkeypatch.setenv("SSM_SCAN_TEST_STALL", "1")
    monkeypatch.setenv("SSM_SCAN_WAIT_LIMIT_NS", "20000000")  # 20 ms
    gpu_scan(inp, workspace=ws)
    assert ssm_scan_status(ws, *dims, torch.bfloat16) == -5
    monkeypatch.delenv("SSM_SCAN_TEST_STALL")
    monkeypatch.delenv("SSM_SCAN_WAIT_LIMIT_NS")
    y, hl = gpu_scan(inp, workspace=ws)
    assert ssm_scan_status(ws, *dims, torch.bfloat16) == 0
    yr, hr = oracle_scan(inp, "bf16")
    assert rel_err(host(y), yr) <= TOL["bf16"] and rel_err(host(hl), hr) <= TOL["bf16"]

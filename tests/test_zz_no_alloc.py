"""ssm_scan_fwd_noalloc, the entry point for callers that cannot allocate
device memory (it takes its scratch from an array the library reserves on
each GPU), through the C ABI:

  * against ssm_scan_fwd, which uses a caller-provided workspace, on two
    calls in a row that share the reserved scratch;
  * against the fp64 oracle, on the tiny fp32 workload in full and on the
    8 x 2048 x 1536 bf16 layer on sampled channels;
  * a bounded wait made to run out inside a no-alloc call is reported by
    ssm_scan_status_noalloc, and the next call succeeds.

This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import ssm_inputs as gen
from tests.gpu_util import TOL, dev, host, oracle_scan, rel_err, sample_channels

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_env(monkeypatch):
    for k in ("SSM_SCAN_SEGMENTS", "SSM_SCAN_DISABLE_TMA", "SSM_SCAN_CTAS_PER_SM",
              "SSM_SCAN_WAIT_LIMIT_NS", "SSM_SCAN_TEST_STALL"):
        monkeypatch.delenv(k, raising=False)
    yield


def _args(inp):
    args = (dev(inp["x"]), dev(inp["delta"]), dev(inp["A"]), dev(inp["B"]), dev(inp["C"]))
    kw = dict(D=dev(inp["D"]), z=dev(inp["z"]), delta_bias=dev(inp["delta_bias"]),
              h0=dev(inp["h0"]))
    return args, kw


def _both(inp):
    from selective_state_space_39_b200 import ssm_scan_fwd, ssm_scan_fwd_noalloc
    args, kw = _args(inp)
    y_ref, h_ref = ssm_scan_fwd(*args, **kw)
    y, h = ssm_scan_fwd_noalloc(*args, **kw)
    torch.cuda.synchronize()
    return y, h, y_ref, h_ref


def test_noalloc_matches_workspace_entry_on_consecutive_calls():
    first = gen.make_scan_inputs(3, 700, 1024, 16, "bf16", 101, with_h0=True)
    second = gen.make_scan_inputs(2, 1500, 768, 16, "bf16", 202, with_h0=False)
    for inp, io in ((first, "bf16"), (second, "bf16")):
        y, h, y_ref, h_ref = _both(inp)
        assert rel_err(host(y), host(y_ref)) <= TOL[io]
        assert rel_err(host(h), host(h_ref)) <= TOL[io]


def test_noalloc_multisegment_fp32_twice(monkeypatch):
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", "5")
    inp = gen.make_scan_inputs(2, 333, 300, 16, "f32", 303, with_h0=True)
    for _ in range(2):
        y, h, y_ref, h_ref = _both(inp)
        assert rel_err(host(y), host(y_ref)) <= TOL["f32"]
        assert rel_err(host(h), host(h_ref)) <= TOL["f32"]


def test_noalloc_matches_oracle_tiny_f32():
    """The 1 x 256 x 64 fp32 workload in full, twice in a row."""
    from selective_state_space_39_b200 import ssm_scan_fwd_noalloc
    inp = gen.workload_inputs(gen.SCAN_WORKLOADS["tiny_f32_b1_l256_d64"])
    yr, hr = oracle_scan(inp, "f32")
    args, kw = _args(inp)
    for _ in range(2):
        y, h = ssm_scan_fwd_noalloc(*args, **kw)
        assert rel_err(host(y), yr) <= TOL["f32"]
        assert rel_err(host(h), hr) <= TOL["f32"]


def test_noalloc_matches_oracle_mamba130m_sampled():
    """The 8 x 2048 x 1536 bf16 layer (the bench workload) in the library's
    own split, every step of sampled channels against the oracle."""
    from selective_state_space_39_b200 import scan_workspace_bytes, ssm_scan_fwd_noalloc
    w = gen.SCAN_WORKLOADS["mamba130m_layer_b8_l2048_d1536"]
    assert scan_workspace_bytes(w.batch, w.seqlen, w.dim, w.dstate, torch.bfloat16) <= 16 << 20
    inp = gen.workload_inputs(w)
    args, kw = _args(inp)
    y, h = ssm_scan_fwd_noalloc(*args, **kw)
    chans = sample_channels(w.batch, w.dim, 10)
    yr, hr = oracle_scan(inp, w.io, channels=chans)
    yg, hg = host(y), host(h)
    ys = np.stack([yg[b, :, d] for b, d in chans])
    hs = np.stack([hg[b, d] for b, d in chans])
    assert rel_err(ys, yr) <= TOL[w.io] and rel_err(hs, hr) <= TOL[w.io]


def test_noalloc_timeout_is_reported(monkeypatch):
    """One CTA waits for 16 bytes that no copy delivers (test hook): its
    bounded wait runs out, the status words in the reserved scratch say so,
    and the next call on the same context is correct."""
    from selective_state_space_39_b200 import ssm_scan_fwd_noalloc, ssm_scan_status_noalloc
    inp = gen.make_scan_inputs(2, 200, 512, 16, "bf16", 41, with_h0=True)
    args, kw = _args(inp)
    monkeypatch.setenv("SSM_SCAN_TEST_STALL", "1")
    monkeypatch.setenv("SSM_SCAN_WAIT_LIMIT_NS", "20000000")  # 20 ms
    ssm_scan_fwd_noalloc(*args, **kw)
    assert ssm_scan_status_noalloc(2, 200, 512, 16, torch.bfloat16) == -5
    monkeypatch.delenv("SSM_SCAN_TEST_STALL")
    monkeypatch.delenv("SSM_SCAN_WAIT_LIMIT_NS")
    y, h = ssm_scan_fwd_noalloc(*args, **kw)
    assert ssm_scan_status_noalloc(2, 200, 512, 16, torch.bfloat16) == 0
    yr, hr = oracle_scan(inp, "bf16")
    assert rel_err(host(y), yr) <= TOL["bf16"] and rel_err(host(h), hr) <= TOL["bf16"]


def test_noalloc_rejects_problems_beyond_its_scratch(monkeypatch):
    from selective_state_space_39_b200 import (SsmError, scan_workspace_bytes,
                                               ssm_scan_fwd_noalloc, ssm_scan_status_noalloc)
    monkeypatch.setenv("SSM_SCAN_SEGMENTS", "64")
    batch, L, dim, N = 8, 4096, 2048, 16
    assert scan_workspace_bytes(batch, L, dim, N, torch.bfloat16) > (16 << 20)
    x = torch.zeros((batch, L, dim), dtype=torch.bfloat16, device="cuda")
    bc = torch.zeros((batch, L, N), dtype=torch.bfloat16, device="cuda")
    A = -torch.ones((dim, N), dtype=torch.float32, device="cuda")
    with pytest.raises(SsmError, match="scratch"):
        ssm_scan_fwd_noalloc(x, x, A, bc, bc)
    assert ssm_scan_status_noalloc(batch, L, dim, N, torch.bfloat16) == -3

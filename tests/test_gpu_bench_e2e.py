"""GPU check of the bench's end-to-end step: pinned host inputs copied in by
batch-row chunks, the scan run on each chunk as it lands, and the results
copied back chunk by chunk, must give the oracle's y and h_last on every row,
with a ragged chunk split (5 rows in 3 chunks) and with one chunk."""
import os
import sys

import numpy as np
import pytest
import torch

import ssm_inputs as gen
from tests.gpu_util import TOL, host, oracle_scan, rel_err

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io,nch", [("bf16", 3), ("f32", 1), ("f32", 5)])
def test_pipelined_host_step_matches_oracle(io, nch):
    w = gen.ScanWorkload(f"e2e_{io}_b5_l512_d128", 5, 512, 128, 16, io, 11, with_h0=True)
    device = torch.device("cuda", 0)
    run = bench.time_scan(w, w.batch, 0, device, K=1, warmup=3)
    inp, d, y, h_last = run["inp"], run["d"], run["y"], run["h_last"]
    dtype = y.dtype
    pinned = {k: (torch.from_numpy(v.view(np.int16) if v.dtype == np.uint16 else v)
                  .view(dtype if v.dtype == np.uint16 else torch.float32).pin_memory()
                  if v is not None else None) for k, v in inp.items()}
    # the device copies of the batched inputs and the outputs start as garbage,
    # so every row the host gets back was copied in and scanned by this step
    for k in bench.SCAN_BATCHED_INPUTS:
        if d.get(k) is not None:
            d[k].fill_(float("nan"))
    y.fill_(float("nan"))
    h_last.fill_(float("nan"))
    y_host = torch.full(y.shape, float("nan"), dtype=dtype).pin_memory()
    h_host = torch.full(h_last.shape, float("nan"), dtype=torch.float32).pin_memory()
    streams = (torch.cuda.Stream(device), torch.cuda.Stream(device))
    bench.pipelined_host_step(pinned, d, y, h_last, y_host, h_host, run["step_rows"],
                              w.batch, nch, streams)
    torch.cuda.current_stream(device).synchronize()
    yr, hr = oracle_scan(inp, io)
    yg, hg = host(y_host), host(h_host)
    assert np.all(np.isfinite(yg)) and np.all(np.isfinite(hg))
    for b in range(w.batch):
        ey, eh = rel_err(yg[b], yr[b]), rel_err(hg[b], hr[b])
        assert ey <= TOL[io], f"row {b}: y rel err {ey:.3e}"
        assert eh <= TOL[io], f"row {b}: h_last rel err {eh:.3e}"

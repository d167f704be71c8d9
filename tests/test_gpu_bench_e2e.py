"""GPU check of the bench's end-to-end step: pinned host inputs copied in by
batch-row chunks, the scan run on each chunk as it lands, and the results
copied back chunk by chunk, must give the oracle's y and h_last on every row,
with a ragged chunk split (5 rows in 3 chunks) and with one chunk; and the
bench's JSON line on one GPU keeps its contract."""
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


def test_bench_line_contract():
    """`python bench.py` on one GPU prints one JSON line with the keys the
    driver reads, and its figures agree with each other: value from the
    elements and ms_per_step, the roofline fraction from achieved / peak and
    the algorithmic bytes, the end-to-end bytes from the tensors copied."""
    import json
    import subprocess

    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "5",
                          "--warmup", "3", "--no-per-config", "--no-cpu-baseline",
                          "--e2e-steps", "2"], cwd=ROOT, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in j, k
    w = gen.SCAN_WORKLOADS[j["config"]["workload"]]
    assert j["n_gpus"] == 1 and j["steps"] == 5 and j["warmup"] >= 3
    assert j["higher_is_better"] is True and j["scaling"] == "weak"
    assert abs(j["value"] - w.elements / (j["ms_per_step"] * 1e-3)) <= 1e-6 * j["value"]
    r = j["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["algorithmic_bytes_per_launch"] == bench.algorithmic_bytes(w, w.batch)
    assert abs(r["frac"] - r["achieved"] / r["peak"]) <= 1e-3
    assert 0 < r["frac"] < 1.2
    e = j["e2e"]
    es = 2 if w.io == "bf16" else 4
    per_row_in = w.seqlen * (w.dim * es * (3 if w.gate else 2) + 2 * w.dstate * es)
    assert e["h2d_bytes_per_step"] >= w.batch * per_row_in
    assert e["d2h_bytes_per_step"] == w.batch * (w.seqlen * w.dim * es + w.dim * w.dstate * 4)
    assert 0 < e["value"] < j["value"]
    assert j["gpu_launches"] >= 5
    c = j["clocks"]
    assert "sm_mhz" in c and "sm_max_mhz" in c and "reasons" in c

"""Host-side parts of bench.py (no GPU): the algorithmic byte and FLOP counts
the roofline fractions divide by, and the reference arm's JSON line for
every workload family (the fp64 oracle on the host, a few small steps)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import ssm_inputs as gen  # noqa: E402


def test_scan_algorithmic_bytes():
    """x, delta, z read and y written in bf16 (8 B per element), B and C per
    (b, t), h_last (+ h0) per (b, d), A, bias and D once: the counts the HBM
    fractions of the scan use."""
    want = {"tiny_f32_b1_l256_d64": 303_616,
            "mamba130m_layer_b8_l2048_d1536": 203_272_192,
            "pythia1b_layer_b4_l4096_d4096_h0": 540_311_552,
            "long_b1_l262144_d1536": 3_238_211_584}
    for name, n in want.items():
        w = gen.SCAN_WORKLOADS[name]
        assert bench.algorithmic_bytes(w, w.batch) == n, name


def test_ssd_cost():
    """SSD: x read and y written (bf16), B, C, dt, h0 and h_last; products of
    the chunked dual form (Q = 32): Q P + 4 N P per (b, t, h) and Q N per
    (b, t)."""
    w = gen.SSD_WORKLOADS["ssd_mamba2_b4_l4096_h64_p64_n128"]
    nbytes, flops = bench.ssd_cost(w)
    tok = 4 * 4096
    assert nbytes == 2 * 2 * tok * 64 * 64 + 2 * 2 * tok * 128 + 2 * tok * 64 + 4 * 4 * 64 * 64 * 128 * 2
    assert flops == tok * 64 * (32 * 64 + 4 * 128 * 64) + tok * 32 * 128
    # the tensor-core kernel's chunk of 128 steps
    _, flops128 = bench.ssd_cost(w, Q=128)
    assert flops128 == tok * 64 * (128 * 64 + 4 * 128 * 64) + tok * 128 * 128


@pytest.mark.parametrize("workload", ["mamba130m_layer_b8_l2048_d1536",
                                      "ssd_mamba2_b4_l4096_h64_p64_n128",
                                      "decode_b128_d4096_x1000",
                                      "ssd_decode_b64_h64_p64_n128_x1000"])
def test_reference_arm_line(workload):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", workload, "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, check=True)
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["workload"] == workload
    for key in ("metric", "unit", "ms_per_step", "higher_is_better", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0

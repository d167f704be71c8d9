"""The seeded input generator: Philox4x32-10 known answers, C vs numpy
restatement, bf16 rounding, and the workload recipe."""
import numpy as np
import pytest

import ssm_inputs as gen

# Known-answer vectors published with Philox4x32-10 (Random123 distribution).
KAT = [
    ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
    ((0xFFFFFFFF,) * 4, (0xFFFFFFFF,) * 2, (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
    ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
     (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
]


@pytest.mark.parametrize("ctr,key,want", KAT)
def test_philox_known_answers(ctr, key, want):
    got = gen.philox4x32_10_np(np.array([ctr], np.uint32), np.array([key], np.uint32))[0]
    assert tuple(int(v) for v in got) == want
    import ctypes
    lib = gen._get_lib()
    c = (ctypes.c_uint32 * 4)(*ctr)
    k = (ctypes.c_uint32 * 2)(*key)
    o = (ctypes.c_uint32 * 4)()
    lib.philox4x32_10(c, k, o)
    assert tuple(o) == want


@pytest.mark.parametrize("out", ["f64", "f32", "bf16"])
def test_c_generator_matches_numpy(out):
    for kind, a, b in [(gen.KIND_NORMAL, 0.0, 1.0), (gen.KIND_NORMAL, 0.0, 0.5),
                       (gen.KIND_UNIFORM, 0.001, 0.1)]:
        c = gen.fill((7, 300), 12345, 3, kind, a, b, out=out, offset=2 ** 33 + 5, nthreads=3)
        n = gen.fill_np((7, 300), 12345, 3, kind, a, b, out=out, offset=2 ** 33 + 5)
        if out == "f64":
            np.testing.assert_allclose(c, n, rtol=1e-15, atol=1e-15)
        else:
            assert np.array_equal(c, n)


def test_threads_do_not_change_values():
    a = gen.fill((300000,), 9, 1, nthreads=1)
    b = gen.fill((300000,), 9, 1, nthreads=7)
    assert np.array_equal(a, b)


def test_offset_slices_are_consistent():
    whole = gen.fill((10, 64), 4, 2, out="bf16")
    part = gen.fill((64,), 4, 2, out="bf16", offset=3 * 64)
    assert np.array_equal(whole[3], part)


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e38],
                 dtype=np.float32)
    bits = gen.f32_to_bf16_bits(f)
    back = gen.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins
    assert back[1] == 1.0
    assert back[2] == np.float32(1.0 + 2 ** -6)  # tie, rounds up to even
    assert back[0] == 1.0 and back[3] == 1.0 and back[4] == -2.5
    rng = np.random.default_rng(0)
    v = rng.standard_normal(100000).astype(np.float32)
    w = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(v))
    assert np.all(np.abs(w - v) <= np.abs(v) * 2.0 ** -8)


def test_normal_moments():
    v = gen.fill((400000,), 1, gen.STREAM_X, out="f64")
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1) < 0.01
    d = gen.fill((400000,), 1, gen.STREAM_DELTA, b=0.5, out="f64")
    assert abs(d.std() - 0.5) < 0.005


def test_workload_recipe():
    w = gen.SCAN_WORKLOADS["tiny_f32_b1_l256_d64"]
    inp = gen.workload_inputs(w)
    assert inp["x"].shape == (1, 256, 64) and inp["x"].dtype == np.float32
    assert inp["B"].shape == (1, 256, 16)
    assert np.array_equal(inp["A"][5], -np.arange(1, 17, dtype=np.float32))
    assert np.all(inp["D"] == 1.0) and inp["h0"] is None
    # softplus(bias) = u ~ U[0.001, 0.1]
    u = np.log1p(np.exp(inp["delta_bias"].astype(np.float64)))
    assert np.all((u > 0.00099) & (u < 0.1001))
    w2 = gen.SCAN_WORKLOADS["pythia1b_layer_b4_l4096_d4096_h0"]
    assert w2.with_h0 and w2.io == "bf16" and w2.elements == 4 * 4096 * 4096
    small = gen.make_scan_inputs(2, 8, 16, 16, "bf16", 2, with_h0=True)
    assert small["x"].dtype == np.uint16 and small["h0"].dtype == np.float32


def test_decode_steps_are_stream_slices():
    s3 = gen.make_decode_inputs(4, 8, 16, "bf16", 4, step=3)
    full = gen.fill((5, 4, 8), 4, gen.STREAM_X, out="bf16")
    assert np.array_equal(s3["x"], full[3])


def test_ssd_recipe():
    w = gen.SSD_WORKLOADS["ssd_mamba2_b4_l4096_h64_p64_n128"]
    assert (w.batch, w.seqlen, w.nheads, w.headdim, w.dstate) == (4, 4096, 64, 64, 128)
    assert w.with_h0 and w.elements == 4 * 4096 * 64 * 64
    inp = gen.make_ssd_inputs(2, 9, 5, 64, 32, "bf16", 6, with_h0=True)
    assert inp["x"].shape == (2, 9, 5, 64) and inp["x"].dtype == np.uint16
    assert inp["dt"].shape == (2, 9, 5) and inp["B"].shape == (2, 9, 32)
    assert inp["h0"].shape == (2, 5, 64, 32) and inp["h0"].dtype == np.float32
    c = gen.ssd_constants(64, 6)
    assert np.all((c["A"] <= -1.0) & (c["A"] >= -16.0)) and np.all(c["D"] == 1.0)
    u = np.log1p(np.exp(c["dt_bias"].astype(np.float64)))
    assert np.all((u > 0.00099) & (u < 0.1001))
    # the scan's inputs carry the same per-head constants
    assert np.array_equal(gen.make_ssd_inputs(1, 2, 64, 64, 32, "bf16", 6)["A"], c["A"])


def test_ssd_decode_steps_are_stream_slices():
    s3 = gen.make_ssd_decode_inputs(2, 3, 4, 32, "bf16", 7, step=3)
    full = gen.fill((5, 2, 3, 4), 7, gen.STREAM_X, out="bf16")
    assert np.array_equal(s3["x"], full[3])
    full_b = gen.fill((5, 2, 32), 7, gen.STREAM_B, out="bf16")
    assert np.array_equal(s3["B"], full_b[3])

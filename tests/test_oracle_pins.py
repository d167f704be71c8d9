"""The oracle against its pins (CPU only), and mutation checks: copies of the
oracle source with one plausible mistake planted each must fail a pin."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins


@pytest.fixture(scope="module")
def o():
    return oracle.get()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(o, pin):
    pin(o)


def test_bf16_inputs_widen_exactly(o):
    """bf16 storage is read as the exact binary32 value it denotes."""
    import ssm_inputs as gen
    c = pins.random_case(41, batch=2, L=8, dim=3, N=4)
    bits = {k: gen.f32_to_bf16_bits(c[k]) for k in ("x", "delta", "B", "C", "z")}
    wide = {k: gen.bf16_bits_to_f32(v) for k, v in bits.items()}
    y16, h16 = o.selective_scan(bits["x"], bits["delta"], c["A"], bits["B"], bits["C"], D=c["D"],
                                z=bits["z"], delta_bias=c["delta_bias"], h0=c["h0"], io="bf16")
    y32, h32 = o.selective_scan(wide["x"], wide["delta"], c["A"], wide["B"], wide["C"], D=c["D"],
                                z=wide["z"], delta_bias=c["delta_bias"], h0=c["h0"], io="f32")
    assert np.array_equal(y16, y32) and np.array_equal(h16, h32)


def test_channel_subset_and_threads_agree(o):
    c = pins.random_case(43, batch=3, L=20, dim=5, N=4)
    kw = dict(D=c["D"], z=c["z"], delta_bias=c["delta_bias"], h0=c["h0"])
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], **kw)
    y4, hl4 = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], nthreads=4, **kw)
    assert np.array_equal(y, y4) and np.array_equal(hl, hl4)
    chans = [(2, 4), (0, 0), (1, 3)]
    ys, hs = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], channels=chans, **kw)
    for k, (b, d) in enumerate(chans):
        assert np.array_equal(ys[k], y[b, :, d]) and np.array_equal(hs[k], hl[b, d])


def test_oracle_rejects_bad_channels(o):
    c = pins.random_case(47)
    with pytest.raises(ValueError):
        o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], channels=[(5, 0)])


# (original, mutated) snippets of ssm_oracle.c: each is a plausible mistake.
MUTANTS = {
    "drop_skip": ("    y += Dd * xv;\n    if (j->z)", "    if (j->z)"),
    "sign_of_A": ("exp(dt * (double)j->A[d * N + n])", "exp(-dt * (double)j->A[d * N + n])"),
    "readout_before_update": (
        "      h[n] = dA * h[n] + dB * xv;\n      y += widen(j->C, i_bln + n, j->is_bf16) * h[n];",
        "      y += widen(j->C, i_bln + n, j->is_bf16) * h[n];\n      h[n] = dA * h[n] + dB * xv;"),
    "B_C_swapped": ("                        widen(j->B, i_bln + n, j->is_bf16);\n      h[n] = dA * h[n] + dB * xv;\n      y += widen(j->C,",
                    "                        widen(j->C, i_bln + n, j->is_bf16);\n      h[n] = dA * h[n] + dB * xv;\n      y += widen(j->B,"),
    "bias_dropped": ("widen(j->delta, i_bld, j->is_bf16) + bias;", "widen(j->delta, i_bld, j->is_bf16);"),
    "softplus_as_exp": ("return v > 20.0 ? v : log1p(exp(v));", "return v > 20.0 ? v : exp(v);"),
    "sigmoid_not_silu": ("return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    "h0_ignored": ("h[n] = j->h0 ? (double)j->h0[(b * Dm + d) * N + n] : 0.0;", "h[n] = 0.0;"),
    "A_transposed": ("exp(dt * (double)j->A[d * N + n])", "exp(dt * (double)j->A[(n * Dm + d) % (Dm * N)])"),
    "x_index_wrong": ("const double xv = widen(j->x, i_bld, j->is_bf16);",
                      "const double xv = widen(j->x, (i_bld + 1) % (j->batch * L * Dm), j->is_bf16);"),
    "dB_without_delta": ("      const double dB = input_coef(dt, (double)j->A[d * N + n], j->zoh) *\n",
                         "      const double dB = 1.0 *\n"),
    "decode_drops_gate": ("      if (z) acc *= silu(widen(z, i_bd, is_bf16));\n", ""),
    "decode_state_not_kept": ("        h[n] = dA * h[n] + dB * xv;\n        acc +=",
                              "        const double hn = dA * h[n] + dB * xv;\n        acc += 0 * hn +"),
    # backward pass
    "bwd_drops_A_term_of_dDelta": ("const double ddt = xv * sum_lb + sum_la;",
                                   "const double ddt = xv * sum_lb;"),
    "bwd_dA_uses_new_state": ("acc->dA[d * N + n] += lam[n] * dt * a * hprev;",
                              "acc->dA[d * N + n] += lam[n] * dt * hist[(t + 1) * N + n];"),
    "bwd_adjoint_not_decayed": ("      lam[n] *= a;\n", "      lam[n] *= 1.0;\n"),
    "bwd_silu_derivative_is_sigmoid": ("sg * (1.0 + zv * (1.0 - sg))", "sg"),
    "bwd_softplus_derivative_dropped": ("(v > 20.0 ? ddt : ddt * sigmoid(v))", "ddt"),
    "bwd_dB_without_delta": ("acc->dB[i_bln + n] += lam[n] * dt * xv;",
                             "acc->dB[i_bln + n] += lam[n] * xv;"),
    "bwd_dC_ignores_gate": ("acc->dC[i_bln + n] += g * hist[(t + 1) * N + n];",
                            "acc->dC[i_bln + n] += dyv * hist[(t + 1) * N + n];"),
    "bwd_dh_last_ignored": ("lam[n] = j->dh_last ? (double)j->dh_last[(b * Dm + d) * N + n] : 0.0;",
                            "lam[n] = 0.0;"),
    "bwd_dx_drops_skip": ("j->dx[k * L + t] = Dd * g + dt * sum_lb;",
                          "j->dx[k * L + t] = dt * sum_lb;"),
    "bwd_dh0_before_decay": ("      lam[n] *= a;\n", "      if (t > 0) lam[n] *= a;\n"),
    # causal conv1d + SiLU
    "conv_taps_flipped": ("u += (double)w[d * width + k] * widen(x, (b * L + s) * Dm + d, is_bf16);",
                          "u += (double)w[d * width + (width - 1 - k)] * widen(x, (b * L + s) * Dm + d, is_bf16);"),
    "conv_off_by_one": ("    const int64_t s = t - (width - 1) + k;\n    if (s < 0) continue;",
                        "    const int64_t s = t - width + k;\n    if (s < 0) continue;"),
    "conv_bias_dropped": ("  double u = bias ? (double)bias[d] : 0.0;", "  double u = 0.0;"),
    "conv_bwd_silu_derivative": ("du[t] = g * sg * (1.0 + u * (1.0 - sg));", "du[t] = g * sg;"),
    "conv_bwd_dx_not_transposed": ("          const int64_t t = s + (width - 1) - k;",
                                   "          const int64_t t = s - (width - 1) + k;"),
    "conv_bwd_dw_wrong_step": ("if (s >= 0) dw[d * width + k] += du[t] * widen(x, (b * seqlen + s) * dim + d, is_bf16);",
                               "if (s >= 0) dw[d * width + k] += du[t] * widen(x, (b * seqlen + t) * dim + d, is_bf16);"),
    "conv_bwd_dbias_from_dout": ("        dbias[d] += du[t];", "        dbias[d] += g;"),
    "conv_update_state_not_shifted": ("      for (int64_t k = 0; k + 1 < S; ++k) st[k] = st[k + 1];\n", ""),
    # exact zero-order hold
    "zoh_is_euler": ("  return An == 0.0 ? dt : expm1(dt * An) / An;", "  return dt;"),
    "zoh_no_division_by_A": ("  return An == 0.0 ? dt : expm1(dt * An) / An;",
                             "  return An == 0.0 ? dt : expm1(dt * An);"),
    # Mamba-2 SSD
    "ssd_readout_before_update": (
        "          S[p * N + n] = a * S[p * N + n] + delta * bn * xv;\n          acc += widen(Cm, (b * L + t) * N + n, is_bf16) * S[p * N + n];",
        "          acc += widen(Cm, (b * L + t) * N + n, is_bf16) * S[p * N + n];\n          S[p * N + n] = a * S[p * N + n] + delta * bn * xv;"),
    "ssd_B_C_swapped": ("const double bn = widen(Bm, (b * L + t) * N + n, is_bf16);",
                        "const double bn = widen(Cm, (b * L + t) * N + n, is_bf16);"),
    "ssd_bias_dropped": ("const double v = widen(dt, (b * L + t) * H + h, is_bf16) + bias;",
                         "const double v = widen(dt, (b * L + t) * H + h, is_bf16);"),
    "ssd_skip_dropped": ("y_out[(k * L + t) * P + p] = acc + Dh * xv;",
                         "y_out[(k * L + t) * P + p] = acc;"),
    "ssd_h0_ignored": ("S[p * N + n] = h0 ? (double)h0[((b * H + h) * P + p) * N + n] : 0.0;",
                       "S[p * N + n] = 0.0;"),
    "ssd_input_without_delta": ("S[p * N + n] = a * S[p * N + n] + delta * bn * xv;",
                                "S[p * N + n] = a * S[p * N + n] + bn * xv;"),
    "ssd_sign_of_A": ("const double a = exp(delta * (double)A[h]);",
                      "const double a = exp(-delta * (double)A[h]);"),
    "ssd_x_of_head_zero": ("const double xv = widen(x, ((b * L + t) * H + h) * P + p, is_bf16);",
                           "const double xv = widen(x, ((b * L + t) * H + 0) * P + p, is_bf16);"),
    "ssd_decode_state_not_kept": (
        "          S[n] = a * S[n] + delta * widen(Bm, b * N + n, is_bf16) * xv;\n          acc += widen(Cm, b * N + n, is_bf16) * S[n];",
        "          const double sn = a * S[n] + delta * widen(Bm, b * N + n, is_bf16) * xv;\n          acc += widen(Cm, b * N + n, is_bf16) * sn;"),
    "ssd_decode_skip_dropped": ("        y[(b * H + h) * P + p] = acc + (D ? (double)D[h] : 0.0) * xv;",
                                "        y[(b * H + h) * P + p] = acc;"),
    "ssd_decode_bias_dropped": (
        "const double v = widen(dt, b * H + h, is_bf16) + (dt_bias ? (double)dt_bias[h] : 0.0);",
        "const double v = widen(dt, b * H + h, is_bf16);"),
    "zoh_sign_flipped": ("  return An == 0.0 ? dt : expm1(dt * An) / An;",
                         "  return An == 0.0 ? dt : -expm1(dt * An) / An;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(oracle.SOURCE).read()
    before, after = MUTANTS[name]
    assert src.count(before) >= 1, f"mutation anchor for {name} not found in the oracle source"
    mutated = tmp_path / "ssm_oracle_mutant.c"
    mutated.write_text(src.replace(before, after, 1))
    lib = oracle.compile_library(str(mutated), str(tmp_path / "libmutant.so"))
    m = oracle.Oracle(lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(m)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"


# ---- property checks over random small shapes (CPU) ----------------------
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(batch=st.integers(1, 2), L=st.integers(1, 9), H=st.integers(1, 3), P=st.integers(1, 4),
       N=st.integers(1, 5), seed=st.integers(0, 2**31 - 1), h0=st.booleans())
def test_ssd_equals_tied_scan_any_shape(o, batch, L, H, P, N, seed, h0):
    """For any small shape, an SSD head equals the per-channel scan with A tied
    across states and Delta, D, bias tied across the head's channels."""
    c = pins._ssd_case(seed, batch=batch, L=L, H=H, P=P, N=N, h0=h0)
    y, hl = pins._ssd(o, c)
    dim = H * P
    tie = lambda v: np.repeat(v, P, axis=-1)  # noqa: E731
    h0v = None if c["h0"] is None else c["h0"].reshape(batch, dim, N)
    ys, hs = o.selective_scan(c["x"].reshape(batch, L, dim), tie(c["dt"]),
                              np.repeat(tie(c["A"])[:, None], N, axis=1), c["B"], c["C"],
                              D=tie(c["D"]), delta_bias=tie(c["dt_bias"]), h0=h0v)
    assert np.allclose(y, ys.reshape(batch, L, H, P), rtol=1e-12, atol=1e-12)
    assert np.allclose(hl, hs.reshape(batch, H, P, N), rtol=1e-12, atol=1e-12)


@settings(max_examples=25, deadline=None)
@given(L=st.integers(1, 12), split=st.integers(0, 12), seed=st.integers(0, 2**31 - 1))
def test_scan_split_anywhere(o, L, split, seed):
    """Scanning [0, k) and then [k, L) from the state reached equals one scan,
    for every k (the state carries everything; fp32 hand-over of the state)."""
    k = min(split, L)
    c = pins.random_case(seed, batch=1, L=L, dim=2, N=3, gate=False)
    kw = dict(D=c["D"], delta_bias=c["delta_bias"])
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], h0=c["h0"], **kw)
    part = lambda a, s: np.ascontiguousarray(a[:, s])  # noqa: E731
    y1, h1 = o.selective_scan(part(c["x"], slice(0, k)), part(c["delta"], slice(0, k)), c["A"],
                              part(c["B"], slice(0, k)), part(c["C"], slice(0, k)),
                              h0=c["h0"], **kw)
    y2, h2 = o.selective_scan(part(c["x"], slice(k, L)), part(c["delta"], slice(k, L)), c["A"],
                              part(c["B"], slice(k, L)), part(c["C"], slice(k, L)),
                              h0=h1.astype(np.float32), **kw)
    assert np.allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-6, atol=1e-6)
    assert np.allclose(h2, hl, rtol=1e-6, atol=1e-6)

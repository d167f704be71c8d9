"""The chunked form the SSD kernel evaluates, restated in fp64 numpy and
checked against the oracle's sequential loop (CPU only).

Per chunk of Q steps, with cum_t the in-chunk sum of Delta_r A[h]:
  G[t][s] = (C_t . B_s) e^{cum_t - cum_s} Delta_s  (s <= t), Y = G X + diag(e^cum) C H + D X,
  H <- e^{cum_end} H + (w X)^T B,  w_s = e^{cum_end - cum_s} Delta_s,
with steps past the end of the sequence taken as Delta = 0 (zero-filled
chunks change nothing). This is the algebra of the §4.1 dual form split at
chunk boundaries; the kernel's tiling of these products is checked on the
GPU against the oracle."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins


def chunked_ssd(c, Q):
    x, dt, A, B, C = (c[k].astype(np.float64) for k in ("x", "dt", "A", "B", "C"))
    D, bias = c["D"].astype(np.float64), c["dt_bias"].astype(np.float64)
    batch, L, H, P = x.shape
    N = B.shape[-1]
    y = np.zeros_like(x)
    h_last = np.zeros((batch, H, P, N))
    for b in range(batch):
        for h in range(H):
            S = (c["h0"][b, h].astype(np.float64).T.copy() if c["h0"] is not None
                 else np.zeros((N, P)))  # state as N x P
            for t0 in range(0, L, Q):
                idx = np.arange(t0, t0 + Q)
                ok = idx < L
                d = np.zeros(Q)
                d[ok] = np.logaddexp(0.0, dt[b, idx[ok], h] + bias[h])
                X = np.zeros((Q, P)); X[ok] = x[b, idx[ok], h]
                Bc = np.zeros((Q, N)); Bc[ok] = B[b, idx[ok]]
                Cc = np.zeros((Q, N)); Cc[ok] = C[b, idx[ok]]
                cum = np.cumsum(d * A[h])
                causal = np.arange(Q)[None, :] <= np.arange(Q)[:, None]
                G = np.where(causal, (Cc @ Bc.T) * np.exp(cum[:, None] - cum[None, :]) * d, 0.0)
                Y = G @ X + np.exp(cum)[:, None] * (Cc @ S) + D[h] * X
                w = np.exp(cum[-1] - cum) * d
                S = np.exp(cum[-1]) * S + Bc.T @ (w[:, None] * X)
                y[b, idx[ok], h] = Y[ok]
            h_last[b, h] = S.T
    return y, h_last


@pytest.mark.parametrize("Q,L", [(32, 75), (32, 32), (7, 20), (4, 1)])
def test_chunked_form_equals_oracle(Q, L):
    c = pins._ssd_case(401 + L, batch=2, L=L, H=3, P=5, N=6)
    y, hl = chunked_ssd(c, Q)
    yr, hr = oracle.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"],
                             dt_bias=c["dt_bias"], h0=c["h0"])
    np.testing.assert_allclose(y, yr, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(hl, hr, rtol=1e-10, atol=1e-10)

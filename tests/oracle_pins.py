"""Pins of the fp64 oracle to things other than itself.

Each pin takes an ``oracle.Oracle`` handle and raises AssertionError when
the oracle disagrees with a closed form, a brute-force evaluation of a
different formula, a library routine, an invariant of the recurrence or a
hand-worked example. ``tests/test_oracle_pins.py`` runs them against the
real oracle and against deliberately broken copies of it (every broken copy
must fail at least one pin).

Source of the definitions: page "Mamba 논문 리뷰: Selective State Space
Models로 Transformer를 넘어서" (youngju.dev) -- §2.2 discretised recurrence,
§3.1 softplus step, §3.3 selective_scan, §3.4 D skip and SiLU gate, §4.1 the
SSM as a (semi-separable) matrix acting on the sequence -- and the linear
attention recurrence s_t = s_{t-1} + phi(k_t)^T v_t of the page "[논문 리뷰]
Attention to Mamba: A Recipe for Cross-Architecture Distillation"
(suanlab.com, stage 2), which is the A = 0 special case.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
from scipy.special import expit

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _f32(a):
    return np.asarray(a, dtype=np.float32)


def _softplus_lib(v):
    return np.logaddexp(0.0, v)  # library log(1 + e^v)


def _close(a, b, rtol, atol=0.0, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.abs(a - b)
    tol = atol + rtol * np.abs(b)
    if not np.all(err <= tol):
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: mismatch at {i}: got {a[i]!r}, want {b[i]!r}")


def random_case(seed, batch=2, L=9, dim=3, N=4, gate=True, skip=True, h0=True, A=None,
                softplus=True):
    r = _rng(seed)
    case = dict(
        x=_f32(r.standard_normal((batch, L, dim))),
        delta=_f32(0.5 * r.standard_normal((batch, L, dim))),
        A=_f32(-r.uniform(0.2, 3.0, (dim, N))) if A is None else _f32(A),
        B=_f32(r.standard_normal((batch, L, N))),
        C=_f32(r.standard_normal((batch, L, N))),
        D=_f32(r.uniform(-1, 1, dim)) if skip else None,
        z=_f32(r.standard_normal((batch, L, dim))) if gate else None,
        delta_bias=_f32(r.uniform(-2, 0.5, dim)),
        h0=_f32(r.standard_normal((batch, dim, N))) if h0 else None,
        softplus=softplus,
    )
    return case


def _delta_f64(case):
    v = case["delta"].astype(np.float64)
    if case["delta_bias"] is not None:
        v = v + case["delta_bias"].astype(np.float64)[None, None, :]
    return _softplus_lib(v) if case["softplus"] else v


def _gate(y, case):
    if case["z"] is None:
        return y
    z = case["z"].astype(np.float64)
    return y * z * expit(z)


def _skip(case):
    if case["D"] is None:
        return 0.0
    return case["D"].astype(np.float64)[None, None, :] * case["x"].astype(np.float64)


# --------------------------------------------------------------------------
# pins
def pin_softplus_library(o):
    """L = 1, A = 0, B = C = x = 1, no skip: y = Delta = softplus(delta)."""
    v = _f32(np.concatenate([np.linspace(-30, 40, 141), [0.0, 19.99, 20.0, 20.01, 25.0]]))
    n = v.size
    one = np.ones((1, 1, n), np.float32)
    y, _ = o.selective_scan(one, v.reshape(1, 1, n), np.zeros((n, 1), np.float32),
                            np.ones((1, 1, 1), np.float32), np.ones((1, 1, 1), np.float32),
                            softplus=True)
    _close(y[0, 0], _softplus_lib(v.astype(np.float64)), 3e-9, what="softplus")


def pin_silu_library(o):
    """Delta = 1 (softplus off), A = 0, B = C = x = 1: y = SiLU(z) = z sigmoid(z)."""
    z = _f32(np.linspace(-12, 12, 97))
    n = z.size
    one = np.ones((1, 1, n), np.float32)
    y, _ = o.selective_scan(one, one, np.zeros((n, 1), np.float32),
                            np.ones((1, 1, 1), np.float32), np.ones((1, 1, 1), np.float32),
                            z=z.reshape(1, 1, n), softplus=False)
    zz = z.astype(np.float64)
    _close(y[0, 0], zz * expit(zz), 1e-13, 1e-300, what="silu")


def pin_A_zero_is_cumulative_sum(o):
    """A = 0 => deltaA = 1: h_t = h0 + cumsum_s(Delta_s x_s B_s) (linear
    attention's s_t = s_{t-1} + k_t^T v_t); y from a library prefix sum."""
    c = random_case(11, batch=2, L=17, dim=3, N=4, A=np.zeros((3, 4)))
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=True, h0=c["h0"])
    dt = _delta_f64(c)  # (b, L, d)
    inc = (dt * c["x"].astype(np.float64))[..., None] * c["B"].astype(np.float64)[:, :, None, :]
    h = c["h0"].astype(np.float64)[:, None] + np.cumsum(inc, axis=1)  # (b, L, d, n)
    yy = np.einsum("bln,bldn->bld", c["C"].astype(np.float64), h) + _skip(c)
    _close(y, _gate(yy, c), 1e-12, 1e-12, what="cumsum y")
    _close(hl, h[:, -1], 1e-12, 1e-12, what="cumsum h_last")


def pin_geometric_series(o):
    """Constant Delta, B, C, x in t: h_t = a^(t+1) h0 + Delta B x (1 - a^(t+1)) / (1 - a)."""
    r = _rng(5)
    batch, L, dim, N = 2, 40, 3, 4
    x = np.repeat(_f32(r.standard_normal((batch, 1, dim))), L, axis=1)
    delta = np.repeat(_f32(0.4 * r.standard_normal((batch, 1, dim))), L, axis=1)
    B = np.repeat(_f32(r.standard_normal((batch, 1, N))), L, axis=1)
    C = np.repeat(_f32(r.standard_normal((batch, 1, N))), L, axis=1)
    A = _f32(-r.uniform(0.3, 2.0, (dim, N)))
    D = _f32(r.uniform(-1, 1, dim))
    bias = _f32(r.uniform(-1, 0.5, dim))
    h0 = _f32(r.standard_normal((batch, dim, N)))
    y, hl = o.selective_scan(x, delta, A, B, C, D=D, delta_bias=bias, softplus=True, h0=h0)
    dt = _softplus_lib(delta[:, 0].astype(np.float64) + bias)  # (b, d)
    a = np.exp(dt[..., None] * A.astype(np.float64)[None])  # (b, d, n)
    u = dt[..., None] * B[:, 0].astype(np.float64)[:, None, :] * x[:, 0].astype(np.float64)[..., None]
    t = np.arange(1, L + 1, dtype=np.float64)[None, :, None, None]
    h = a[:, None] ** t * h0.astype(np.float64)[:, None] + u[:, None] * (1 - a[:, None] ** t) / (1 - a[:, None])
    yy = np.einsum("bn,bldn->bld", C[:, 0].astype(np.float64), h) + D[None, None] * x.astype(np.float64)
    _close(y, yy, 1e-12, 1e-12, what="geometric y")
    _close(hl, h[:, -1], 1e-12, 1e-12, what="geometric h_last")


def pin_single_step_by_hand(o):
    """L = 1: y = (C . (exp(Delta A) h0 + Delta B x) + D x) SiLU(z), written out."""
    c = random_case(3, batch=2, L=1, dim=3, N=4)
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=True, h0=c["h0"])
    for b in range(2):
        for d in range(3):
            v = float(c["delta"][b, 0, d]) + float(c["delta_bias"][d])
            dt = math.log1p(math.exp(v))
            h = [math.exp(dt * float(c["A"][d, n])) * float(c["h0"][b, d, n])
                 + dt * float(c["B"][b, 0, n]) * float(c["x"][b, 0, d]) for n in range(4)]
            yy = sum(float(c["C"][b, 0, n]) * h[n] for n in range(4)) + float(c["D"][d]) * float(c["x"][b, 0, d])
            zz = float(c["z"][b, 0, d])
            yy *= zz / (1 + math.exp(-zz))
            _close(y[b, 0, d], yy, 1e-13, 1e-15, what="one step y")
            _close(hl[b, d], h, 1e-13, 1e-15, what="one step h")


def pin_dual_matrix_form(o):
    """Brute force the sequence-mixing matrix (the SSM as a matrix, §4.1):
    y_t = sum_{s<=t} M_ts x_s + C_t.(prod_{r<=t} a_r) h0 + D x_t with
    M_ts = sum_n C_tn [prod_{s<r<=t} exp(Delta_r A_n)] Delta_s B_sn."""
    c = random_case(7, batch=2, L=12, dim=3, N=4)
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=True, h0=c["h0"])
    dt = _delta_f64(c)
    batch, L, dim = c["x"].shape
    N = c["A"].shape[1]
    yy = np.zeros((batch, L, dim))
    for b in range(batch):
        for d in range(dim):
            A = c["A"][d].astype(np.float64)
            for t in range(L):
                acc = 0.0
                for s in range(t + 1):
                    for n in range(N):
                        decay = 1.0
                        for rr in range(s + 1, t + 1):
                            decay *= math.exp(dt[b, rr, d] * A[n])
                        acc += float(c["C"][b, t, n]) * decay * dt[b, s, d] * float(c["B"][b, s, n]) * float(c["x"][b, s, d])
                for n in range(N):
                    decay = 1.0
                    for rr in range(0, t + 1):
                        decay *= math.exp(dt[b, rr, d] * A[n])
                    acc += float(c["C"][b, t, n]) * decay * float(c["h0"][b, d, n])
                yy[b, t, d] = acc
    yy = _gate(yy + _skip(c), c)
    _close(y, yy, 1e-11, 1e-12, what="dual form")


def pin_linear_in_x_and_h0(o):
    """Without the gate, y is affine in (x, h0): y(x, h0) = y(x, 0) + y(0, h0),
    and y(a x1 + b x2, 0) = a y(x1, 0) + b y(x2, 0)."""
    c = random_case(13, gate=False)
    x2 = _f32(_rng(14).standard_normal(c["x"].shape))
    run = lambda x, h0: o.selective_scan(x, c["delta"], c["A"], c["B"], c["C"], D=c["D"],
                                         delta_bias=c["delta_bias"], softplus=True, h0=h0)[0]
    zero_x = np.zeros_like(c["x"])
    _close(run(c["x"], c["h0"]), run(c["x"], None) + run(zero_x, c["h0"]), 1e-11, 1e-12,
           what="affine in h0")
    a, b = 0.75, -1.5
    lhs = run(_f32(a * c["x"].astype(np.float64) + b * x2), None)
    rhs = a * run(c["x"], None) + b * run(x2, None)
    # a*x + b*x2 is rounded once to fp32 on the left: tolerance 1e-6
    _close(lhs, rhs, 1e-6, 1e-6, what="linear in x")


def pin_split_invariance(o):
    """scan(L1) then scan(L2, h0 = h_last) equals scan(L1 + L2)."""
    c = random_case(17, batch=2, L=23, dim=3, N=4)
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=True, h0=c["h0"])
    k = 10
    part = lambda sl, h0: o.selective_scan(c["x"][:, sl], c["delta"][:, sl], c["A"],
                                           c["B"][:, sl], c["C"][:, sl], D=c["D"],
                                           z=c["z"][:, sl], delta_bias=c["delta_bias"],
                                           softplus=True, h0=h0)
    y1, h1 = part(slice(0, k), c["h0"])
    # h0 is fp32 at the boundary: compare against the full run in fp64 with tolerance
    y2, h2 = part(slice(k, None), _f32(h1))
    _close(y1, y[:, :k], 0, 0, what="prefix identical")
    _close(y2, y[:, k:], 1e-6, 1e-7, what="suffix")
    _close(h2, hl, 1e-6, 1e-7, what="h_last")


def pin_zero_step_keeps_state(o):
    """Delta = 0 (softplus off, delta = bias = 0): deltaA = 1, deltaB = 0, so
    h_t = h0 and y_t = C_t . h0 + D x_t."""
    c = random_case(19, gate=False, softplus=False)
    zero = np.zeros_like(c["delta"])
    y, hl = o.selective_scan(c["x"], zero, c["A"], c["B"], c["C"], D=c["D"], softplus=False,
                             h0=c["h0"])
    yy = np.einsum("bln,bdn->bld", c["C"].astype(np.float64), c["h0"].astype(np.float64)) + _skip(c)
    _close(y, yy, 1e-13, 1e-13, what="zero step y")
    _close(hl, c["h0"], 0, 0, what="zero step h")


def pin_large_step_is_memoryless(o):
    """Delta = 60 with A <= -1: exp(Delta A) < 1e-26, so h_t = Delta B_t x_t
    (the page's forgetting role of Delta, by the equations)."""
    c = random_case(23, gate=False, softplus=False, A=-np.ones((3, 4)) * np.arange(1, 5))
    big = np.full_like(c["delta"], 60.0)
    y, hl = o.selective_scan(c["x"], big, c["A"], c["B"], c["C"], D=c["D"], softplus=False,
                             h0=c["h0"])
    h = 60.0 * c["x"].astype(np.float64)[..., None] * c["B"].astype(np.float64)[:, :, None, :]
    yy = np.einsum("bln,bldn->bld", c["C"].astype(np.float64), h) + _skip(c)
    _close(y, yy, 1e-14, 1e-14, what="memoryless y")
    _close(hl, h[:, -1], 1e-14, 1e-14, what="memoryless h")


def pin_golden_hand_worked(o):
    with open(os.path.join(GOLDEN, "hand_worked_scan.json")) as f:
        spec = json.load(f)
    env = {"exp": math.exp, "log": math.log}
    for case in spec["cases"]:
        dims = case["dims"]
        batch, L, dim, N = dims["batch"], dims["seqlen"], dims["dim"], dims["dstate"]
        arr = lambda v, shape: None if v is None else _f32(v).reshape(shape)
        y, hl = o.selective_scan(
            arr(case["x"], (batch, L, dim)), arr(case["delta"], (batch, L, dim)),
            arr(case["A"], (dim, N)), arr(case["B"], (batch, L, N)), arr(case["C"], (batch, L, N)),
            D=arr(case["D"], (dim,)), z=arr(case["z"], (batch, L, dim)),
            delta_bias=arr(case["delta_bias"], (dim,)), softplus=case["softplus"],
            h0=arr(case["h0"], (batch, dim, N)))
        want_y = np.array([eval(e, {"__builtins__": {}}, env) for e in case["y"]])
        want_h = np.array([eval(e, {"__builtins__": {}}, env) for e in case["h_last"]])
        _close(y.reshape(-1), want_y, 1e-14, 1e-15, what=case["name"] + " y")
        _close(hl.reshape(-1), want_h, 1e-14, 1e-15, what=case["name"] + " h_last")


def pin_decode_steps_equal_scan(o):
    """L decode steps on a carried fp64 state equal one scan over the same tokens."""
    c = random_case(29, batch=2, L=15, dim=3, N=4)
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=True, h0=c["h0"])
    state = np.ascontiguousarray(c["h0"].astype(np.float64))
    for t in range(c["x"].shape[1]):
        yt = o.state_update(state, c["x"][:, t], c["delta"][:, t], c["A"], c["B"][:, t],
                            c["C"][:, t], D=c["D"], z=c["z"][:, t], delta_bias=c["delta_bias"],
                            softplus=True)
        _close(yt, y[:, t], 1e-14, 1e-14, what=f"decode step {t}")
    _close(state, hl, 1e-14, 1e-14, what="decode state")


def pin_decode_single_step_by_hand(o):
    c = random_case(31, batch=2, L=1, dim=3, N=4)
    state = np.ascontiguousarray(c["h0"].astype(np.float64))
    yt = o.state_update(state, c["x"][:, 0], c["delta"][:, 0], c["A"], c["B"][:, 0],
                        c["C"][:, 0], D=c["D"], z=c["z"][:, 0], delta_bias=c["delta_bias"],
                        softplus=True)
    for b in range(2):
        for d in range(3):
            dt = math.log1p(math.exp(float(c["delta"][b, 0, d]) + float(c["delta_bias"][d])))
            h = [math.exp(dt * float(c["A"][d, n])) * float(c["h0"][b, d, n])
                 + dt * float(c["B"][b, 0, n]) * float(c["x"][b, 0, d]) for n in range(4)]
            yy = sum(float(c["C"][b, 0, n]) * h[n] for n in range(4)) + float(c["D"][d]) * float(c["x"][b, 0, d])
            zz = float(c["z"][b, 0, d])
            yy *= zz / (1 + math.exp(-zz))
            _close(yt[b, d], yy, 1e-13, 1e-15, what="decode by hand y")
            _close(state[b, d], h, 1e-13, 1e-15, what="decode by hand h")


# --------------------------------------------------------------------------
# pins of the backward pass (gradients of the scan)
_GRAD_OF = {"x": "dx", "delta": "ddelta", "z": "dz", "B": "dB", "C": "dC", "A": "dA",
            "D": "dD", "delta_bias": "ddelta_bias", "h0": "dh0"}


def _loss(o, c, dy, dh_last):
    """sum dy * y + sum dh_last * h_last, in fp64, through the forward oracle."""
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=c["softplus"], h0=c["h0"])
    return float(np.sum(dy.astype(np.float64) * y) + np.sum(dh_last.astype(np.float64) * hl))


def _bwd(o, c, dy, dh_last):
    return o.selective_scan_bwd(c["x"], c["delta"], c["A"], c["B"], c["C"], dy, D=c["D"],
                                z=c["z"], delta_bias=c["delta_bias"], softplus=c["softplus"],
                                h0=c["h0"], dh_last=dh_last)


def _finite_differences(o, c, dy, dh_last, name):
    """Central differences of the loss in every fp32 element of input `name`,
    using the step the fp32 rounding actually takes."""
    base = c[name]
    fd = np.zeros(base.shape, dtype=np.float64)
    for i in np.ndindex(base.shape):
        v = float(base[i])
        h = 2.0 ** -11 * max(2.0 ** -4, abs(v))
        hi, lo = np.float32(v + h), np.float32(v - h)
        cc = dict(c)
        arr = base.copy()
        arr[i] = hi
        cc[name] = arr
        f_hi = _loss(o, cc, dy, dh_last)
        arr = base.copy()
        arr[i] = lo
        cc[name] = arr
        f_lo = _loss(o, cc, dy, dh_last)
        fd[i] = (f_hi - f_lo) / (float(hi) - float(lo))
    return fd


def _check_fd(o, c, seed, what):
    r = _rng(seed)
    dy = _f32(r.standard_normal(c["x"].shape))
    dh_last = _f32(r.standard_normal((c["x"].shape[0], c["x"].shape[2], c["A"].shape[1])))
    g = _bwd(o, c, dy, dh_last)
    for name, gname in _GRAD_OF.items():
        if c.get(name) is None:
            if name == "z":
                assert g["dz"] is None, f"{what}: dz without z"
            continue
        fd = _finite_differences(o, c, dy, dh_last, name)
        scale = max(1.0, float(np.max(np.abs(fd))))
        _close(g[gname], fd, 0.0, 2e-6 * scale, what=f"{what}: {gname} vs central differences")


def pin_bwd_finite_differences(o):
    """Every gradient of the backward pass equals central differences of the
    (separately pinned) forward oracle: gate, skip, h0, bias and softplus on."""
    c = random_case(101, batch=2, L=6, dim=3, N=4)
    _check_fd(o, c, 102, "all terms")


def pin_bwd_finite_differences_plain(o):
    """The same without gate, skip, h0 or softplus, and with a bias so large
    that softplus would sit above its cutoff of 20 (checked separately)."""
    c = random_case(103, batch=2, L=5, dim=2, N=3, gate=False, skip=False, h0=False,
                    softplus=False)
    # without softplus keep Delta > 0, so the recurrence decays
    c["delta"] = _f32(np.abs(c["delta"]))
    c["delta_bias"] = _f32(np.abs(c["delta_bias"]))
    _check_fd(o, c, 104, "plain")
    c = random_case(105, batch=1, L=4, dim=2, N=2)
    c["delta_bias"] = _f32([21.0, 0.3])  # channel 0 above the softplus cutoff
    c["A"] = _f32([[-0.01, -0.02], [-1.0, -2.0]])
    _check_fd(o, c, 106, "softplus cutoff")


def pin_bwd_autograd(o):
    """Reverse-mode autodiff (torch, fp64, CPU) of the §3.3 loop with the
    §3.4 skip and gate, written here from the page, agrees with the
    hand-derived adjoint loop of the oracle."""
    import torch
    c = random_case(107, batch=2, L=5, dim=3, N=4)
    r = _rng(108)
    dy = _f32(r.standard_normal(c["x"].shape))
    dh_last = _f32(r.standard_normal((2, 3, 4)))
    t = {k: torch.tensor(v.astype(np.float64), requires_grad=True)
         for k, v in c.items() if isinstance(v, np.ndarray)}
    dt = torch.nn.functional.softplus(t["delta"] + t["delta_bias"], threshold=20.0)
    h = t["h0"]
    ys = []
    for s in range(c["x"].shape[1]):
        dA = torch.exp(dt[:, s, :, None] * t["A"])
        dBx = dt[:, s, :, None] * t["B"][:, s, None, :] * t["x"][:, s, :, None]
        h = dA * h + dBx
        yy = (h * t["C"][:, s, None, :]).sum(-1) + t["D"] * t["x"][:, s]
        ys.append(yy * torch.nn.functional.silu(t["z"][:, s]))
    y = torch.stack(ys, dim=1)
    loss = (y * torch.tensor(dy.astype(np.float64))).sum() + \
        (h * torch.tensor(dh_last.astype(np.float64))).sum()
    loss.backward()
    g = _bwd(o, c, dy, dh_last)
    for name, gname in _GRAD_OF.items():
        _close(g[gname], t[name].grad.numpy(), 1e-10, 1e-12, what=f"autograd {gname}")


# --------------------------------------------------------------------------
# pins of the block's causal depthwise conv1d + SiLU (§3.4 Mamba Block)
def _conv_case(seed, batch=2, L=9, dim=3, width=4):
    r = _rng(seed)
    return (_f32(r.standard_normal((batch, L, dim))), _f32(0.5 * r.standard_normal((dim, width))),
            _f32(r.uniform(-0.5, 0.5, dim)))


def pin_conv_matches_torch_conv1d(o):
    """The page's own formulation: nn.Conv1d(groups=dim, padding=width-1) (torch's
    conv1d, fp64 CPU) cut to the first L outputs, then SiLU."""
    import torch
    for width in (2, 3, 4):
        x, w, b = _conv_case(201 + width, width=width)
        xt = torch.tensor(x.astype(np.float64)).transpose(1, 2)
        u = torch.nn.functional.conv1d(xt, torch.tensor(w.astype(np.float64))[:, None, :],
                                       torch.tensor(b.astype(np.float64)), padding=width - 1,
                                       groups=x.shape[2])[:, :, :x.shape[1]].transpose(1, 2)
        _close(o.conv1d_silu(x, w, b, silu=False), u.numpy(), 1e-13, 1e-14, what="conv, no SiLU")
        _close(o.conv1d_silu(x, w, b, silu=True), torch.nn.functional.silu(u).numpy(), 1e-13,
               1e-14, what="conv + SiLU")


def pin_conv_by_hand(o):
    """One channel, width 4, x = 1..5, w = (0.5, -1, 2, 0.25), bias 0.1:
    u_t = 0.1 + sum_k w_k x_(t-3+k) written out term by term."""
    x = _f32([1, 2, 3, 4, 5]).reshape(1, 5, 1)
    w = _f32([[0.5, -1.0, 2.0, 0.25]])
    b = _f32([0.1])
    bias = float(np.float32(0.1))
    want = [bias + 0.25 * 1,
            bias + 2.0 * 1 + 0.25 * 2,
            bias - 1.0 * 1 + 2.0 * 2 + 0.25 * 3,
            bias + 0.5 * 1 - 1.0 * 2 + 2.0 * 3 + 0.25 * 4,
            bias + 0.5 * 2 - 1.0 * 3 + 2.0 * 4 + 0.25 * 5]
    _close(o.conv1d_silu(x, w, b, silu=False)[0, :, 0], want, 1e-15, 0, what="conv by hand")
    _close(o.conv1d_silu(x, w, b, silu=True)[0, :, 0], [v / (1 + math.exp(-v)) for v in want],
           1e-15, 0, what="conv + SiLU by hand")


def pin_conv_is_causal(o):
    """Changing x at step s changes the output at steps s .. s+width-1 only."""
    x, w, b = _conv_case(207, L=12)
    base = o.conv1d_silu(x, w, b)
    s = 5
    x2 = x.copy()
    x2[:, s, :] += 1.0
    diff = np.abs(o.conv1d_silu(x2, w, b) - base).max(axis=(0, 2))
    assert np.all(diff[:s] == 0) and np.all(diff[s + 4:] == 0), "conv is not causal / too wide"
    assert np.all(diff[s:s + 4] > 0), "conv ignores a tap"


def pin_conv_bwd_finite_differences(o):
    """dx, dw, dbias of the conv backward equal central differences of the
    (separately pinned) forward, with and without SiLU."""
    for silu in (True, False):
        x, w, b = _conv_case(209, batch=2, L=7, dim=2)
        dout = _f32(_rng(210).standard_normal(x.shape))
        dx, dw, db = o.conv1d_silu_bwd(x, w, dout, b, silu=silu)
        args = {"x": x, "w": w, "b": b}
        for name, g in (("x", dx), ("w", dw), ("b", db)):
            base = args[name]
            fd = np.zeros(base.shape)
            for i in np.ndindex(base.shape):
                v = float(base[i])
                h = 2.0 ** -11 * max(2.0 ** -4, abs(v))
                vals = []
                for vv in (np.float32(v + h), np.float32(v - h)):
                    a = dict(args)
                    arr = base.copy()
                    arr[i] = vv
                    a[name] = arr
                    vals.append(float(np.sum(dout.astype(np.float64) *
                                             o.conv1d_silu(a["x"], a["w"], a["b"], silu=silu))))
                fd[i] = (vals[0] - vals[1]) / (float(np.float32(v + h)) - float(np.float32(v - h)))
            scale = max(1.0, float(np.max(np.abs(fd))))
            _close(g, fd, 0.0, 2e-6 * scale, what=f"conv d{name} vs central differences")


# --------------------------------------------------------------------------
# pins of the exact zero-order-hold input term (§2.2)
def pin_zoh_matches_scipy_cont2discrete(o):
    """Per step, the ZOH discretisation of dh/dt = diag(A_d) h + B_t x_t
    computed by scipy.signal.cont2discrete(method='zoh') (a matrix exponential
    of the augmented system), chained over the steps, equals the oracle's
    ZOH scan."""
    from scipy.signal import cont2discrete
    c = random_case(301, batch=1, L=6, dim=2, N=3)
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=True, h0=c["h0"], zoh=True)
    dt = _delta_f64(c)
    for d in range(2):
        A = np.diag(c["A"][d].astype(np.float64))
        h = c["h0"][0, d].astype(np.float64)
        for t in range(6):
            Bcol = c["B"][0, t].astype(np.float64).reshape(3, 1)
            Ad, Bd, _, _, _ = cont2discrete((A, Bcol, np.zeros((1, 3)), np.zeros((1, 1))),
                                            float(dt[0, t, d]), method="zoh")
            h = Ad @ h + Bd[:, 0] * float(c["x"][0, t, d])
            yy = float(c["C"][0, t].astype(np.float64) @ h) + float(c["D"][d]) * float(c["x"][0, t, d])
            zz = float(c["z"][0, t, d])
            yy *= zz / (1 + math.exp(-zz))
            _close(y[0, t, d], yy, 1e-10, 1e-12, what="zoh vs cont2discrete y")
        _close(hl[0, d], h, 1e-10, 1e-12, what="zoh vs cont2discrete h_last")


def pin_zoh_small_step_is_euler(o):
    """For Delta |A| -> 0 the ZOH input term (exp(Delta A) - 1) / A tends to
    Delta: with Delta ~ 1e-7 the two discretisations agree to ~1e-7 relative."""
    c = random_case(303, gate=False, softplus=False)
    c["delta"] = _f32(np.full(c["delta"].shape, 1e-7))
    c["delta_bias"] = None
    kw = dict(D=c["D"], softplus=False, h0=c["h0"])
    ye, he = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], **kw)
    yz, hz = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], zoh=True, **kw)
    assert not np.array_equal(yz, ye), "zoh flag ignored"
    _close(yz, ye, 1e-6, 1e-12, what="zoh small-step limit")


def pin_zoh_decode_steps_equal_scan(o):
    """L ZOH decode steps reproduce one ZOH scan."""
    c = random_case(305, batch=2, L=5, dim=3, N=4)
    y, hl = o.selective_scan(c["x"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                             delta_bias=c["delta_bias"], softplus=True, h0=c["h0"], zoh=True)
    state = c["h0"].astype(np.float64).copy()
    for t in range(5):
        yt = o.state_update(state, c["x"][:, t], c["delta"][:, t], c["A"], c["B"][:, t],
                            c["C"][:, t], D=c["D"], z=c["z"][:, t], delta_bias=c["delta_bias"],
                            softplus=True, zoh=True)
        _close(yt, y[:, t], 1e-13, 1e-14, what="zoh decode step")
    _close(state, hl, 1e-13, 1e-14, what="zoh decode state")


def pin_conv_update_steps_equal_conv(o):
    """L conv decode steps from a zero state reproduce the (separately pinned)
    causal conv over the sequence, for widths 2, 3, 4."""
    for width in (2, 3, 4):
        x, w, b = _conv_case(211 + width, batch=2, L=7, dim=3, width=width)
        full = o.conv1d_silu(x, w, b)
        state = np.zeros((2, 3, width - 1))
        for t in range(7):
            out = o.conv1d_silu_update(state, np.ascontiguousarray(x[:, t]), w, b)
            _close(out, full[:, t], 1e-14, 1e-15, what=f"conv step {t} width {width}")


def _ssd_case(seed, batch=2, L=10, H=3, P=4, N=5, h0=True):
    r = _rng(seed)
    return dict(
        x=_f32(r.standard_normal((batch, L, H, P))),
        dt=_f32(0.5 * r.standard_normal((batch, L, H))),
        A=_f32(-r.uniform(0.5, 4.0, H)),
        B=_f32(r.standard_normal((batch, L, N))),
        C=_f32(r.standard_normal((batch, L, N))),
        D=_f32(r.standard_normal(H)),
        dt_bias=_f32(np.log(np.expm1(r.uniform(0.05, 0.5, H)))),
        h0=_f32(r.standard_normal((batch, H, P, N))) if h0 else None,
    )


def _ssd(o, c, **kw):
    return o.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"], dt_bias=c["dt_bias"],
                      h0=c["h0"], **kw)


def pin_ssd_dual_matrix_form(o):
    """The SSD output against §4.1's dual form, brute force: per head,
    Y = (T . M) X with T the causal mask and the semi-separable
    M_ts = (C_t . B_s) [prod_{s<r<=t} exp(Delta_r A)] Delta_s, plus the
    initial state's term C_t (prod_{r<=t} exp(Delta_r A)) h0 and D x_t."""
    c = _ssd_case(301)
    y, _ = _ssd(o, c)
    batch, L, H, P = c["x"].shape
    dt = _softplus_lib(c["dt"].astype(np.float64) + c["dt_bias"].astype(np.float64))
    want = np.zeros((batch, L, H, P))
    for b in range(batch):
        for h in range(H):
            a = np.exp(dt[b, :, h] * float(c["A"][h]))
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    decay = 1.0
                    for r in range(s + 1, t + 1):
                        decay *= a[r]
                    M[t, s] = float(np.dot(c["C"][b, t].astype(np.float64),
                                           c["B"][b, s].astype(np.float64))) * decay * dt[b, s, h]
            X = c["x"][b, :, h].astype(np.float64)
            Y = M @ X
            for t in range(L):
                decay = np.prod(a[: t + 1])
                Y[t] += decay * (c["h0"][b, h].astype(np.float64) @ c["C"][b, t].astype(np.float64))
            want[b, :, h] = Y + float(c["D"][h]) * X
    _close(y, want, 1e-11, 1e-12, what="ssd dual form")


def pin_ssd_is_tied_selective_scan(o):
    """An SSD head is the selective scan over its headdim channels with A
    tied across states (A[d,n] = A[h]) and Delta, D, bias tied across the
    head's channels: the multi-head form against the separately pinned
    per-channel scan."""
    c = _ssd_case(303, batch=2, L=11, H=3, P=4, N=5)
    y, hl = _ssd(o, c)
    batch, L, H, P = c["x"].shape
    N = c["B"].shape[-1]
    dim = H * P
    tie = lambda v: np.repeat(v, P, axis=-1)  # noqa: E731  head value -> its channels
    ys, hs = o.selective_scan(c["x"].reshape(batch, L, dim), tie(c["dt"]),
                              np.repeat(tie(c["A"])[:, None], N, axis=1), c["B"], c["C"],
                              D=tie(c["D"]), delta_bias=tie(c["dt_bias"]),
                              h0=c["h0"].reshape(batch, dim, N))
    _close(y, ys.reshape(batch, L, H, P), 1e-13, 1e-13, what="ssd vs tied scan y")
    _close(hl, hs.reshape(batch, H, P, N), 1e-13, 1e-13, what="ssd vs tied scan h")


def pin_ssd_A_zero_is_cumulative_outer_product(o):
    """A = 0, Delta = 1 (no softplus): the state is the running sum of the
    outer products x_s B_s^T (linear attention), y_t = S_t C_t; computed with
    the library cumulative sum."""
    c = _ssd_case(305, h0=False)
    batch, L, H, P = c["x"].shape
    y, hl = o.ssd_scan(c["x"], np.ones((batch, L, H), np.float32), np.zeros(H, np.float32),
                       c["B"], c["C"], softplus=False)
    outer = np.einsum("blhp,bln->blhpn", c["x"].astype(np.float64), c["B"].astype(np.float64))
    S = np.cumsum(outer, axis=1)
    _close(y, np.einsum("blhpn,bln->blhp", S, c["C"].astype(np.float64)), 1e-12, 1e-12,
           what="ssd A=0 y")
    _close(hl, S[:, -1], 1e-12, 1e-12, what="ssd A=0 h")


def pin_ssd_split_invariance(o):
    """Running the first k steps, then the rest from the state reached,
    equals one run (the state carries everything)."""
    c = _ssd_case(307, L=13)
    y, hl = _ssd(o, c)
    k = 6
    first = {key: (v[:, :k] if key in ("x", "dt", "B", "C") else v) for key, v in c.items()}
    y1, h1 = _ssd(o, first)
    second = {key: (np.ascontiguousarray(v[:, k:]) if key in ("x", "dt", "B", "C") else v)
              for key, v in c.items()}
    second["h0"] = h1.astype(np.float32)
    y2, h2 = _ssd(o, second)
    _close(y1, y[:, :k], 1e-14, 1e-15, what="ssd first part")
    # the carried state is rounded to fp32 for the second run
    _close(y2, y[:, k:], 1e-6, 1e-6, what="ssd second part")
    _close(h2, hl, 1e-6, 1e-6, what="ssd end state")


def pin_ssd_zero_step_keeps_state(o):
    """Delta = 0 (no softplus, dt = 0, no bias): the state stays h0 and
    y_t = C_t . h0 + D x_t, for every step."""
    c = _ssd_case(315, L=6)
    zero = np.zeros_like(c["dt"])
    y, hl = o.ssd_scan(c["x"], zero, c["A"], c["B"], c["C"], D=c["D"], softplus=False,
                       h0=c["h0"])
    _close(hl, c["h0"], 0.0, 0.0, what="ssd zero step state")
    want = (np.einsum("bhpn,btn->bthp", c["h0"].astype(np.float64), c["C"].astype(np.float64))
            + c["D"].astype(np.float64)[None, None, :, None] * c["x"])
    _close(y, want, 1e-13, 1e-13, what="ssd zero step y")


def pin_ssd_large_step_is_memoryless(o):
    """Delta = 2000 with A <= -0.5: exp(Delta A) <= e^-1000 underflows to an
    exact zero in fp64, so the state after each step is Delta B_t x_t alone
    (no softplus, no skip)."""
    c = _ssd_case(317, L=5)
    big = np.full_like(c["dt"], 2000.0)
    y, hl = o.ssd_scan(c["x"], big, c["A"], c["B"], c["C"], softplus=False, h0=c["h0"])
    S = 2000.0 * np.einsum("bhp,bn->bhpn", c["x"][:, -1].astype(np.float64),
                           c["B"][:, -1].astype(np.float64))
    _close(hl, S, 1e-14, 0.0, what="ssd memoryless state")
    yt = 2000.0 * np.einsum("bthp,btn,btn->bthp", c["x"].astype(np.float64),
                            c["B"].astype(np.float64), c["C"].astype(np.float64))
    _close(y, yt, 1e-12, 1e-9, what="ssd memoryless y")


def pin_ssd_decode_steps_equal_scan(o):
    """L SSD decode steps from h0 reproduce the (separately pinned) SSD scan:
    every y_t and the end state."""
    c = _ssd_case(311, batch=2, L=7, H=3, P=4, N=5)
    y, hl = _ssd(o, c)
    state = c["h0"].astype(np.float64).copy()
    for t in range(7):
        yt = o.ssd_state_update(state, np.ascontiguousarray(c["x"][:, t]),
                                np.ascontiguousarray(c["dt"][:, t]), c["A"],
                                np.ascontiguousarray(c["B"][:, t]),
                                np.ascontiguousarray(c["C"][:, t]), D=c["D"],
                                dt_bias=c["dt_bias"])
        _close(yt, y[:, t], 1e-13, 1e-14, what=f"ssd decode step {t}")
    _close(state, hl, 1e-13, 1e-14, what="ssd decode state")


def pin_ssd_decode_single_step_by_hand(o):
    """One SSD decode step written out element by element."""
    c = _ssd_case(313, batch=1, L=1, H=2, P=3, N=4)
    state = c["h0"].astype(np.float64).copy()
    before = state.copy()
    y = o.ssd_state_update(state, c["x"][:, 0], c["dt"][:, 0], c["A"], c["B"][:, 0],
                           c["C"][:, 0], D=c["D"], dt_bias=c["dt_bias"])
    for h in range(2):
        v = float(c["dt"][0, 0, h]) + float(c["dt_bias"][h])
        delta = math.log1p(math.exp(v))
        a = math.exp(delta * float(c["A"][h]))
        for p in range(3):
            xv = float(c["x"][0, 0, h, p])
            acc = 0.0
            for n in range(4):
                hn = a * before[0, h, p, n] + delta * float(c["B"][0, 0, n]) * xv
                _close(state[0, h, p, n], hn, 1e-14, 1e-15, what="ssd step state")
                acc += float(c["C"][0, 0, n]) * hn
            _close(y[0, h, p], acc + float(c["D"][h]) * xv, 1e-13, 1e-15, what="ssd step y")


ALL_PINS = [
    pin_softplus_library,
    pin_silu_library,
    pin_A_zero_is_cumulative_sum,
    pin_geometric_series,
    pin_single_step_by_hand,
    pin_dual_matrix_form,
    pin_linear_in_x_and_h0,
    pin_split_invariance,
    pin_zero_step_keeps_state,
    pin_large_step_is_memoryless,
    pin_golden_hand_worked,
    pin_decode_steps_equal_scan,
    pin_decode_single_step_by_hand,
    pin_bwd_finite_differences,
    pin_bwd_finite_differences_plain,
    pin_bwd_autograd,
    pin_conv_matches_torch_conv1d,
    pin_conv_by_hand,
    pin_conv_is_causal,
    pin_conv_bwd_finite_differences,
    pin_conv_update_steps_equal_conv,
    pin_zoh_matches_scipy_cont2discrete,
    pin_zoh_small_step_is_euler,
    pin_zoh_decode_steps_equal_scan,
    pin_ssd_dual_matrix_form,
    pin_ssd_is_tied_selective_scan,
    pin_ssd_A_zero_is_cumulative_outer_product,
    pin_ssd_split_invariance,
    pin_ssd_zero_step_keeps_state,
    pin_ssd_large_step_is_memoryless,
    pin_ssd_decode_steps_equal_scan,
    pin_ssd_decode_single_step_by_hand,
]

"""fp64 CPU oracle for the Mamba selective-SSM scan and decode state update.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path
(``selective_state_space_39_b200``) never imports it, and this package never
imports the product: the two share no code. The only shared module is the
seeded input generator ``ssm_inputs``, which holds none of the method's
arithmetic.

The arithmetic lives in ``ssm_oracle.c`` (plain sequential fp64 loops). This
module compiles it with gcc on first use and marshals numpy arrays to it.
The backward pass (``selective_scan_bwd``) is the reverse-mode derivative
of the same loop, written out in ``ssm_oracle.c``. What it computes follows
the page "Mamba 논문 리뷰: Selective State Space Models로 Transformer를
넘어서" (youngju.dev): §2.2 discretised recurrence,
§3.1 softplus step size, §3.3 simplified ``selective_scan``, §3.4 block gate,
D skip and the causal depthwise conv1d + SiLU (``conv1d_silu``), §4.1 the
multi-head SSD form (``ssd_scan``) and its recurrent decode step
(``ssd_state_update``). Every function here is pinned by
``tests/test_oracle_pins.py``
against closed forms, brute force and invariants.

bf16 arrays are passed as numpy ``uint16`` holding the raw bf16 bits with
``io="bf16"``; fp32 arrays as ``float32`` with ``io="f32"``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "ssm_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()


def compile_library(source: str = SOURCE, out_path: str = LIB_PATH) -> str:
    """Compile the oracle C source into a shared library with gcc (-O2, no
    fast-math, so fp64 semantics are IEEE)."""
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    tmp = out_path + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-o", tmp, source, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


def _needs_build(src: str, lib: str) -> bool:
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


_F32P = ctypes.POINTER(ctypes.c_float)
_F64P = ctypes.POINTER(ctypes.c_double)
_I64P = ctypes.POINTER(ctypes.c_int64)


class Oracle:
    """Handle on one compiled oracle library (the default one, or a test's
    deliberately mutated copy)."""

    def __init__(self, lib_path: str):
        self.lib = ctypes.CDLL(lib_path)
        f = self.lib.oracle_selective_scan
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                      _F32P, ctypes.c_void_p, ctypes.c_void_p, _F32P, ctypes.c_void_p,
                      _F32P, ctypes.c_int, _F32P, _I64P, ctypes.c_int64, _F64P, _F64P,
                      ctypes.c_int]
        fz = self.lib.oracle_selective_scan_zoh
        fz.restype = ctypes.c_int
        fz.argtypes = f.argtypes
        gz = self.lib.oracle_state_update_zoh
        gz.restype = ctypes.c_int
        fb = self.lib.oracle_selective_scan_bwd
        fb.restype = ctypes.c_int
        fb.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                       _F32P, ctypes.c_void_p, ctypes.c_void_p, _F32P, ctypes.c_void_p,
                       _F32P, ctypes.c_int, _F32P, ctypes.c_void_p, _F32P, _I64P,
                       ctypes.c_int64] + [_F64P] * 9 + [ctypes.c_int]
        cf = self.lib.oracle_conv1d_silu
        cf.restype = ctypes.c_int
        cf.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int, ctypes.c_void_p, _F32P, _F32P,
                                              ctypes.c_int, _F64P]
        cb = self.lib.oracle_conv1d_silu_bwd
        cb.restype = ctypes.c_int
        cb.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int, ctypes.c_void_p, _F32P, _F32P,
                                              ctypes.c_int, ctypes.c_void_p, _F64P, _F64P, _F64P]
        cu = self.lib.oracle_conv1d_silu_update
        cu.restype = ctypes.c_int
        cu.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_int, _F64P, ctypes.c_void_p, _F32P, _F32P,
                                              ctypes.c_int, _F64P]
        g = self.lib.oracle_state_update
        g.restype = ctypes.c_int
        g.argtypes = [ctypes.c_int64] * 3 + [ctypes.c_int, _F64P, ctypes.c_void_p,
                      ctypes.c_void_p, _F32P, ctypes.c_void_p, ctypes.c_void_p, _F32P,
                      ctypes.c_void_p, _F32P, ctypes.c_int, _F64P]
        gz.argtypes = g.argtypes
        su = self.lib.oracle_ssd_state_update
        su.restype = ctypes.c_int
        su.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int, _F64P, ctypes.c_void_p,
                                              ctypes.c_void_p, _F32P, ctypes.c_void_p,
                                              ctypes.c_void_p, _F32P, _F32P, ctypes.c_int, _F64P]
        sd = self.lib.oracle_ssd_scan
        sd.restype = ctypes.c_int
        sd.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                              _F32P, ctypes.c_void_p, ctypes.c_void_p, _F32P,
                                              _F32P, ctypes.c_int, _F32P, _I64P, ctypes.c_int64,
                                              _F64P, _F64P]

    # -- helpers -----------------------------------------------------------
    @staticmethod
    def _io_array(a, io, shape, name, optional=False):
        if a is None:
            if optional:
                return None
            raise ValueError(f"{name} is required")
        want = np.uint16 if io == "bf16" else np.float32
        a = np.ascontiguousarray(a)
        if a.dtype != want:
            raise TypeError(f"{name}: expected {want} for io={io}, got {a.dtype}")
        if tuple(a.shape) != tuple(shape):
            raise ValueError(f"{name}: expected shape {shape}, got {a.shape}")
        return a

    @staticmethod
    def _f32_array(a, shape, name, optional=True):
        if a is None:
            if optional:
                return None
            raise ValueError(f"{name} is required")
        a = np.ascontiguousarray(a, dtype=np.float32)
        if tuple(a.shape) != tuple(shape):
            raise ValueError(f"{name}: expected shape {shape}, got {a.shape}")
        return a

    @staticmethod
    def _ptr(a, ctype=None):
        if a is None:
            return None
        if ctype is None:
            return ctypes.c_void_p(a.ctypes.data)
        return a.ctypes.data_as(ctypes.POINTER(ctype))

    # -- the scan ----------------------------------------------------------
    def selective_scan(self, x, delta, A, B, C, D=None, z=None, delta_bias=None,
                       softplus=True, h0=None, io="f32", channels=None, nthreads=1, zoh=False):
        """Selective scan over all channels, or over ``channels`` (a list of
        (b, d) pairs). Returns ``(y, h_last)`` in fp64: for all channels
        y is (batch, L, dim) and h_last (batch, dim, N); for a channel list
        y is (nchan, L) and h_last (nchan, N). ``zoh``: the exact zero-order
        hold input term (exp(Delta A) - 1) / A * B instead of Delta * B."""
        x = np.asarray(x)
        batch, L, dim = x.shape
        N = np.asarray(A).shape[1]
        x = self._io_array(x, io, (batch, L, dim), "x")
        delta = self._io_array(delta, io, (batch, L, dim), "delta")
        B = self._io_array(B, io, (batch, L, N), "B")
        C = self._io_array(C, io, (batch, L, N), "C")
        z = self._io_array(z, io, (batch, L, dim), "z", optional=True)
        A = self._f32_array(A, (dim, N), "A", optional=False)
        D = self._f32_array(D, (dim,), "D")
        delta_bias = self._f32_array(delta_bias, (dim,), "delta_bias")
        h0 = self._f32_array(h0, (batch, dim, N), "h0")
        full = channels is None
        if full:
            bb, dd = np.meshgrid(np.arange(batch), np.arange(dim), indexing="ij")
            chans = np.stack([bb.ravel(), dd.ravel()], axis=1).astype(np.int64)
        else:
            chans = np.ascontiguousarray(np.asarray(channels, dtype=np.int64).reshape(-1, 2))
        nchan = chans.shape[0]
        y = np.empty((nchan, L), dtype=np.float64)
        h_last = np.empty((nchan, N), dtype=np.float64)
        fn = self.lib.oracle_selective_scan_zoh if zoh else self.lib.oracle_selective_scan
        rc = fn(
            batch, L, dim, N, 1 if io == "bf16" else 0, self._ptr(x), self._ptr(delta),
            self._ptr(A, ctypes.c_float), self._ptr(B), self._ptr(C),
            self._ptr(D, ctypes.c_float), self._ptr(z), self._ptr(delta_bias, ctypes.c_float),
            1 if softplus else 0, self._ptr(h0, ctypes.c_float),
            self._ptr(chans, ctypes.c_int64), nchan, self._ptr(y, ctypes.c_double),
            self._ptr(h_last, ctypes.c_double), int(nthreads))
        if rc != 0:
            raise ValueError("oracle_selective_scan rejected its arguments")
        if full:
            y = y.reshape(batch, dim, L).transpose(0, 2, 1).copy()
            h_last = h_last.reshape(batch, dim, N)
        return y, h_last

    # -- the scan's gradients ----------------------------------------------
    def selective_scan_bwd(self, x, delta, A, B, C, dy, D=None, z=None, delta_bias=None,
                           softplus=True, h0=None, dh_last=None, io="f32", channels=None,
                           nthreads=1):
        """Gradients of the loss sum(dy * y) + sum(dh_last * h_last) with
        respect to every input of ``selective_scan`` (same arguments, plus the
        upstream ``dy`` in the io type and ``dh_last`` fp32 or None).

        Returns a dict of fp64 arrays: ``dx, ddelta, dz`` (batch, L, dim) —
        ``dz`` None without z — ``dh0`` (batch, dim, N), and ``dA`` (dim, N),
        ``dB, dC`` (batch, L, N), ``dD, ddelta_bias`` (dim). ``ddelta`` is the
        gradient with respect to the raw delta (before bias and softplus).
        With ``channels`` (a list of (b, d) pairs) the per-channel outputs are
        (nchan, L) / (nchan, N) and the summed ones cover the listed channels
        only."""
        x = np.asarray(x)
        batch, L, dim = x.shape
        N = np.asarray(A).shape[1]
        x = self._io_array(x, io, (batch, L, dim), "x")
        delta = self._io_array(delta, io, (batch, L, dim), "delta")
        B = self._io_array(B, io, (batch, L, N), "B")
        C = self._io_array(C, io, (batch, L, N), "C")
        z = self._io_array(z, io, (batch, L, dim), "z", optional=True)
        dy = self._io_array(dy, io, (batch, L, dim), "dy")
        A = self._f32_array(A, (dim, N), "A", optional=False)
        D = self._f32_array(D, (dim,), "D")
        delta_bias = self._f32_array(delta_bias, (dim,), "delta_bias")
        h0 = self._f32_array(h0, (batch, dim, N), "h0")
        dh_last = self._f32_array(dh_last, (batch, dim, N), "dh_last")
        full = channels is None
        if full:
            bb, dd = np.meshgrid(np.arange(batch), np.arange(dim), indexing="ij")
            chans = np.stack([bb.ravel(), dd.ravel()], axis=1).astype(np.int64)
        else:
            chans = np.ascontiguousarray(np.asarray(channels, dtype=np.int64).reshape(-1, 2))
        nchan = chans.shape[0]
        out = {k: np.empty((nchan, L), dtype=np.float64) for k in ("dx", "ddelta", "dz")}
        out["dh0"] = np.empty((nchan, N), dtype=np.float64)
        out["dA"] = np.empty((dim, N), dtype=np.float64)
        out["dB"] = np.empty((batch, L, N), dtype=np.float64)
        out["dC"] = np.empty((batch, L, N), dtype=np.float64)
        out["dD"] = np.empty((dim,), dtype=np.float64)
        out["ddelta_bias"] = np.empty((dim,), dtype=np.float64)
        f64 = lambda k: self._ptr(out[k], ctypes.c_double)  # noqa: E731
        rc = self.lib.oracle_selective_scan_bwd(
            batch, L, dim, N, 1 if io == "bf16" else 0, self._ptr(x), self._ptr(delta),
            self._ptr(A, ctypes.c_float), self._ptr(B), self._ptr(C),
            self._ptr(D, ctypes.c_float), self._ptr(z), self._ptr(delta_bias, ctypes.c_float),
            1 if softplus else 0, self._ptr(h0, ctypes.c_float), self._ptr(dy),
            self._ptr(dh_last, ctypes.c_float), self._ptr(chans, ctypes.c_int64), nchan,
            f64("dx"), f64("ddelta"), f64("dz"), f64("dh0"), f64("dA"), f64("dB"), f64("dC"),
            f64("dD"), f64("ddelta_bias"), int(nthreads))
        if rc == -2:
            raise MemoryError("oracle_selective_scan_bwd ran out of memory")
        if rc != 0:
            raise ValueError("oracle_selective_scan_bwd rejected its arguments")
        if z is None:
            out["dz"] = None
        if full:
            for k in ("dx", "ddelta", "dz"):
                if out[k] is not None:
                    out[k] = out[k].reshape(batch, dim, L).transpose(0, 2, 1).copy()
            out["dh0"] = out["dh0"].reshape(batch, dim, N)
        return out

    # -- the block's causal depthwise conv1d + SiLU ---------------------------
    def conv1d_silu(self, x, w, bias=None, silu=True, io="f32"):
        """out[b,t,d] = SiLU(bias[d] + sum_k w[d,k] x[b, t-(width-1)+k, d]) with
        zero padding before t = 0; x (batch, L, dim) in the io type, w (dim,
        width) and bias (dim,) fp32. Returns out in fp64."""
        x = np.asarray(x)
        batch, L, dim = x.shape
        width = np.asarray(w).shape[1]
        x = self._io_array(x, io, (batch, L, dim), "x")
        w = self._f32_array(w, (dim, width), "w", optional=False)
        bias = self._f32_array(bias, (dim,), "bias")
        out = np.empty((batch, L, dim), dtype=np.float64)
        rc = self.lib.oracle_conv1d_silu(batch, L, dim, width, 1 if io == "bf16" else 0,
                                         self._ptr(x), self._ptr(w, ctypes.c_float),
                                         self._ptr(bias, ctypes.c_float), 1 if silu else 0,
                                         self._ptr(out, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_conv1d_silu rejected its arguments")
        return out

    def conv1d_silu_bwd(self, x, w, dout, bias=None, silu=True, io="f32"):
        """Gradients of sum(dout * out) for conv1d_silu: returns (dx (batch, L,
        dim), dw (dim, width), dbias (dim,)) in fp64."""
        x = np.asarray(x)
        batch, L, dim = x.shape
        width = np.asarray(w).shape[1]
        x = self._io_array(x, io, (batch, L, dim), "x")
        dout = self._io_array(dout, io, (batch, L, dim), "dout")
        w = self._f32_array(w, (dim, width), "w", optional=False)
        bias = self._f32_array(bias, (dim,), "bias")
        dx = np.empty((batch, L, dim), dtype=np.float64)
        dw = np.empty((dim, width), dtype=np.float64)
        db = np.empty((dim,), dtype=np.float64)
        rc = self.lib.oracle_conv1d_silu_bwd(batch, L, dim, width, 1 if io == "bf16" else 0,
                                             self._ptr(x), self._ptr(w, ctypes.c_float),
                                             self._ptr(bias, ctypes.c_float), 1 if silu else 0,
                                             self._ptr(dout), self._ptr(dx, ctypes.c_double),
                                             self._ptr(dw, ctypes.c_double),
                                             self._ptr(db, ctypes.c_double))
        if rc == -2:
            raise MemoryError("oracle_conv1d_silu_bwd ran out of memory")
        if rc != 0:
            raise ValueError("oracle_conv1d_silu_bwd rejected its arguments")
        return dx, dw, db

    def conv1d_silu_update(self, state, x, w, bias=None, silu=True, io="f32"):
        """One decode step of the causal conv on the fp64 ``state`` (batch,
        dim, width-1; oldest input first), in place. x is (batch, dim).
        Returns out (batch, dim) in fp64."""
        if state.dtype != np.float64 or not state.flags.c_contiguous:
            raise TypeError("state must be a C-contiguous float64 array")
        batch, dim, S = state.shape
        width = S + 1
        x = self._io_array(x, io, (batch, dim), "x")
        w = self._f32_array(w, (dim, width), "w", optional=False)
        bias = self._f32_array(bias, (dim,), "bias")
        out = np.empty((batch, dim), dtype=np.float64)
        rc = self.lib.oracle_conv1d_silu_update(batch, dim, width, 1 if io == "bf16" else 0,
                                                self._ptr(state, ctypes.c_double), self._ptr(x),
                                                self._ptr(w, ctypes.c_float),
                                                self._ptr(bias, ctypes.c_float), 1 if silu else 0,
                                                self._ptr(out, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_conv1d_silu_update rejected its arguments")
        return out

    # -- decode ------------------------------------------------------------
    def state_update(self, state, x, delta, A, B, C, D=None, z=None, delta_bias=None,
                     softplus=True, io="f32", zoh=False):
        """One decode step on the fp64 ``state`` (batch, dim, N), in place.
        Returns y (batch, dim) in fp64."""
        if state.dtype != np.float64 or not state.flags.c_contiguous:
            raise TypeError("state must be a C-contiguous float64 array")
        batch, dim, N = state.shape
        x = self._io_array(x, io, (batch, dim), "x")
        delta = self._io_array(delta, io, (batch, dim), "delta")
        B = self._io_array(B, io, (batch, N), "B")
        C = self._io_array(C, io, (batch, N), "C")
        z = self._io_array(z, io, (batch, dim), "z", optional=True)
        A = self._f32_array(A, (dim, N), "A", optional=False)
        D = self._f32_array(D, (dim,), "D")
        delta_bias = self._f32_array(delta_bias, (dim,), "delta_bias")
        y = np.empty((batch, dim), dtype=np.float64)
        fn = self.lib.oracle_state_update_zoh if zoh else self.lib.oracle_state_update
        rc = fn(
            batch, dim, N, 1 if io == "bf16" else 0, self._ptr(state, ctypes.c_double),
            self._ptr(x), self._ptr(delta), self._ptr(A, ctypes.c_float), self._ptr(B),
            self._ptr(C), self._ptr(D, ctypes.c_float), self._ptr(z),
            self._ptr(delta_bias, ctypes.c_float), 1 if softplus else 0,
            self._ptr(y, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_state_update rejected its arguments")
        return y


    # -- Mamba-2 SSD ---------------------------------------------------------
    def ssd_scan(self, x, dt, A, B, C, D=None, dt_bias=None, softplus=True, h0=None, io="f32",
                 pairs=None):
        """The multi-head SSD scan (scalar A per head, B and C shared by the
        heads). x (batch, L, heads, headdim), dt (batch, L, heads), A (heads,),
        B, C (batch, L, dstate), D, dt_bias (heads,) or None, h0 (batch, heads,
        headdim, dstate) or None. Returns y (batch, L, heads, headdim) and
        h_last (batch, heads, headdim, dstate) in fp64; with ``pairs`` (a list
        of (b, h)) y is (npairs, L, headdim) and h_last (npairs, headdim,
        dstate)."""
        x = np.asarray(x)
        batch, L, H, P = x.shape
        N = np.asarray(B).shape[-1]
        x = self._io_array(x, io, (batch, L, H, P), "x")
        dt = self._io_array(dt, io, (batch, L, H), "dt")
        B = self._io_array(B, io, (batch, L, N), "B")
        C = self._io_array(C, io, (batch, L, N), "C")
        A = self._f32_array(A, (H,), "A", optional=False)
        D = self._f32_array(D, (H,), "D")
        dt_bias = self._f32_array(dt_bias, (H,), "dt_bias")
        h0 = self._f32_array(h0, (batch, H, P, N), "h0")
        full = pairs is None
        if full:
            bb, hh = np.meshgrid(np.arange(batch), np.arange(H), indexing="ij")
            pr = np.stack([bb.ravel(), hh.ravel()], axis=1).astype(np.int64)
        else:
            pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
        npairs = pr.shape[0]
        y = np.empty((npairs, L, P), dtype=np.float64)
        h_last = np.empty((npairs, P, N), dtype=np.float64)
        rc = self.lib.oracle_ssd_scan(
            batch, L, H, P, N, 1 if io == "bf16" else 0, self._ptr(x), self._ptr(dt),
            self._ptr(A, ctypes.c_float), self._ptr(B), self._ptr(C),
            self._ptr(D, ctypes.c_float), self._ptr(dt_bias, ctypes.c_float),
            1 if softplus else 0, self._ptr(h0, ctypes.c_float), self._ptr(pr, ctypes.c_int64),
            npairs, self._ptr(y, ctypes.c_double), self._ptr(h_last, ctypes.c_double))
        if rc == -2:
            raise MemoryError("oracle_ssd_scan ran out of memory")
        if rc != 0:
            raise ValueError("oracle_ssd_scan rejected its arguments")
        if full:
            y = y.reshape(batch, H, L, P).transpose(0, 2, 1, 3).copy()
            h_last = h_last.reshape(batch, H, P, N)
        return y, h_last


    def ssd_state_update(self, state, x, dt, A, B, C, D=None, dt_bias=None, softplus=True,
                         io="f32"):
        """One SSD decode step on the fp64 ``state`` (batch, heads, headdim,
        dstate), in place. x (batch, heads, headdim), dt (batch, heads), B, C
        (batch, dstate). Returns y (batch, heads, headdim) in fp64."""
        if state.dtype != np.float64 or not state.flags.c_contiguous:
            raise TypeError("state must be a C-contiguous float64 array")
        batch, H, P, N = state.shape
        x = self._io_array(x, io, (batch, H, P), "x")
        dt = self._io_array(dt, io, (batch, H), "dt")
        B = self._io_array(B, io, (batch, N), "B")
        C = self._io_array(C, io, (batch, N), "C")
        A = self._f32_array(A, (H,), "A", optional=False)
        D = self._f32_array(D, (H,), "D")
        dt_bias = self._f32_array(dt_bias, (H,), "dt_bias")
        y = np.empty((batch, H, P), dtype=np.float64)
        rc = self.lib.oracle_ssd_state_update(
            batch, H, P, N, 1 if io == "bf16" else 0, self._ptr(state, ctypes.c_double),
            self._ptr(x), self._ptr(dt), self._ptr(A, ctypes.c_float), self._ptr(B),
            self._ptr(C), self._ptr(D, ctypes.c_float), self._ptr(dt_bias, ctypes.c_float),
            1 if softplus else 0, self._ptr(y, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle_ssd_state_update rejected its arguments")
        return y


_default = None


def get() -> Oracle:
    """The oracle built from ``ssm_oracle.c`` (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            if _needs_build(SOURCE, LIB_PATH):
                compile_library()
            _default = Oracle(LIB_PATH)
        return _default


def selective_scan(*args, **kwargs):
    return get().selective_scan(*args, **kwargs)


def state_update(*args, **kwargs):
    return get().state_update(*args, **kwargs)


def selective_scan_bwd(*args, **kwargs):
    return get().selective_scan_bwd(*args, **kwargs)


def conv1d_silu(*args, **kwargs):
    return get().conv1d_silu(*args, **kwargs)


def conv1d_silu_bwd(*args, **kwargs):
    return get().conv1d_silu_bwd(*args, **kwargs)


def conv1d_silu_update(*args, **kwargs):
    return get().conv1d_silu_update(*args, **kwargs)


def ssd_scan(*args, **kwargs):
    return get().ssd_scan(*args, **kwargs)


def ssd_state_update(*args, **kwargs):
    return get().ssd_state_update(*args, **kwargs)


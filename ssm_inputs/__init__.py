"""Seeded synthetic inputs for the selective-scan workloads.

This module is the only code shared by the CUDA path's callers (benchmark,
smoke check, GPU tests) and the CPU oracle's callers. It draws random numbers
and rounds them to the storage type; it holds none of the scan's arithmetic.

Generator: Philox4x32-10 (counter-based; Salmon et al., SC'11) with
Box-Muller, implemented in ``philox_gen.c`` (multi-threaded) and restated in
numpy here (``philox4x32_10_np``, ``fill_np``) so the two can be checked
against each other and against the published known-answer vectors.

Recipe (the Mamba-shaped synthetic workload):
  x, z, B, C ~ N(0, 1)          delta_raw ~ N(0, 0.5^2)
  delta_bias[d] = log(expm1(u_d)),  u_d ~ U[0.001, 0.1]   (so softplus(bias) = u_d)
  A[d, n] = -(n + 1)  (S4D-real init: A = -exp(log(arange(1, N+1))))
  D[d] = 1            h0 = 0 or, where requested, h0 ~ N(0, 1) fp32
bf16 tensors are rounded once (binary32 RNE, then bf16 RNE) and both sides
consume the same bytes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "philox_gen.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD_DIR, "libssmgen.so")
_lock = threading.Lock()
_lib = None

# stream ids, one per tensor role
STREAM_X, STREAM_DELTA, STREAM_Z, STREAM_B, STREAM_C, STREAM_H0, STREAM_BIAS = 1, 2, 3, 4, 5, 6, 7
# upstream gradients of the backward pass
STREAM_DY, STREAM_DH_LAST = 8, 9
# the block's causal conv1d: raw input, taps, bias, upstream gradient
STREAM_CONV_X, STREAM_CONV_W, STREAM_CONV_BIAS, STREAM_CONV_DOUT = 10, 11, 12, 13
# a learned-looking A (no (n + 1) A[d, 0] structure)
STREAM_A_LEARNED = 14
# Mamba-2 SSD: per-head A and step bias
STREAM_SSD_A, STREAM_SSD_BIAS = 15, 16
KIND_NORMAL, KIND_UNIFORM = 0, 1
OUT_F64, OUT_F32, OUT_BF16 = 0, 1, 2


def compile_library(out_path: str = _LIB) -> str:
    os.makedirs(os.path.dirname(out_path), exist_ok=True)
    tmp = out_path + ".tmp.%d" % os.getpid()
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                    "-o", tmp, _SRC, "-lm", "-lpthread"], check=True)
    os.replace(tmp, out_path)
    return out_path


def _get_lib():
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
                compile_library()
            lib = ctypes.CDLL(_LIB)
            lib.ssm_gen_fill.restype = ctypes.c_int
            lib.ssm_gen_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                         ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                         ctypes.c_double, ctypes.c_int, ctypes.c_void_p,
                                         ctypes.c_int]
            lib.philox4x32_10.restype = None
            lib.philox4x32_10.argtypes = [ctypes.POINTER(ctypes.c_uint32)] * 3
            _lib = lib
        return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def fill(shape, seed, stream, kind=KIND_NORMAL, a=0.0, b=1.0, out="f32", offset=0,
         nthreads=None):
    """Array of ``shape`` whose element i is the generator's value for counter
    ``offset + i`` of ``stream``. ``out`` is "f64", "f32" or "bf16" (raw bf16
    bits as uint16). For normals a = mean, b = sigma; for uniforms [a, b)."""
    count = int(np.prod(shape)) if len(shape) else 1
    dtype, code = {"f64": (np.float64, OUT_F64), "f32": (np.float32, OUT_F32),
                   "bf16": (np.uint16, OUT_BF16)}[out]
    arr = np.empty(shape, dtype=dtype)
    _get_lib().ssm_gen_fill(seed, stream, offset, count, kind, float(a), float(b), code,
                            arr.ctypes.data, nthreads or default_threads())
    return arr


# ---------------------------------------------------------------------------
# numpy restatement (checks the C generator; also used for tiny cases)
_M0, _M1, _W0, _W1 = 0xD2511F53, 0xCD9E8D57, 0x9E3779B9, 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10_np(ctr, key):
    """Philox4x32-10 on arrays: ctr (..., 4) and key (..., 2) of uint32."""
    c = [np.asarray(ctr[..., i], dtype=np.uint64) for i in range(4)]
    k0 = np.asarray(key[..., 0], dtype=np.uint64)
    k1 = np.asarray(key[..., 1], dtype=np.uint64)
    for _ in range(10):
        p0 = np.uint64(_M0) * c[0]
        p1 = np.uint64(_M1) * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        c = [(hi1 ^ c[1] ^ k0) & _MASK, lo1, (hi0 ^ c[3] ^ k1) & _MASK, lo0]
        k0 = (k0 + np.uint64(_W0)) & _MASK
        k1 = (k1 + np.uint64(_W1)) & _MASK
    return np.stack(c, axis=-1).astype(np.uint32)


def _u53_np(a, b):
    a = (a >> np.uint32(5)).astype(np.float64)
    b = (b >> np.uint32(6)).astype(np.float64)
    return (a * 67108864.0 + b) * (1.0 / 9007199254740992.0)


def f32_to_bf16_bits(f):
    """Round binary32 values to bf16 (nearest even); returns uint16 bits."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u >> np.uint64(16)) & np.uint64(0xFFFF)).astype(np.uint16)


def bf16_bits_to_f32(bits):
    """Exact widening of bf16 bits (uint16) to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def fill_np(shape, seed, stream, kind=KIND_NORMAL, a=0.0, b=1.0, out="f32", offset=0):
    count = int(np.prod(shape)) if len(shape) else 1
    idx = np.arange(count, dtype=np.uint64) + np.uint64(offset)
    ctr = np.zeros((count, 4), dtype=np.uint32)
    ctr[:, 0] = (idx & _MASK).astype(np.uint32)
    ctr[:, 1] = (idx >> np.uint64(32)).astype(np.uint32)
    ctr[:, 2] = np.uint32(stream)
    key = np.zeros((count, 2), dtype=np.uint32)
    key[:, 0] = np.uint32(seed & 0xFFFFFFFF)
    key[:, 1] = np.uint32((seed >> 32) & 0xFFFFFFFF)
    w = philox4x32_10_np(ctr, key)
    u2 = _u53_np(w[:, 2], w[:, 3])
    if kind == KIND_NORMAL:
        u1 = 1.0 - _u53_np(w[:, 0], w[:, 1])
        v = a + b * np.sqrt(-2.0 * np.log(u1)) * np.cos(6.283185307179586 * u2)
    else:
        v = a + (b - a) * u2
    if out == "f64":
        return v.reshape(shape)
    f = v.astype(np.float32)
    if out == "f32":
        return f.reshape(shape)
    return f32_to_bf16_bits(f).reshape(shape)


# ---------------------------------------------------------------------------
# workloads
@dataclass(frozen=True)
class ScanWorkload:
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int
    io: str          # "f32" or "bf16"
    seed: int
    gate: bool = True
    skip: bool = True
    with_h0: bool = False

    @property
    def elements(self) -> int:
        return self.batch * self.seqlen * self.dim


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    dim: int
    dstate: int
    io: str
    seed: int
    steps: int


SCAN_WORKLOADS = {
    "tiny_f32_b1_l256_d64": ScanWorkload("tiny_f32_b1_l256_d64", 1, 256, 64, 16, "f32", 0),
    "mamba130m_layer_b8_l2048_d1536": ScanWorkload(
        "mamba130m_layer_b8_l2048_d1536", 8, 2048, 1536, 16, "bf16", 1),
    "pythia1b_layer_b4_l4096_d4096_h0": ScanWorkload(
        "pythia1b_layer_b4_l4096_d4096_h0", 4, 4096, 4096, 16, "bf16", 2, with_h0=True),
    "long_b1_l262144_d1536": ScanWorkload("long_b1_l262144_d1536", 1, 262144, 1536, 16, "bf16", 3),
}
@dataclass(frozen=True)
class SsdWorkload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    io: str
    seed: int
    with_h0: bool = False

    @property
    def elements(self) -> int:
        return self.batch * self.seqlen * self.nheads * self.headdim


# The Mamba-2 layer of d_model 2048 (expand 2: 4096 channels = 64 heads of 64,
# d_state 128): the pages' example input (1 x 1024) and the 4 x 4096 batch of
# the 1B-scale scan.
SSD_WORKLOADS = {
    "ssd_mamba2_b1_l1024_h64_p64_n128": SsdWorkload(
        "ssd_mamba2_b1_l1024_h64_p64_n128", 1, 1024, 64, 64, 128, "bf16", 5),
    "ssd_mamba2_b4_l4096_h64_p64_n128": SsdWorkload(
        "ssd_mamba2_b4_l4096_h64_p64_n128", 4, 4096, 64, 64, 128, "bf16", 6, with_h0=True),
}

@dataclass(frozen=True)
class SsdDecodeWorkload:
    name: str
    batch: int
    nheads: int
    headdim: int
    dstate: int
    io: str
    seed: int
    steps: int


# Decode on the same Mamba-2 layer: 64 sequences, 64 heads of 64, d_state 128
# (a 134 MB fp32 state, larger than L2), 1000 generated tokens.
SSD_DECODE_WORKLOADS = {
    "ssd_decode_b64_h64_p64_n128_x1000": SsdDecodeWorkload(
        "ssd_decode_b64_h64_p64_n128_x1000", 64, 64, 64, 128, "bf16", 7, 1000),
}

DECODE_WORKLOADS = {
    "decode_b128_d4096_x1000": DecodeWorkload("decode_b128_d4096_x1000", 128, 4096, 16, "bf16", 4, 1000),
}


def a_matrix(dim, dstate):
    """A[d, n] = -(n + 1) for every channel, as fp32."""
    return np.tile(-np.arange(1, dstate + 1, dtype=np.float32), (dim, 1))


def a_matrix_learned(dim, dstate, seed):
    """A[d, n] = -exp(A_log[d, n]) with A_log = log(n + 1) + U[-0.5, 0.5]: the
    initial values perturbed per (d, n) as training moves them, so that A has
    no (n + 1) A[d, 0] structure (fp32)."""
    jitter = fill((dim, dstate), seed, STREAM_A_LEARNED, KIND_UNIFORM, -0.5, 0.5, out="f64")
    a_log = np.log(np.arange(1, dstate + 1, dtype=np.float64))[None, :] + jitter
    return (-np.exp(a_log)).astype(np.float32)


def delta_bias(dim, seed, nthreads=None):
    u = fill((dim,), seed, STREAM_BIAS, KIND_UNIFORM, 0.001, 0.1, out="f64", nthreads=nthreads)
    return np.log(np.expm1(u)).astype(np.float32)


def make_scan_inputs(batch, seqlen, dim, dstate, io, seed, *, gate=True, skip=True,
                     with_h0=False, nthreads=None, batch_offset=0):
    """All inputs of one scan, as numpy arrays (io tensors as float32, or as
    uint16 bf16 bits when io == "bf16"). ``batch_offset`` selects rows
    batch_offset .. batch_offset+batch of a larger global batch (the values
    of a row do not depend on how the batch is split)."""
    bld, bln = (batch, seqlen, dim), (batch, seqlen, dstate)
    o_ld, o_ln, o_dn = (batch_offset * seqlen * dim, batch_offset * seqlen * dstate,
                        batch_offset * dim * dstate)
    out = {
        "x": fill(bld, seed, STREAM_X, out=io, offset=o_ld, nthreads=nthreads),
        "delta": fill(bld, seed, STREAM_DELTA, b=0.5, out=io, offset=o_ld, nthreads=nthreads),
        "B": fill(bln, seed, STREAM_B, out=io, offset=o_ln, nthreads=nthreads),
        "C": fill(bln, seed, STREAM_C, out=io, offset=o_ln, nthreads=nthreads),
        "z": fill(bld, seed, STREAM_Z, out=io, offset=o_ld, nthreads=nthreads) if gate else None,
        "A": a_matrix(dim, dstate),
        "D": np.ones(dim, dtype=np.float32) if skip else None,
        "delta_bias": delta_bias(dim, seed, nthreads),
        "h0": (fill((batch, dim, dstate), seed, STREAM_H0, out="f32", offset=o_dn,
                    nthreads=nthreads) if with_h0 else None),
    }
    return out


def workload_inputs(w: ScanWorkload, nthreads=None, batch=None, batch_offset=0):
    return make_scan_inputs(w.batch if batch is None else batch, w.seqlen, w.dim, w.dstate,
                            w.io, w.seed, gate=w.gate, skip=w.skip, with_h0=w.with_h0,
                            nthreads=nthreads, batch_offset=batch_offset)


def make_grad_inputs(batch, seqlen, dim, dstate, io, seed, *, with_dh_last=True, nthreads=None,
                     batch_offset=0):
    """Upstream gradients for the backward pass: dy (batch, L, dim) in the io
    type and dh_last (batch, dim, dstate) fp32, both N(0, 1)."""
    o_ld, o_dn = batch_offset * seqlen * dim, batch_offset * dim * dstate
    return {
        "dy": fill((batch, seqlen, dim), seed, STREAM_DY, out=io, offset=o_ld, nthreads=nthreads),
        "dh_last": (fill((batch, dim, dstate), seed, STREAM_DH_LAST, out="f32", offset=o_dn,
                         nthreads=nthreads) if with_dh_last else None),
    }


def make_conv_inputs(batch, seqlen, dim, width, io, seed, *, nthreads=None):
    """Inputs of the block's causal depthwise conv1d: x (batch, L, dim) ~ N(0, 1)
    in the io type, taps w (dim, width) and bias (dim,) ~ U[-0.5, 0.5] fp32
    (the range of nn.Conv1d's default initialisation for groups = channels
    and 4 taps), dout (batch, L, dim) ~ N(0, 1) in the io type."""
    shape = (batch, seqlen, dim)
    return {
        "x": fill(shape, seed, STREAM_CONV_X, out=io, nthreads=nthreads),
        "w": fill((dim, width), seed, STREAM_CONV_W, KIND_UNIFORM, -0.5, 0.5, out="f32"),
        "bias": fill((dim,), seed, STREAM_CONV_BIAS, KIND_UNIFORM, -0.5, 0.5, out="f32"),
        "dout": fill(shape, seed, STREAM_CONV_DOUT, out=io, nthreads=nthreads),
    }


def make_ssd_inputs(batch, seqlen, nheads, headdim, dstate, io, seed, *, with_h0=False,
                    nthreads=None):
    """Inputs of one multi-head SSD scan: x (batch, L, heads, headdim) ~ N(0, 1),
    dt (batch, L, heads) ~ N(0, 0.5^2), B, C (batch, L, dstate) ~ N(0, 1), all
    in the io type; per head A ~ -U[1, 16], dt_bias = log(expm1(U[0.001, 0.1])),
    D = 1 (fp32); h0 (batch, heads, headdim, dstate) ~ N(0, 1) fp32 or None."""
    return {
        "x": fill((batch, seqlen, nheads, headdim), seed, STREAM_X, out=io, nthreads=nthreads),
        "dt": fill((batch, seqlen, nheads), seed, STREAM_DELTA, b=0.5, out=io, nthreads=nthreads),
        "B": fill((batch, seqlen, dstate), seed, STREAM_B, out=io, nthreads=nthreads),
        "C": fill((batch, seqlen, dstate), seed, STREAM_C, out=io, nthreads=nthreads),
        **ssd_constants(nheads, seed),
        "h0": (fill((batch, nheads, headdim, dstate), seed, STREAM_H0, out="f32",
                    nthreads=nthreads) if with_h0 else None),
    }


def ssd_constants(nheads, seed):
    """Per-head parameters of the SSD recipe: A ~ -U[1, 16], dt_bias =
    log(expm1(U[0.001, 0.1])), D = 1 (fp32)."""
    return {
        "A": (-fill((nheads,), seed, STREAM_SSD_A, KIND_UNIFORM, 1.0, 16.0, out="f64")).astype(
            np.float32),
        "D": np.ones(nheads, dtype=np.float32),
        "dt_bias": np.log(np.expm1(fill((nheads,), seed, STREAM_SSD_BIAS, KIND_UNIFORM, 0.001,
                                        0.1, out="f64"))).astype(np.float32),
    }


def make_ssd_decode_inputs(batch, nheads, headdim, dstate, io, seed, step, nthreads=None):
    """Inputs of SSD decode step `step`: the step's slice of a (steps, ...)
    stream (x (batch, heads, headdim), dt (batch, heads), B, C (batch,
    dstate)), so step k's values do not depend on how many steps are drawn."""
    nx, nd, nn = batch * nheads * headdim, batch * nheads, batch * dstate
    return {
        "x": fill((batch, nheads, headdim), seed, STREAM_X, out=io, offset=step * nx,
                  nthreads=nthreads),
        "dt": fill((batch, nheads), seed, STREAM_DELTA, b=0.5, out=io, offset=step * nd,
                   nthreads=nthreads),
        "B": fill((batch, dstate), seed, STREAM_B, out=io, offset=step * nn, nthreads=nthreads),
        "C": fill((batch, dstate), seed, STREAM_C, out=io, offset=step * nn, nthreads=nthreads),
    }


def ssd_workload_inputs(w: SsdWorkload, nthreads=None):
    return make_ssd_inputs(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.io, w.seed,
                           with_h0=w.with_h0, nthreads=nthreads)


def make_decode_inputs(batch, dim, dstate, io, seed, step, nthreads=None):
    """Inputs of decode step `step`: the step's slice of a (steps, batch, ...)
    stream, so step k's values do not depend on how many steps are drawn."""
    bd, bn = (batch, dim), (batch, dstate)
    return {
        "x": fill(bd, seed, STREAM_X, out=io, offset=step * batch * dim, nthreads=nthreads),
        "delta": fill(bd, seed, STREAM_DELTA, b=0.5, out=io, offset=step * batch * dim,
                      nthreads=nthreads),
        "z": fill(bd, seed, STREAM_Z, out=io, offset=step * batch * dim, nthreads=nthreads),
        "B": fill(bn, seed, STREAM_B, out=io, offset=step * batch * dstate, nthreads=nthreads),
        "C": fill(bn, seed, STREAM_C, out=io, offset=step * batch * dstate, nthreads=nthreads),
    }


def decode_constants(dim, dstate, seed):
    return {"A": a_matrix(dim, dstate), "D": np.ones(dim, dtype=np.float32),
            "delta_bias": delta_bias(dim, seed)}


def as_float(a, io):
    """Widen io-typed numpy data to float32 (exact)."""
    if a is None:
        return None
    return bf16_bits_to_f32(a) if io == "bf16" else np.asarray(a, dtype=np.float32)


"""ctypes binding of libssmscan.so: argument marshalling only.

Every step of the scan runs in the library's CUDA kernels; this module only
checks tensor metadata, allocates outputs/workspace with torch when the
caller does not pass them, and forwards raw device pointers and the current
CUDA stream. There is no CPU fallback: without the built library (or without
a GPU) calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

SSM_DTYPE_F32, SSM_DTYPE_BF16 = 0, 1
_STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported size or dtype",
           -3: "workspace missing or too small", -4: "CUDA error",
           -5: "a kernel wait timed out"}


class SsmError(RuntimeError):
    def __init__(self, code: int, where: str, with_detail: bool = False):
        self.code = code
        detail = ""
        if (with_detail or code in (-4, -5)) and _lib is not None:
            detail = _lib.ssm_last_error_detail().decode(errors="replace")
        msg = f"{where}: {_STATUS.get(code, 'unknown status')} ({code})"
        super().__init__(msg + (f": {detail}" if detail else ""))


class ScanPlan(ctypes.Structure):
    _fields_ = [("segments", ctypes.c_int32), ("segment_steps", ctypes.c_int32),
                ("channel_tiles", ctypes.c_int32), ("channels_per_cta", ctypes.c_int32),
                ("ctas_carry", ctypes.c_int32), ("ctas_main", ctypes.c_int32),
                ("kernels", ctypes.c_int32), ("workspace_bytes", ctypes.c_int64)]


_lib = None
_VP = ctypes.c_void_p
_I64 = ctypes.c_int64


def lib() -> ctypes.CDLL:
    """Load libssmscan.so from the package directory, or the build named by
    $SSM_SCAN_LIBRARY (raises if absent)."""
    global _lib
    if _lib is None:
        # SSM_SCAN_LIBRARY may point at another build of the same library
        path = os.environ.get("SSM_SCAN_LIBRARY") or _build.LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m selective_state_space_39_b200.build`"
                " (the CUDA library is required; there is no CPU fallback)")
        L = ctypes.CDLL(path)
        L.ssm_scan_version.restype = ctypes.c_int
        L.ssm_status_string.restype = ctypes.c_char_p
        L.ssm_status_string.argtypes = [ctypes.c_int]
        L.ssm_last_error_detail.restype = ctypes.c_char_p
        L.ssm_last_error_detail.argtypes = []
        L.ssm_scan_workspace_bytes.restype = ctypes.c_size_t
        L.ssm_scan_workspace_bytes.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int]
        L.ssm_scan_plan.restype = ctypes.c_int
        L.ssm_scan_plan.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int, ctypes.POINTER(ScanPlan)]
        L.ssm_scan_fwd.restype = ctypes.c_int
        L.ssm_scan_fwd.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int, _VP, _VP, _VP, _VP, _VP,
                                   _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP, _VP,
                                   ctypes.c_size_t, _VP]
        L.ssm_scan_fwd_zoh.restype = ctypes.c_int
        L.ssm_scan_fwd_zoh.argtypes = L.ssm_scan_fwd.argtypes
        L.ssm_scan_fwd_noalloc.restype = ctypes.c_int
        L.ssm_scan_fwd_noalloc.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int, _VP, _VP, _VP,
                                           _VP, _VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP, _VP,
                                           _VP]
        L.ssm_scan_status.restype = ctypes.c_int
        L.ssm_scan_status.argtypes = [_VP, ctypes.c_size_t, _I64, _I64, _I64, _I64, ctypes.c_int,
                                      _VP]
        L.ssm_scan_status_noalloc.restype = ctypes.c_int
        L.ssm_scan_status_noalloc.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int, _VP]
        L.ssm_scan_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.ssm_scan_bwd_workspace_bytes.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int]
        L.ssm_scan_bwd.restype = ctypes.c_int
        L.ssm_scan_bwd.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int] + [_VP] * 8 + \
            [ctypes.c_int] + [_VP] * 13 + [ctypes.c_size_t, _VP]
        L.ssm_conv1d_silu_fwd.restype = ctypes.c_int
        L.ssm_conv1d_silu_fwd.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int, _VP, _VP, _VP,
                                          ctypes.c_int, _VP, _VP]
        L.ssm_conv1d_silu_update.restype = ctypes.c_int
        L.ssm_conv1d_silu_update.argtypes = [_I64, _I64, _I64, ctypes.c_int, _VP, _VP, _VP, _VP,
                                             ctypes.c_int, _VP, _VP]
        L.ssm_conv1d_silu_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.ssm_conv1d_silu_bwd_workspace_bytes.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int]
        L.ssm_conv1d_silu_bwd.restype = ctypes.c_int
        L.ssm_conv1d_silu_bwd.argtypes = [_I64, _I64, _I64, _I64, ctypes.c_int, _VP, _VP, _VP,
                                          ctypes.c_int, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t,
                                          _VP]
        L.ssm_state_update.restype = ctypes.c_int
        L.ssm_state_update.argtypes = [_I64, _I64, _I64, ctypes.c_int, _VP, _VP, _VP, _VP, _VP,
                                       _VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP]
        L.ssm_delta_sum.restype = ctypes.c_int
        L.ssm_delta_sum.argtypes = [_I64, _I64, _I64, ctypes.c_int, _VP, _VP, ctypes.c_int, _VP,
                                    _VP]
        L.ssm_compose_carries.restype = ctypes.c_int
        L.ssm_compose_carries.argtypes = [_I64, _I64, _I64, _I64, _VP, _VP, _VP, _VP, _VP, _VP]
        L.ssm_state_update_zoh.restype = ctypes.c_int
        L.ssm_state_update_zoh.argtypes = L.ssm_state_update.argtypes
        L.ssm_ssd_state_update.restype = ctypes.c_int
        L.ssm_ssd_state_update.argtypes = [_I64] * 4 + [ctypes.c_int] + [_VP] * 8 + \
            [ctypes.c_int, _VP, _VP]
        L.ssm_ssd_scan_status.restype = ctypes.c_int
        L.ssm_ssd_scan_status.argtypes = [_VP]
        L.ssm_ssd_scan_fwd.restype = ctypes.c_int
        L.ssm_ssd_scan_fwd.argtypes = [_I64] * 5 + [ctypes.c_int] + [_VP] * 7 + \
            [ctypes.c_int, _VP, _VP, _VP, _VP]
        _lib = L
    return _lib


def _io_code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return SSM_DTYPE_F32
    if dtype == torch.bfloat16:
        return SSM_DTYPE_BF16
    raise TypeError(f"io tensors must be float32 or bfloat16, got {dtype}")


def _ptr(t, name, dtype=None, shape=None, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _stream_ptr(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def scan_plan(batch, seqlen, dim, dstate, dtype=torch.bfloat16) -> ScanPlan:
    out = ScanPlan()
    rc = lib().ssm_scan_plan(batch, seqlen, dim, dstate, _io_code(dtype), ctypes.byref(out))
    if rc != 0:
        raise SsmError(rc, "ssm_scan_plan")
    return out


def scan_workspace_bytes(batch, seqlen, dim, dstate, dtype=torch.bfloat16) -> int:
    return int(lib().ssm_scan_workspace_bytes(batch, seqlen, dim, dstate, _io_code(dtype)))


def ssm_scan_fwd(x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, h0=None,
                 y=None, h_last=None, workspace=None, return_last_state=True, stream=None,
                 zoh=False, return_y=True):
    """Selective scan through ssm_scan_fwd of libssmscan.so (ssm_scan_fwd_zoh
    with ``zoh=True``: the exact zero-order-hold input term).

    x, delta, z: (batch, L, dim); B, C: (batch, L, N) -- all float32 or all
    bfloat16. A: (dim, N), D and delta_bias: (dim,), h0: (batch, dim, N),
    float32. Returns (y, h_last); h_last is None when not requested, y is None
    with ``return_y=False`` (the final state only: no y is written)."""
    if x.dim() != 3:
        raise ValueError("x must be (batch, seqlen, dim)")
    batch, L, dim = x.shape
    if A.dim() != 2 or A.shape[0] != dim:
        raise ValueError("A must be (dim, dstate)")
    N = A.shape[1]
    dev = x.device
    io = _io_code(x.dtype)
    bld, bln = (batch, L, dim), (batch, L, N)
    args_io = [_ptr(x, "x", x.dtype, bld), _ptr(delta, "delta", x.dtype, bld, dev)]
    pA = _ptr(A, "A", torch.float32, (dim, N), dev)
    pB = _ptr(B, "B", x.dtype, bln, dev)
    pC = _ptr(C, "C", x.dtype, bln, dev)
    pD = _ptr(D, "D", torch.float32, (dim,), dev)
    pz = _ptr(z, "z", x.dtype, bld, dev)
    pbias = _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev)
    ph0 = _ptr(h0, "h0", torch.float32, (batch, dim, N), dev)
    if y is None and return_y:
        y = torch.empty(bld, dtype=x.dtype, device=dev)
    py = _ptr(y, "y", x.dtype, bld, dev)
    if h_last is None and (return_last_state or not return_y):
        h_last = torch.empty((batch, dim, N), dtype=torch.float32, device=dev)
    ph = _ptr(h_last, "h_last", torch.float32, (batch, dim, N), dev)
    with torch.cuda.device(dev):
        need = scan_workspace_bytes(batch, L, dim, N, x.dtype)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        pws = _ptr(workspace, "workspace", None, None, dev)
        fn = lib().ssm_scan_fwd_zoh if zoh else lib().ssm_scan_fwd
        rc = fn(batch, L, dim, N, io, args_io[0], args_io[1], pA, pB, pC, pD, pz,
                pbias, 1 if softplus else 0, ph0, py, ph, pws,
                workspace.numel() * workspace.element_size(), _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_scan_fwd_zoh" if zoh else "ssm_scan_fwd")
    return y, h_last


def scan_bwd_workspace_bytes(batch, seqlen, dim, dstate, dtype=torch.bfloat16) -> int:
    return int(lib().ssm_scan_bwd_workspace_bytes(batch, seqlen, dim, dstate, _io_code(dtype)))


def ssm_scan_bwd(x, delta, A, B, C, dy, D=None, z=None, delta_bias=None, softplus=True, h0=None,
                 dh_last=None, workspace=None, want_dD=True, want_ddelta_bias=True, want_dh0=True,
                 stream=None):
    """Gradients of the selective scan through ssm_scan_bwd of libssmscan.so,
    for the loss sum(dy * y) + sum(dh_last * h_last) (dh_last may be None).

    Inputs as for ssm_scan_fwd, plus dy (batch, L, dim) in the io dtype and
    dh_last (batch, dim, N) float32. Returns a dict: dx, ddelta, dz (io
    dtype; dz None without z), dA (dim, N), dB, dC (batch, L, N), dD,
    ddelta_bias (dim,), dh0 (batch, dim, N), all float32 except the first
    three (a gradient not asked for is None)."""
    if x.dim() != 3:
        raise ValueError("x must be (batch, seqlen, dim)")
    batch, L, dim = x.shape
    if A.dim() != 2 or A.shape[0] != dim:
        raise ValueError("A must be (dim, dstate)")
    N = A.shape[1]
    dev = x.device
    io = _io_code(x.dtype)
    bld, bln, bdn = (batch, L, dim), (batch, L, N), (batch, dim, N)
    f32 = torch.float32
    ins = [_ptr(x, "x", x.dtype, bld), _ptr(delta, "delta", x.dtype, bld, dev),
           _ptr(A, "A", f32, (dim, N), dev), _ptr(B, "B", x.dtype, bln, dev),
           _ptr(C, "C", x.dtype, bln, dev), _ptr(D, "D", f32, (dim,), dev),
           _ptr(z, "z", x.dtype, bld, dev), _ptr(delta_bias, "delta_bias", f32, (dim,), dev)]
    ph0 = _ptr(h0, "h0", f32, bdn, dev)
    pdy = _ptr(dy, "dy", x.dtype, bld, dev)
    pdh = _ptr(dh_last, "dh_last", f32, bdn, dev)
    g = {"dx": torch.empty(bld, dtype=x.dtype, device=dev),
         "ddelta": torch.empty(bld, dtype=x.dtype, device=dev),
         "dz": torch.empty(bld, dtype=x.dtype, device=dev) if z is not None else None,
         "dA": torch.empty((dim, N), dtype=f32, device=dev),
         "dB": torch.empty(bln, dtype=f32, device=dev),
         "dC": torch.empty(bln, dtype=f32, device=dev),
         "dD": torch.empty((dim,), dtype=f32, device=dev) if want_dD else None,
         "ddelta_bias": torch.empty((dim,), dtype=f32, device=dev) if want_ddelta_bias else None,
         "dh0": torch.empty(bdn, dtype=f32, device=dev) if want_dh0 else None}
    P = {k: (v.data_ptr() if v is not None else None) for k, v in g.items()}
    with torch.cuda.device(dev):
        need = scan_bwd_workspace_bytes(batch, L, dim, N, x.dtype)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        pws = _ptr(workspace, "workspace", None, None, dev)
        rc = lib().ssm_scan_bwd(batch, L, dim, N, io, *ins, 1 if softplus else 0, ph0, pdy, pdh,
                                P["dx"], P["ddelta"], P["dA"], P["dB"], P["dC"], P["dD"],
                                P["dz"], P["ddelta_bias"], P["dh0"], pws,
                                workspace.numel() * workspace.element_size(),
                                _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_scan_bwd", with_detail=True)
    return g


def ssm_conv1d_silu_fwd(x, w, bias=None, silu=True, out=None, stream=None):
    """The Mamba block's causal depthwise conv1d (+ SiLU) through
    ssm_conv1d_silu_fwd of libssmscan.so. x: (batch, L, dim) float32 or
    bfloat16; w: (dim, width) float32; bias: (dim,) float32. Returns out
    (batch, L, dim) in x's dtype."""
    if x.dim() != 3 or w.dim() != 2:
        raise ValueError("x must be (batch, seqlen, dim) and w (dim, width)")
    batch, L, dim = x.shape
    width = w.shape[1]
    dev = x.device
    px = _ptr(x, "x", x.dtype, (batch, L, dim))
    pw = _ptr(w, "w", torch.float32, (dim, width), dev)
    pb = _ptr(bias, "bias", torch.float32, (dim,), dev)
    if out is None:
        out = torch.empty((batch, L, dim), dtype=x.dtype, device=dev)
    po = _ptr(out, "out", x.dtype, (batch, L, dim), dev)
    with torch.cuda.device(dev):
        rc = lib().ssm_conv1d_silu_fwd(batch, L, dim, width, _io_code(x.dtype), px, pw, pb,
                                       1 if silu else 0, po, _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_conv1d_silu_fwd", with_detail=True)
    return out


def ssm_conv1d_silu_update(conv_state, x, w, bias=None, silu=True, out=None, stream=None):
    """One decode step of the causal conv through ssm_conv1d_silu_update of
    libssmscan.so: conv_state (batch, dim, width-1) in x's dtype (the last
    inputs, oldest first) is updated in place; returns out (batch, dim)."""
    if x.dim() != 2 or conv_state.dim() != 3:
        raise ValueError("x must be (batch, dim) and conv_state (batch, dim, width-1)")
    batch, dim = x.shape
    width = conv_state.shape[2] + 1
    dev = x.device
    ps = _ptr(conv_state, "conv_state", x.dtype, (batch, dim, width - 1), dev)
    px = _ptr(x, "x", x.dtype, (batch, dim))
    pw = _ptr(w, "w", torch.float32, (dim, width), dev)
    pb = _ptr(bias, "bias", torch.float32, (dim,), dev)
    if out is None:
        out = torch.empty((batch, dim), dtype=x.dtype, device=dev)
    po = _ptr(out, "out", x.dtype, (batch, dim), dev)
    with torch.cuda.device(dev):
        rc = lib().ssm_conv1d_silu_update(batch, dim, width, _io_code(x.dtype), ps, px, pw, pb,
                                          1 if silu else 0, po, _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_conv1d_silu_update", with_detail=True)
    return out


def conv1d_silu_bwd_workspace_bytes(batch, seqlen, dim, width, dtype=torch.bfloat16) -> int:
    return int(lib().ssm_conv1d_silu_bwd_workspace_bytes(batch, seqlen, dim, width,
                                                         _io_code(dtype)))


def ssm_conv1d_silu_bwd(x, w, dout, bias=None, silu=True, workspace=None, stream=None):
    """Gradients of sum(dout * out) for ssm_conv1d_silu_fwd: returns a dict
    dx (batch, L, dim) in x's dtype, dw (dim, width) and dbias (dim,) float32."""
    if x.dim() != 3 or w.dim() != 2:
        raise ValueError("x must be (batch, seqlen, dim) and w (dim, width)")
    batch, L, dim = x.shape
    width = w.shape[1]
    dev = x.device
    px = _ptr(x, "x", x.dtype, (batch, L, dim))
    pw = _ptr(w, "w", torch.float32, (dim, width), dev)
    pb = _ptr(bias, "bias", torch.float32, (dim,), dev)
    pg = _ptr(dout, "dout", x.dtype, (batch, L, dim), dev)
    g = {"dx": torch.empty((batch, L, dim), dtype=x.dtype, device=dev),
         "dw": torch.empty((dim, width), dtype=torch.float32, device=dev),
         "dbias": torch.empty((dim,), dtype=torch.float32, device=dev)}
    with torch.cuda.device(dev):
        need = conv1d_silu_bwd_workspace_bytes(batch, L, dim, width, x.dtype)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        pws = _ptr(workspace, "workspace", None, None, dev)
        rc = lib().ssm_conv1d_silu_bwd(batch, L, dim, width, _io_code(x.dtype), px, pw, pb,
                                       1 if silu else 0, pg, g["dx"].data_ptr(),
                                       g["dw"].data_ptr(), g["dbias"].data_ptr(), pws,
                                       workspace.numel() * workspace.element_size(),
                                       _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_conv1d_silu_bwd", with_detail=True)
    return g


def ssm_delta_sum(delta, delta_bias=None, softplus=True, out=None, stream=None):
    """dsum (batch, dim) float32 = sum over the sequence of Delta =
    softplus(delta + delta_bias), through ssm_delta_sum of libssmscan.so."""
    if delta.dim() != 3:
        raise ValueError("delta must be (batch, seqlen, dim)")
    batch, L, dim = delta.shape
    dev = delta.device
    pd = _ptr(delta, "delta", delta.dtype, (batch, L, dim))
    pb = _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev)
    if out is None:
        out = torch.empty((batch, dim), dtype=torch.float32, device=dev)
    po = _ptr(out, "out", torch.float32, (batch, dim), dev)
    with torch.cuda.device(dev):
        rc = lib().ssm_delta_sum(batch, L, dim, _io_code(delta.dtype), pd, pb, 1 if softplus else 0,
                                 po, _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_delta_sum")
    return out


def ssm_compose_carries(rank, A, hend_all, dsum_all, h0=None, out=None, stream=None):
    """The state entering chunk `rank` of a sequence cut into chunks: h0 (or
    zero) carried through chunks 0..rank-1, each given by its end state from
    zero (hend_all[r], (batch, dim, N)) and its sum of Delta (dsum_all[r],
    (batch, dim)), through ssm_compose_carries of libssmscan.so."""
    R, batch, dim, N = hend_all.shape
    dev = hend_all.device
    pA = _ptr(A, "A", torch.float32, (dim, N), dev)
    ph = _ptr(hend_all, "hend_all", torch.float32, (R, batch, dim, N), dev)
    pd = _ptr(dsum_all, "dsum_all", torch.float32, (R, batch, dim), dev)
    p0 = _ptr(h0, "h0", torch.float32, (batch, dim, N), dev)
    if not 0 <= rank <= R:
        raise ValueError("rank out of range")
    if out is None:
        out = torch.empty((batch, dim, N), dtype=torch.float32, device=dev)
    po = _ptr(out, "out", torch.float32, (batch, dim, N), dev)
    with torch.cuda.device(dev):
        rc = lib().ssm_compose_carries(rank, batch, dim, N, pA, p0, ph, pd, po,
                                       _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_compose_carries")
    return out


def ssm_scan_fwd_noalloc(x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                         h0=None, y=None, h_last=None, return_last_state=True, stream=None):
    """The selective scan through ssm_scan_fwd_noalloc of libssmscan.so.

    For callers that cannot allocate device memory around the call: the
    library takes its scratch from a 16 MiB array it reserves on each GPU, so
    apart from the outputs (allocated here only when not passed in) nothing
    is allocated. Problems needing more scratch raise SsmError (-3). Calls
    that may overlap on the GPU share that scratch and must be ordered by the
    caller. Same arguments and results as ssm_scan_fwd."""
    if x.dim() != 3:
        raise ValueError("x must be (batch, seqlen, dim)")
    batch, L, dim = x.shape
    if A.dim() != 2 or A.shape[0] != dim:
        raise ValueError("A must be (dim, dstate)")
    N = A.shape[1]
    dev = x.device
    bld, bln = (batch, L, dim), (batch, L, N)
    px = _ptr(x, "x", x.dtype, bld)
    pdl = _ptr(delta, "delta", x.dtype, bld, dev)
    pA = _ptr(A, "A", torch.float32, (dim, N), dev)
    pB = _ptr(B, "B", x.dtype, bln, dev)
    pC = _ptr(C, "C", x.dtype, bln, dev)
    pD = _ptr(D, "D", torch.float32, (dim,), dev)
    pz = _ptr(z, "z", x.dtype, bld, dev)
    pbias = _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev)
    ph0 = _ptr(h0, "h0", torch.float32, (batch, dim, N), dev)
    if y is None:
        y = torch.empty(bld, dtype=x.dtype, device=dev)
    py = _ptr(y, "y", x.dtype, bld, dev)
    if h_last is None and return_last_state:
        h_last = torch.empty((batch, dim, N), dtype=torch.float32, device=dev)
    ph = _ptr(h_last, "h_last", torch.float32, (batch, dim, N), dev)
    with torch.cuda.device(dev):
        rc = lib().ssm_scan_fwd_noalloc(batch, L, dim, N, _io_code(x.dtype), px, pdl, pA, pB, pC,
                                        pD, pz, pbias, 1 if softplus else 0, ph0, py, ph,
                                        _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_scan_fwd_noalloc", with_detail=True)
    return y, h_last


def ssm_scan_status(workspace, batch, seqlen, dim, dstate, dtype=torch.bfloat16, stream=None):
    """Synchronise the stream and return the status code of the last scan that
    used `workspace` (0 = every CTA finished; -5 = a bounded wait timed out)."""
    dev = workspace.device
    with torch.cuda.device(dev):
        return int(lib().ssm_scan_status(workspace.data_ptr(),
                                         workspace.numel() * workspace.element_size(), batch,
                                         seqlen, dim, dstate, _io_code(dtype),
                                         _stream_ptr(stream, dev)))


def ssm_scan_status_noalloc(batch, seqlen, dim, dstate, dtype=torch.bfloat16, device=None,
                            stream=None):
    """Synchronise the stream and return the status code of the last
    ssm_scan_fwd_noalloc call on the device (0 = every CTA finished; -5 = a
    bounded wait timed out), read from the library's reserved scratch."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return int(lib().ssm_scan_status_noalloc(batch, seqlen, dim, dstate, _io_code(dtype),
                                                 _stream_ptr(stream, dev)))


def ssm_ssd_scan_status(device=None, stream=None):
    """Synchronise the stream and return 0, or -5 if a CTA of an SSD scan on
    the device gave up a bounded wait since the last call (the flag is then
    cleared)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return int(lib().ssm_ssd_scan_status(_stream_ptr(stream, dev)))


def ssm_state_update(state, x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                     y=None, stream=None, zoh=False):
    """One decode step through ssm_state_update of libssmscan.so
    (ssm_state_update_zoh with ``zoh=True``); updates the float32 state
    (batch, dim, N) in place and returns y (batch, dim)."""
    if state.dim() != 3:
        raise ValueError("state must be (batch, dim, dstate)")
    batch, dim, N = state.shape
    dev = state.device
    io = _io_code(x.dtype)
    bd, bn = (batch, dim), (batch, N)
    ps = _ptr(state, "state", torch.float32, (batch, dim, N))
    px = _ptr(x, "x", x.dtype, bd, dev)
    pdl = _ptr(delta, "delta", x.dtype, bd, dev)
    pA = _ptr(A, "A", torch.float32, (dim, N), dev)
    pB = _ptr(B, "B", x.dtype, bn, dev)
    pC = _ptr(C, "C", x.dtype, bn, dev)
    pD = _ptr(D, "D", torch.float32, (dim,), dev)
    pz = _ptr(z, "z", x.dtype, bd, dev)
    pbias = _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev)
    if y is None:
        y = torch.empty(bd, dtype=x.dtype, device=dev)
    py = _ptr(y, "y", x.dtype, bd, dev)
    with torch.cuda.device(dev):
        fn = lib().ssm_state_update_zoh if zoh else lib().ssm_state_update
        rc = fn(batch, dim, N, io, ps, px, pdl, pA, pB, pC, pD, pz, pbias,
                1 if softplus else 0, py, _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_state_update_zoh" if zoh else "ssm_state_update")
    return y


def ssm_ssd_scan_fwd(x, dt, A, B, C, D=None, dt_bias=None, softplus=True, h0=None,
                     return_last_state=False, y=None, stream=None, h_last=None):
    """The multi-head SSD scan through ssm_ssd_scan_fwd of libssmscan.so:
    x (batch, L, heads, headdim) bf16, dt (batch, L, heads) bf16, A (heads,)
    fp32, B, C (batch, L, dstate) bf16, D and dt_bias (heads,) fp32 or None,
    h0 (batch, heads, headdim, dstate) fp32 or None. Returns y (and h_last
    with ``return_last_state``; ``h_last`` may be given, and may be h0)."""
    if x.dim() != 4:
        raise ValueError("x must be (batch, seqlen, heads, headdim)")
    batch, L, H, P = x.shape
    N = B.shape[-1]
    dev = x.device
    io = _io_code(x.dtype)
    px = _ptr(x, "x", x.dtype)
    pdt = _ptr(dt, "dt", x.dtype, (batch, L, H), dev)
    pA = _ptr(A, "A", torch.float32, (H,), dev)
    pB = _ptr(B, "B", x.dtype, (batch, L, N), dev)
    pC = _ptr(C, "C", x.dtype, (batch, L, N), dev)
    pD = _ptr(D, "D", torch.float32, (H,), dev)
    pbias = _ptr(dt_bias, "dt_bias", torch.float32, (H,), dev)
    ph0 = _ptr(h0, "h0", torch.float32, (batch, H, P, N), dev)
    if y is None:
        y = torch.empty((batch, L, H, P), dtype=x.dtype, device=dev)
    py = _ptr(y, "y", x.dtype, (batch, L, H, P), dev)
    if h_last is None and return_last_state:
        h_last = torch.empty((batch, H, P, N), dtype=torch.float32, device=dev)
    ph = _ptr(h_last, "h_last", torch.float32, (batch, H, P, N), dev)
    with torch.cuda.device(dev):
        rc = lib().ssm_ssd_scan_fwd(batch, L, H, P, N, io, px, pdt, pA, pB, pC, pD, pbias,
                                    1 if softplus else 0, ph0, py, ph, _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_ssd_scan_fwd", with_detail=True)
    return (y, h_last) if return_last_state else y


def ssm_ssd_state_update(state, x, dt, A, B, C, D=None, dt_bias=None, softplus=True, y=None,
                         stream=None):
    """One SSD decode step through ssm_ssd_state_update of libssmscan.so:
    updates the float32 state (batch, heads, headdim, dstate) in place and
    returns y (batch, heads, headdim) in x's dtype."""
    if state.dim() != 4:
        raise ValueError("state must be (batch, heads, headdim, dstate)")
    batch, H, P, N = state.shape
    dev = state.device
    io = _io_code(x.dtype)
    ps = _ptr(state, "state", torch.float32)
    px = _ptr(x, "x", x.dtype, (batch, H, P), dev)
    pdt = _ptr(dt, "dt", x.dtype, (batch, H), dev)
    pA = _ptr(A, "A", torch.float32, (H,), dev)
    pB = _ptr(B, "B", x.dtype, (batch, N), dev)
    pC = _ptr(C, "C", x.dtype, (batch, N), dev)
    pD = _ptr(D, "D", torch.float32, (H,), dev)
    pbias = _ptr(dt_bias, "dt_bias", torch.float32, (H,), dev)
    if y is None:
        y = torch.empty((batch, H, P), dtype=x.dtype, device=dev)
    py = _ptr(y, "y", x.dtype, (batch, H, P), dev)
    with torch.cuda.device(dev):
        rc = lib().ssm_ssd_state_update(batch, H, P, N, io, ps, px, pdt, pA, pB, pC, pD, pbias,
                                        1 if softplus else 0, py, _stream_ptr(stream, dev))
    if rc != 0:
        raise SsmError(rc, "ssm_ssd_state_update", with_detail=True)
    return y


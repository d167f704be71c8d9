"""Helpers shared by the GPU parity tests: moving generator output to the
device, calling the CUDA path, and the parity metric."""
import numpy as np
import torch

import ssm_inputs as gen

# Parity bound: max|y - y_ref| / max|y_ref| (and the same for h_last).
TOL = {"f32": 1e-5, "bf16": 1e-2}


def dev(a, io="f32"):
    """numpy generator output -> CUDA tensor (bf16 arrays are uint16 bits)."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    """CUDA tensor -> float64 numpy."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    num = np.max(np.abs(got - ref))
    return float(num / den) if den > 0 else float(num)


def gpu_scan(inp, softplus=True, **kw):
    from selective_state_space_39_b200 import ssm_scan_fwd
    return ssm_scan_fwd(dev(inp["x"]), dev(inp["delta"]), dev(inp["A"]), dev(inp["B"]),
                        dev(inp["C"]), D=dev(inp.get("D")), z=dev(inp.get("z")),
                        delta_bias=dev(inp.get("delta_bias")), softplus=softplus,
                        h0=dev(inp.get("h0")), **kw)


def oracle_scan(inp, io, softplus=True, channels=None, nthreads=None):
    import oracle
    return oracle.selective_scan(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                 D=inp.get("D"), z=inp.get("z"), delta_bias=inp.get("delta_bias"),
                                 softplus=softplus, h0=inp.get("h0"), io=io, channels=channels,
                                 nthreads=nthreads or gen.default_threads())


def sample_channels(batch, dim, per_batch=16, seed=0):
    """Channels to check at full size: tile edges plus random ones."""
    rng = np.random.default_rng(seed)
    edges = [0, 1, 127, 128, 254, 255, 256, 257, dim // 2, dim - 2, dim - 1]
    chans = []
    for b in sorted(set([0, batch - 1] + list(rng.integers(0, batch, 2)))):
        ds = set(d for d in edges if 0 <= d < dim) | set(rng.integers(0, dim, per_batch).tolist())
        chans += [(int(b), int(d)) for d in sorted(ds)]
    return chans

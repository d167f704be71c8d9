"""GPU parity of the decode state update (through the C ABI) against the
oracle's sequential loop over the same tokens."""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as gen
from tests.gpu_util import TOL, dev, gpu_scan, host, rel_err

pytestmark = pytest.mark.gpu


def test_decode_workload_1000_steps():
    """B=128 sequences, D=4096, N=16, bf16: 1000 carried steps; the oracle
    runs the same 1000 steps on sampled (batch, channel) pairs."""
    from selective_state_space_39_b200 import ssm_state_update
    w = gen.DECODE_WORKLOADS["decode_b128_d4096_x1000"]
    const = gen.decode_constants(w.dim, w.dstate, w.seed)
    A, D, bias = dev(const["A"]), dev(const["D"]), dev(const["delta_bias"])
    state = torch.zeros((w.batch, w.dim, w.dstate), dtype=torch.float32, device="cuda")
    bs = np.array([0, 1, 63, 127])
    ds = np.array([0, 1, 2, 3, 255, 256, 1000, 2047, 2048, 4094, 4095])
    ref_state = np.zeros((len(bs), len(ds), w.dstate))
    sub = lambda a: np.ascontiguousarray(a[bs][:, ds])
    ys, yrs = [], []
    for step in range(w.steps):
        inp = gen.make_decode_inputs(w.batch, w.dim, w.dstate, w.io, w.seed, step)
        y = ssm_state_update(state, dev(inp["x"]), dev(inp["delta"]), A, dev(inp["B"]),
                             dev(inp["C"]), D=D, z=dev(inp["z"]), delta_bias=bias)
        ys.append(host(y)[bs][:, ds])
        yrs.append(oracle.state_update(ref_state, sub(inp["x"]), sub(inp["delta"]),
                                       np.ascontiguousarray(const["A"][ds]),
                                       np.ascontiguousarray(inp["B"][bs]),
                                       np.ascontiguousarray(inp["C"][bs]), D=const["D"][ds],
                                       z=sub(inp["z"]), delta_bias=const["delta_bias"][ds],
                                       io=w.io))
    hs = host(state)[bs][:, ds]
    ey, eh = rel_err(np.stack(ys), np.stack(yrs)), rel_err(hs, ref_state)
    print(f"decode 1000 steps: rel err y {ey:.3e} state {eh:.3e}")
    assert torch.isfinite(state).all()
    assert ey <= TOL["bf16"] and eh <= TOL["bf16"]


@pytest.mark.parametrize("N", [2, 4, 8, 16, 32, 64])
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("optional", [True, False])
def test_decode_shapes(N, io, optional):
    from selective_state_space_39_b200 import ssm_state_update
    batch, dim, steps = 3, 130, 12
    seed = N + (7 if optional else 0)
    const = gen.decode_constants(dim, N, seed)
    rng = np.random.default_rng(seed)
    A = (-rng.uniform(0.2, 3.0, (dim, N))).astype(np.float32) if N != 16 else const["A"]
    state = torch.from_numpy(rng.standard_normal((batch, dim, N)).astype(np.float32)).cuda()
    ref = host(state).copy()
    for step in range(steps):
        inp = gen.make_decode_inputs(batch, dim, N, io, seed, step)
        kw = dict(D=const["D"], z=inp["z"], delta_bias=const["delta_bias"]) if optional else {}
        y = ssm_state_update(state, dev(inp["x"]), dev(inp["delta"]), dev(A), dev(inp["B"]),
                             dev(inp["C"]), **{k: dev(v) for k, v in kw.items()})
        yr = oracle.state_update(ref, inp["x"], inp["delta"], A, inp["B"], inp["C"], io=io, **kw)
        assert rel_err(host(y), yr) <= TOL[io], f"step {step}"
    assert rel_err(host(state), ref) <= TOL[io]


def test_decode_steps_equal_the_scan():
    """L decode steps on the GPU match one GPU scan over the same tokens."""
    from selective_state_space_39_b200 import ssm_state_update
    inp = gen.make_scan_inputs(2, 40, 256, 16, "f32", 31, with_h0=True)
    y, hl = gpu_scan(inp)
    state = dev(inp["h0"]).clone()
    for t in range(40):
        yt = ssm_state_update(state, dev(np.ascontiguousarray(inp["x"][:, t])),
                              dev(np.ascontiguousarray(inp["delta"][:, t])), dev(inp["A"]),
                              dev(np.ascontiguousarray(inp["B"][:, t])),
                              dev(np.ascontiguousarray(inp["C"][:, t])), D=dev(inp["D"]),
                              z=dev(np.ascontiguousarray(inp["z"][:, t])),
                              delta_bias=dev(inp["delta_bias"]))
        assert rel_err(host(yt), host(y)[:, t]) <= 1e-5
    assert rel_err(host(state), host(hl)) <= 1e-5


@pytest.mark.parametrize("N,batch,dim", [(8, 80, 4001), (64, 11, 3791)])
def test_decode_large_ragged(N, batch, dim):
    """Large grids (over 600k threads) with a ragged last block: every output
    and state element against the oracle."""
    from selective_state_space_39_b200 import ssm_state_update
    seed = 40 + N
    const = gen.decode_constants(dim, N, seed)
    rng = np.random.default_rng(seed)
    A = (-rng.uniform(0.2, 3.0, (dim, N))).astype(np.float32)
    state = torch.from_numpy(rng.standard_normal((batch, dim, N)).astype(np.float32)).cuda()
    ref = host(state).copy()
    for step in range(3):
        inp = gen.make_decode_inputs(batch, dim, N, "bf16", seed, step)
        kw = dict(D=const["D"], z=inp["z"], delta_bias=const["delta_bias"])
        y = ssm_state_update(state, dev(inp["x"]), dev(inp["delta"]), dev(A), dev(inp["B"]),
                             dev(inp["C"]), **{k: dev(v) for k, v in kw.items()})
        yr = oracle.state_update(ref, inp["x"], inp["delta"], A, inp["B"], inp["C"], io="bf16",
                                 **kw)
        assert rel_err(host(y), yr) <= TOL["bf16"], f"step {step}"
    assert rel_err(host(state), ref) <= TOL["bf16"]


@pytest.mark.parametrize("N,io,optional,batch,dim", [
    (16, "f32", True, 8, 768), (16, "bf16", True, 8, 768), (16, "bf16", False, 8, 768),
    (16, "f32", False, 8, 768), (32, "f32", True, 4, 384), (32, "bf16", False, 12, 384),
    (64, "bf16", True, 4, 192), (64, "f32", False, 8, 192),
    (16, "bf16", True, 96, 4096),  # 1536 tiles: several per CTA
])
def test_pipelined_decode_shapes(monkeypatch, N, io, optional, batch, dim):
    """Shapes the pipelined decode kernel takes (batch a multiple of 4, whole
    tiles of 1024 / N channels, 16-byte aligned rows): against the oracle step
    by step, and bit for bit against the one-shot kernel
    (the default), which does the same arithmetic."""
    from selective_state_space_39_b200 import ssm_state_update
    steps = 6 if batch < 96 else 3
    seed = 100 + N + (7 if optional else 0)
    const = gen.decode_constants(dim, N, seed)
    rng = np.random.default_rng(seed)
    A = (-rng.uniform(0.2, 3.0, (dim, N))).astype(np.float32) if N != 16 else const["A"]
    h0 = rng.standard_normal((batch, dim, N)).astype(np.float32)
    ref = h0.astype(np.float64)
    s2, s1 = dev(h0).clone(), dev(h0).clone()
    for step in range(steps):
        inp = gen.make_decode_inputs(batch, dim, N, io, seed, step)
        kw = dict(D=const["D"], z=inp["z"], delta_bias=const["delta_bias"]) if optional else {}
        args = (dev(inp["x"]), dev(inp["delta"]), dev(A), dev(inp["B"]), dev(inp["C"]))
        dkw = {k: dev(v) for k, v in kw.items()}
        monkeypatch.setenv("SSM_DECODE_PIPELINED", "1")
        y2 = ssm_state_update(s2, *args, **dkw)
        monkeypatch.delenv("SSM_DECODE_PIPELINED")
        y1 = ssm_state_update(s1, *args, **dkw)
        yr = oracle.state_update(ref, inp["x"], inp["delta"], A, inp["B"], inp["C"], io=io, **kw)
        assert rel_err(host(y2), yr) <= TOL[io], f"step {step}"
        assert torch.equal(y1, y2) and torch.equal(s1, s2), f"step {step}"
    assert rel_err(host(s2), ref) <= TOL[io]


@pytest.mark.gpu
@pytest.mark.parametrize("batch,dim,N,io", [(65535, 6, 4, "f32"), (3, 100, 16, "bf16")])
def test_one_shot_decode_grid_edges(monkeypatch, batch, dim, N, io):
    """The one-shot decode kernel's grid: the largest batch the library takes
    (one grid row per batch row) and a partial last block of channels,
    against the oracle step."""
    from selective_state_space_39_b200 import ssm_state_update
    monkeypatch.delenv("SSM_DECODE_PIPELINED", raising=False)
    seed = 500 + N
    rng = np.random.default_rng(seed)
    A = (-rng.uniform(0.2, 3.0, (dim, N))).astype(np.float32)
    const = gen.decode_constants(dim, N, seed)
    h0 = rng.standard_normal((batch, dim, N)).astype(np.float32)
    ref = h0.astype(np.float64)
    s = dev(h0).clone()
    for step in range(2):
        inp = gen.make_decode_inputs(batch, dim, N, io, seed, step)
        kw = dict(D=const["D"], z=inp["z"], delta_bias=const["delta_bias"])
        y = ssm_state_update(s, dev(inp["x"]), dev(inp["delta"]), dev(A), dev(inp["B"]),
                             dev(inp["C"]), **{k: dev(v) for k, v in kw.items()})
        yr = oracle.state_update(ref, inp["x"], inp["delta"], A, inp["B"], inp["C"], io=io, **kw)
        assert rel_err(host(y), yr) <= TOL[io], f"step {step}"
    assert rel_err(host(s), ref) <= TOL[io]

"""The N > 1 path on CPU: two gloo ranks each take their batch shard (no
data-path collective), run the scan on it -- here the fp64 oracle, since this
machine has no GPU -- and the gathered shards equal one scan over the whole
batch. Also checks the shard arithmetic and the max-over-ranks timing
reduction that bench.py uses."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from selective_state_space_39_b200 import dist as sdist


def test_batch_shard_covers_the_batch_once():
    for global_batch in (0, 1, 7, 8, 13):
        for world in (1, 2, 3, 4, 8):
            seen = []
            for r in range(world):
                s, n = sdist.batch_shard(global_batch, world, r)
                seen += list(range(s, s + n))
            assert seen == list(range(global_batch))
            sizes = [sdist.batch_shard(global_batch, world, r)[1] for r in range(world)]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sdist.batch_shard(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle
    import ssm_inputs as gen
    r, w = sdist.init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    global_batch, L, dim, N = 5, 40, 24, 16
    b0, nb = sdist.batch_shard(global_batch, world, rank)
    inp = gen.make_scan_inputs(nb, L, dim, N, "bf16", 7, with_h0=True, batch_offset=b0)
    y, hl = oracle.selective_scan(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                  z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"], io="bf16")
    # gather shards on every rank (test-only check; the bench path has no data collective)
    parts = [None] * world
    dist.all_gather_object(parts, (b0, y, hl))
    t = sdist.max_over_ranks(float(rank + 1))
    sdist.barrier()
    if rank == 0:
        parts.sort(key=lambda p: p[0])
        np.save(os.path.join(out_dir, "y.npy"), np.concatenate([p[1] for p in parts]))
        np.save(os.path.join(out_dir, "h.npy"), np.concatenate([p[2] for p in parts]))
        np.save(os.path.join(out_dir, "t.npy"), np.array([t]))
    sdist.finish()


def test_two_gloo_ranks_shard_the_batch(tmp_path):
    import oracle
    import ssm_inputs as gen
    oracle.get()  # build the oracle library before the ranks start
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    inp = gen.make_scan_inputs(5, 40, 24, 16, "bf16", 7, with_h0=True)
    y, hl = oracle.selective_scan(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                  z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"], io="bf16")
    assert np.array_equal(np.load(tmp_path / "y.npy"), y)
    assert np.array_equal(np.load(tmp_path / "h.npy"), hl)
    assert np.load(tmp_path / "t.npy")[0] == 2.0  # max over ranks


# --------------------------------------------------------------------------
# one sequence split across ranks: the product's orchestration
# (selective_state_space_39_b200.seqpar.seq_parallel_scan: carry, all-gather,
# compose, second pass) over gloo, with the compute steps taken by the fp64
# oracle since this machine has no GPU.
class _OracleOps:
    @staticmethod
    def chunk_carry(x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True):
        import oracle
        np_ = lambda t: None if t is None else t.numpy()  # noqa: E731
        _, e = oracle.selective_scan(np_(x), np_(delta), np_(A), np_(B), np_(C), D=np_(D),
                                     z=np_(z), delta_bias=np_(delta_bias), softplus=softplus)
        v = x.new_tensor(delta.numpy().astype(np.float64) + delta_bias.numpy()[None, None, :],
                         dtype=torch.float64)
        dt = torch.where(v > 20, v, torch.log1p(torch.exp(torch.clamp(v, max=20))))
        return torch.from_numpy(e), dt.sum(dim=1)

    @staticmethod
    def entering_state(rank, A, hend_all, dsum_all, h0=None):
        h = h0.double().clone() if h0 is not None else torch.zeros_like(hend_all[0])
        for r in range(rank):
            h = torch.exp(A.double()[None] * dsum_all[r][..., None]) * h + hend_all[r]
        return h

    @staticmethod
    def scan(x, delta, A, B, C, D, z, delta_bias, softplus, h0):
        import oracle
        y, hl = oracle.selective_scan(x.numpy(), delta.numpy(), A.numpy(), B.numpy(), C.numpy(),
                                      D=D.numpy(), z=z.numpy(), delta_bias=delta_bias.numpy(),
                                      softplus=softplus, h0=h0.float().numpy())
        return torch.from_numpy(y), torch.from_numpy(hl)


CUTS = (0, 33, 70, 120)  # three ranks, uneven chunks


def _seqpar_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import ssm_inputs as gen
    from selective_state_space_39_b200.seqpar import seq_parallel_scan
    sdist.init("gloo", timeout_s=60)
    inp = gen.make_scan_inputs(2, CUTS[-1], 24, 16, "f32", 9, with_h0=True)
    a, b = CUTS[rank], CUTS[rank + 1]
    t = {k: torch.from_numpy(np.ascontiguousarray(v[:, a:b] if k in ("x", "delta", "z", "B", "C")
                                                  else v)) for k, v in inp.items()}
    y, h = seq_parallel_scan(t["x"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                             delta_bias=t["delta_bias"], h0=t["h0"], ops=_OracleOps)
    parts = [None] * world
    dist.all_gather_object(parts, (rank, y.numpy(), h.numpy()))
    if rank == 0:
        parts.sort(key=lambda p: p[0])
        np.save(os.path.join(out_dir, "y.npy"), np.concatenate([p[1] for p in parts], axis=1))
        np.save(os.path.join(out_dir, "h.npy"), parts[-1][2])
    sdist.finish()


def test_three_gloo_ranks_split_one_sequence(tmp_path):
    import oracle
    import ssm_inputs as gen
    oracle.get()
    world, port = 3, _free_port()
    mp.start_processes(_seqpar_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    inp = gen.make_scan_inputs(2, CUTS[-1], 24, 16, "f32", 9, with_h0=True)
    y, hl = oracle.selective_scan(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                  z=inp["z"], delta_bias=inp["delta_bias"], h0=inp["h0"])
    # the entering states pass through fp32 (the h0 argument): 1e-6
    assert np.allclose(np.load(tmp_path / "y.npy"), y, rtol=1e-6, atol=1e-6)
    assert np.allclose(np.load(tmp_path / "h.npy"), hl, rtol=1e-6, atol=1e-6)

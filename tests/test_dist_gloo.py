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

"""The multi-GPU path's host logic on CPU: shard ranges, max-over-ranks timing and the
sharded top-k search merge ("TurboQuant: redefining AI efficiency", "Impact on
high-dimensional vector search"), with two gloo ranks on 127.0.0.1. The per-shard
scores come from the oracle, so the merged answer can be compared with the oracle's
search over the whole database."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from embedding_vector_quantization_b200 import dist as tqdist
from oracle import codebook, ops, quant, rotation


def test_shard_range_covers_and_balances():
    for n in (0, 1, 7, 10, 1000, 1001):
        for world in (1, 2, 3, 8):
            rs = [tqdist.shard_range(n, r, world) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == n
            assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
            sizes = [hi - lo for lo, hi in rs]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        tqdist.shard_range(10, 2, 2)


def _db(n=300, nq=6, d=32, bits=2, seed=3):
    Pi = rotation.rotation(d, seed, 0)[0]
    c, beta = codebook.lloyd_max(d, bits)
    rs = np.random.default_rng(seed)
    x = rs.standard_normal((n, d))
    e = quant.encode_mse(x, Pi, c, beta, "f32")
    q = rs.standard_normal((nq, d))
    return ops.search_scores(q, e["idx"], e["n_stored"], Pi, c)


def test_merge_topk_equals_global_topk_with_ties():
    s = _db()
    s[:, 40] = s[:, 200]          # equal scores across shards: lower index must win
    s[:, 41] = s[:, 41].max() + 1  # a clear winner
    k = 10
    gi, gs = ops.topk(s, k)
    parts = []
    for r in range(3):
        lo, hi = tqdist.shard_range(s.shape[1], r, 3)
        li, ls = ops.topk(s[:, lo:hi], k)
        parts.append((li + lo, ls))
    mi, ms = tqdist.merge_topk(torch.from_numpy(np.concatenate([p[0] for p in parts], 1)),
                               torch.from_numpy(np.concatenate([p[1] for p in parts], 1)), k)
    assert np.array_equal(mi.numpy(), gi) and np.array_equal(ms.numpy(), gs)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        mx = tqdist.max_over_ranks(1.5 + rank)
        s = _db()
        k = 10
        lo, hi = tqdist.shard_range(s.shape[1], rank, world)
        li, ls = ops.topk(s[:, lo:hi], k)
        mi, ms = tqdist.gather_topk(torch.from_numpy(li + lo), torch.from_numpy(ls), k)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), mx=mx, idx=mi.numpy(), score=ms.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_sharded_search(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    gi, gs = ops.topk(_db(), 10)
    for r in range(world):
        z = np.load(tmp_path / f"r{r}.npz")
        assert float(z["mx"]) == 2.5
        assert np.array_equal(z["idx"], gi) and np.array_equal(z["score"], gs)

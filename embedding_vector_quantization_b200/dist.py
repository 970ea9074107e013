"""Host-side plumbing of the multi-GPU path (one process per GPU, torch.distributed).

The hot path shards by independent units, so nothing on the data path is exchanged:
  * KV paths: (sequence, KV head) units; each rank encodes, appends and attends over its
    own units ("replicas" of the decode step in the bench: weak scaling).
  * Search: database rows are split into contiguous ranges (`shard_range`); each rank
    returns its local top-k with global row indices and one all-gather of the
    (index, score) lists (`gather_topk`) lets every rank merge them (`merge_topk`) into the
    global top-k -- the same answer as one search over the whole database, equal scores
    ordered by lower index ("TurboQuant: redefining AI efficiency", "Impact on
    high-dimensional vector search").
  * Timing: every rank times its own work; the job's time is the maximum over ranks
    (`max_over_ranks`).
All of this is independent of the device: the tests run it on CPU with the gloo backend.
"""

import torch


def shard_range(n, rank, world):
    """Contiguous range [lo, hi) of n units owned by `rank`; sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(value, group=None):
    """The maximum of a per-rank float over all ranks (the value itself without a process group)."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device="cuda" if dist.get_backend(group) == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def merge_topk(idx, score, k):
    """Merges candidate lists idx/score [nq, c] into the top k per row: descending score,
    equal scores by lower index. Returns (idx [nq, k] int64, score [nq, k])."""
    idx = idx.to(torch.int64)
    # order by index first, then a stable sort by descending score keeps lower index first on ties
    o = torch.argsort(idx, dim=1, stable=True)
    idx, score = idx.gather(1, o), score.gather(1, o)
    o = torch.argsort(score, dim=1, descending=True, stable=True)[:, :k]
    return idx.gather(1, o), score.gather(1, o)


def gather_topk(idx, score, k, group=None):
    """All-gathers every rank's local top-k (global indices) and merges them on every rank."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return merge_topk(idx, score, k)
    world = dist.get_world_size(group)
    idx_l = [torch.empty_like(idx) for _ in range(world)]
    sc_l = [torch.empty_like(score) for _ in range(world)]
    dist.all_gather(idx_l, idx.contiguous(), group=group)
    dist.all_gather(sc_l, score.contiguous(), group=group)
    return merge_topk(torch.cat(idx_l, dim=1), torch.cat(sc_l, dim=1), k)

"""Splitting one decode layer across ranks by kv-head (tensor-parallel style).

Every (sequence, kv-head) group of the step is independent: selection, estimate, top-p, union and
attention never look at another group ([Summary] B.2: GQA groups are processed separately; the
union is per group).  So a layer splits across W ranks by kv-heads with no exchange inside the
step: rank r owns kv-heads [r Hkv / W, (r + 1) Hkv / W), their paged K/V (and the INT4 copy and
page bounds derived from them), and the q-heads of those groups; the page table and sequence
lengths are the same on every rank.  When a caller needs the whole layer's output on every rank,
one all-gather of o and lse along the q-head axis assembles it.

Host logic only (array slicing and one collective); the step itself runs in libtwl.so on each
rank's shard.
"""
from __future__ import annotations


def kv_head_range(num_kv_heads: int, rank: int, world: int) -> tuple[int, int]:
    """The kv-heads [lo, hi) rank `rank` of `world` owns (contiguous, sizes differing by <= 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if num_kv_heads < world:
        raise ValueError(f"{num_kv_heads} kv-heads cannot be split over {world} ranks")
    lo = num_kv_heads * rank // world
    hi = num_kv_heads * (rank + 1) // world
    return lo, hi


def shard_layer(k, v, q, num_q_heads: int, num_kv_heads: int, rank: int, world: int):
    """The rank's slices of one layer: K and V [P][Hkv][16][128] along the kv-head axis, q
    [B][Hq][128] along the q-head axis (the q-heads of the owned groups).  Works on numpy arrays
    and torch tensors alike; the slices are returned as contiguous copies, the layout the library
    reads.  Returns (k, v, q, num_q_heads, num_kv_heads) of the shard."""
    if num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    g = num_q_heads // num_kv_heads
    lo, hi = kv_head_range(num_kv_heads, rank, world)

    def dense(x):
        if hasattr(x, "contiguous"):
            return x.contiguous()
        import numpy as np
        return np.ascontiguousarray(x)

    return (dense(k[:, lo:hi]), dense(v[:, lo:hi]), dense(q[:, g * lo:g * hi]), g * (hi - lo),
            hi - lo)


def gather_heads(o_local, lse_local, num_q_heads: int, num_kv_heads: int, world: int, group=None):
    """All-gather every rank's (o [B][hq_r][128], lse [B][hq_r]) into the whole layer's
    (o [B][Hq][128], lse [B][Hq]) on every rank (torch.distributed, any backend)."""
    import torch
    import torch.distributed as dist
    g = num_q_heads // num_kv_heads
    # shards differ by at most one group: pad to the largest, gather, then cut
    widths = [g * (kv_head_range(num_kv_heads, r, world)[1] - kv_head_range(num_kv_heads, r, world)[0])
              for r in range(world)]
    wmax = max(widths)
    b = o_local.shape[0]
    o_pad = o_local.new_zeros((b, wmax) + tuple(o_local.shape[2:]))
    l_pad = lse_local.new_zeros((b, wmax))
    o_pad[:, :o_local.shape[1]] = o_local
    l_pad[:, :lse_local.shape[1]] = lse_local
    o_all = [torch.empty_like(o_pad) for _ in range(world)]
    l_all = [torch.empty_like(l_pad) for _ in range(world)]
    dist.all_gather(o_all, o_pad, group=group)
    dist.all_gather(l_all, l_pad, group=group)
    o = torch.cat([o_all[r][:, :widths[r]] for r in range(world)], dim=1)
    lse = torch.cat([l_all[r][:, :widths[r]] for r in range(world)], dim=1)
    return o, lse

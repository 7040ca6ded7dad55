"""Key-sharded attention over several GPUs: one process per GPU, each holding all of Q and
a contiguous shard of K and V.  Each rank computes its shard's partial (O_r, LSE_r) with
fa_fwd_partial, the partials are exchanged in one all-gather (NCCL over NVLink), and every
rank merges them with fa_merge_partials, so every rank ends with the full O and LSE.

The exchange is the only step that crosses GPUs; everything else is this library's
kernels.  The gather is split out (gather_partials) so that its plumbing runs on any
torch.distributed backend."""
from __future__ import annotations

from . import fa_fwd_partial, fa_merge_partials


def shard_range(nk_total: int, rank: int, world: int) -> tuple[int, int]:
    """(key_offset, length) of rank's contiguous shard: the first nk_total % world ranks
    take one key more."""
    if world < 1 or not 0 <= rank < world or nk_total < 0:
        raise ValueError(f"bad shard request: nk_total={nk_total} rank={rank} world={world}")
    base, extra = divmod(nk_total, world)
    length = base + (1 if rank < extra else 0)
    offset = rank * base + min(rank, extra)
    return offset, length


def gather_partials(o_part, lse_part, group=None):
    """All-gather every rank's partial, stacked in rank order: ([R, ...], [R, ...])."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    stacked = []
    for t in (o_part.contiguous(), lse_part.contiguous()):
        # gathered concatenated along dim 0 (what every backend accepts), viewed stacked
        g = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(g, t, group=group)
        stacked.append(g.view((world,) + tuple(t.shape)))
    return stacked[0], stacked[1]


def kshard_attention(q, k_shard, v_shard, *, key_offset: int, nk_total: int, causal: bool = False,
                     scale: float | None = None, group=None):
    """Exact attention of q over the union of every rank's key shard.  Returns (out bf16
    [B, Nq, Hq, d], lse fp32 [B, Hq, Nq]), the same on every rank."""
    o_part, lse_part = fa_fwd_partial(q, k_shard, v_shard, key_offset=key_offset, nk_total=nk_total,
                                      causal=causal, scale=scale)
    o_all, l_all = gather_partials(o_part, lse_part, group)
    return fa_merge_partials(o_all, l_all)

"""Key-sharded attention over several GPUs: one process per GPU, each holding all of Q and
a contiguous shard of K and V.  Each rank computes its shard's partial (O_r, LSE_r) with
fa_fwd_partial; the partials are exchanged by query rows in one all-to-all (NCCL over
NVLink), so that rank s receives every rank's partial for its own block of the B*Nq query
rows only; each rank merges its block with fa_merge_partials.  Optionally the merged bf16
rows are all-gathered so that every rank ends with the full O and LSE.

Bytes a rank receives, with |O| = B*Nq*Hq*d values: (R-1)/R * |O| * 4 in the all-to-all
(fp32 partials) plus (R-1)/R * |O| * 2 in the optional bf16 all-gather, against
(R-1) * |O| * 4 when every rank gathers every partial; the merge work per rank is 1/R of
the rows.  LSE adds 1/d of those figures.

The exchange is the only step that crosses GPUs; everything else is this library's
kernels.  It is split out (exchange_partials, gather_rows) so that its plumbing runs on
any torch.distributed backend."""
from __future__ import annotations

from . import fa_fwd_partial, fa_merge_partials


def shard_range(n_total: int, rank: int, world: int) -> tuple[int, int]:
    """(offset, length) of rank's contiguous share of n_total items (keys or query rows):
    the first n_total % world ranks take one more."""
    if world < 1 or not 0 <= rank < world or n_total < 0:
        raise ValueError(f"bad shard request: n_total={n_total} rank={rank} world={world}")
    base, extra = divmod(n_total, world)
    length = base + (1 if rank < extra else 0)
    offset = rank * base + min(rank, extra)
    return offset, length


def send_blocks(o_part, lse_part, world: int):
    """This rank's partial cut by destination: o_part [B, Nq, Hq, d] and lse_part [B, Hq, Nq]
    become the row-major send buffers o_send [B*Nq, Hq*d] and l_send [B*Nq, Hq] plus the row
    count of each destination's block (contiguous blocks of flat rows (b, i), rank order)."""
    B, Nq, Hq, d = o_part.shape
    rows = B * Nq
    sizes = [shard_range(rows, r, world)[1] for r in range(world)]
    o_send = o_part.contiguous().view(rows, Hq * d)            # row blocks are contiguous
    l_send = lse_part.permute(0, 2, 1).reshape(rows, Hq).contiguous()
    return o_send, l_send, sizes


def received_layout(o_recv, l_recv, world: int, n: int, Hq: int, d: int):
    """The received blocks (o_recv [R*n, Hq*d], l_recv [R*n, Hq], source-rank order) in the
    layout fa_merge_partials takes: ([R, 1, n, Hq, d], [R, 1, Hq, n])."""
    return (o_recv.view(world, 1, n, Hq, d),
            l_recv.view(world, n, Hq).permute(0, 2, 1).contiguous().view(world, 1, Hq, n))


def exchange_partials(o_part, lse_part, group=None):
    """All-to-all by query rows.  o_part [B, Nq, Hq, d] fp32 and lse_part [B, Hq, Nq] fp32 are
    this rank's partial over its key shard; the B*Nq rows (b, i) are cut into contiguous
    blocks in rank order (shard_range).  Returns (o_parts [R, 1, n, Hq, d], lse_parts
    [R, 1, Hq, n], (row0, n)): every rank's partial for this rank's n rows starting at flat
    row row0, stacked in rank order -- the layout fa_merge_partials takes."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, Nq, Hq, d = o_part.shape
    o_send, l_send, sizes = send_blocks(o_part, lse_part, world)
    row0, n = shard_range(B * Nq, rank, world)
    o_recv = torch.empty((world * n, Hq * d), dtype=o_part.dtype, device=o_part.device)
    l_recv = torch.empty((world * n, Hq), dtype=lse_part.dtype, device=lse_part.device)
    dist.all_to_all_single(o_recv, o_send, output_split_sizes=[n] * world, input_split_sizes=sizes, group=group)
    dist.all_to_all_single(l_recv, l_send, output_split_sizes=[n] * world, input_split_sizes=sizes, group=group)
    o_parts, lse_parts = received_layout(o_recv, l_recv, world, n, Hq, d)
    return o_parts, lse_parts, (row0, n)


def gather_rows(out_rows, lse_rows, B: int, Nq: int, group=None):
    """All-gather of every rank's merged rows (out_rows [1, n, Hq, d] bf16, lse_rows [1, Hq, n]
    fp32, blocks in rank order) into out [B, Nq, Hq, d] and lse [B, Hq, Nq] on every rank.
    Blocks differ by at most one row; each is padded to the largest for the collective."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rows = B * Nq
    Hq, d = out_rows.shape[2], out_rows.shape[3]
    sizes = [shard_range(rows, r, world)[1] for r in range(world)]
    m = max(sizes) if sizes else 0
    n = out_rows.shape[1]
    o_pad = torch.zeros((m, Hq * d), dtype=out_rows.dtype, device=out_rows.device)
    o_pad[:n] = out_rows.reshape(n, Hq * d)
    l_pad = torch.zeros((m, Hq), dtype=lse_rows.dtype, device=lse_rows.device)
    l_pad[:n] = lse_rows.reshape(Hq, n).t()
    o_all = torch.empty((world * m, Hq * d), dtype=out_rows.dtype, device=out_rows.device)
    l_all = torch.empty((world * m, Hq), dtype=lse_rows.dtype, device=lse_rows.device)
    dist.all_gather_into_tensor(o_all, o_pad, group=group)
    dist.all_gather_into_tensor(l_all, l_pad, group=group)
    keep = torch.cat([torch.arange(r * m, r * m + sizes[r], device=out_rows.device) for r in range(world)])
    out = o_all.index_select(0, keep).view(B, Nq, Hq, d)
    lse = l_all.index_select(0, keep).view(B, Nq, Hq).permute(0, 2, 1).contiguous()
    return out, lse


def kshard_attention(q, k_shard, v_shard, *, key_offset: int, nk_total: int, causal: bool = False,
                     scale: float | None = None, group=None, gather_output: bool = True):
    """Exact attention of q over the union of every rank's key shard.

    gather_output=True: returns (out bf16 [B, Nq, Hq, d], lse fp32 [B, Hq, Nq]), the same on
    every rank.  False: returns (out_rows [1, n, Hq, d], lse_rows [1, Hq, n], (row0, n)), this
    rank's block of the flattened (b, i) query rows, with no second collective."""
    B, Nq = q.shape[0], q.shape[1]
    o_part, lse_part = fa_fwd_partial(q, k_shard, v_shard, key_offset=key_offset, nk_total=nk_total,
                                      causal=causal, scale=scale)
    o_parts, lse_parts, span = exchange_partials(o_part, lse_part, group)
    out_rows, lse_rows = fa_merge_partials(o_parts, lse_parts)
    if not gather_output:
        return out_rows, lse_rows, span
    return gather_rows(out_rows, lse_rows, B, Nq, group)

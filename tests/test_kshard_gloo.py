"""Key-sharded attention, host side, on CPU with gloo ranks: the shard partition, and the
exchange steps of exact_attention_146_b200.kshard (exchange_partials: an all-to-all that
carries to each rank every rank's partial for that rank's block of query rows; gather_rows:
the merged rows back to every rank).  Each rank's partial here comes from the
oracle on its own key shard (no GPU); merged with the log-sum-exp identity, the gathered
partials must equal the oracle's forward over all keys."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth
from exact_attention_146_b200 import kshard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_range_partitions_the_keys():
    for nk, world in [(0, 3), (1, 2), (10, 3), (4096, 8), (4097, 8), (5, 8)]:
        spans = [kshard.shard_range(nk, r, world) for r in range(world)]
        assert spans[0][0] == 0
        for (o0, n0), (o1, _) in zip(spans, spans[1:]):
            assert o1 == o0 + n0                          # contiguous, in rank order
        assert sum(n for _, n in spans) == nk
        assert max(n for _, n in spans) - min(n for _, n in spans) <= 1
    with pytest.raises(ValueError):
        kshard.shard_range(10, 3, 3)


def _lse_merge(o_parts, l_parts):
    """The log-sum-exp identity the merge kernel applies, in numpy: o_parts [R, B, n, Hq, d],
    l_parts [R, B, Hq, n] -> (O [B, n, Hq, d], LSE [B, Hq, n])."""
    m = l_parts.max(axis=0)
    wts = np.exp(l_parts - m)
    lse = m + np.log(wts.sum(axis=0))
    o = np.einsum("rbhi,rbihd->bihd", wts, o_parts) / wts.sum(axis=0).transpose(0, 2, 1)[..., None]
    return o, lse


SHAPE = dict(B=2, Hq=4, Hkv=2, Nq=9, Nk=23, d=32)


def _worker(rank, world, port, out, shape=None):
    import torch
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sh = shape or SHAPE
        w = synth.Workload("kshard", 77, sh["B"], sh["Hq"], sh["Hkv"], sh["Nq"], sh["Nk"], sh["d"], False, seed=5)
        x = synth.make_inputs(w)
        off, n = kshard.shard_range(w.Nk, rank, world)
        O, L = oracle.default().forward(x["q"], x["k"][:, off:off + n], x["v"][:, off:off + n], w.scale, False)
        o_parts, l_parts, (row0, nrows) = kshard.exchange_partials(torch.from_numpy(O), torch.from_numpy(L))
        assert tuple(o_parts.shape) == (world, 1, nrows, w.Hq, w.d) and tuple(l_parts.shape) == (world, 1, w.Hq, nrows)
        o_rows, l_rows = _lse_merge(o_parts.numpy(), l_parts.numpy())
        o_all, l_all = kshard.gather_rows(torch.from_numpy(o_rows), torch.from_numpy(l_rows), w.B, w.Nq)
        out[rank] = (o_all.numpy(), l_all.numpy(), row0, nrows, int(o_parts.numel()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_by_rows_reproduces_full_attention(world):
    """Each rank receives only its block of query rows from every rank (R x its rows, not R x
    all rows), merges it, and the gathered rows equal the oracle's forward over all keys."""
    import oracle
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    w = synth.Workload("kshard", 77, SHAPE["B"], SHAPE["Hq"], SHAPE["Hkv"], SHAPE["Nq"], SHAPE["Nk"], SHAPE["d"],
                       False, seed=5)
    x = synth.make_inputs(w)
    Oref, Lref = oracle.default().forward(x["q"], x["k"], x["v"], w.scale, False)
    rows = w.B * w.Nq
    assert [out[r][2] for r in range(world)] == [kshard.shard_range(rows, r, world)[0] for r in range(world)]
    for r in range(world):
        o, lse, row0, n, received = out[r]
        assert np.abs(o - Oref).max() < 1e-12 and np.abs(lse - Lref).max() < 1e-12
        assert received == world * n * w.Hq * w.d           # partial values this rank received
    assert sum(out[r][3] for r in range(world)) == rows


def test_exchange_with_fewer_rows_than_ranks():
    """Two query rows over three ranks: one rank owns no row; the exchange and the gather
    still deliver every row, equal to the oracle over all keys."""
    import oracle
    shape = dict(B=1, Hq=2, Hkv=1, Nq=2, Nk=11, d=32)
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 3, port, out, shape)) for r in range(3)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    w = synth.Workload("kshard", 77, 1, 2, 1, 2, 11, 32, False, seed=5)
    x = synth.make_inputs(w)
    Oref, Lref = oracle.default().forward(x["q"], x["k"], x["v"], w.scale, False)
    assert sorted(out[r][3] for r in range(3)) == [0, 1, 1]
    for r in range(3):
        assert np.abs(out[r][0] - Oref).max() < 1e-12 and np.abs(out[r][1] - Lref).max() < 1e-12

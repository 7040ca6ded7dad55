"""Key-sharded attention, host side, on CPU with two gloo ranks: the shard partition, and
the exchange step of exact_attention_146_b200.kshard (gather_partials) carrying every
rank's partial to every rank in rank order.  Each rank's partial here comes from the
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


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.Workload("kshard", 77, 1, 4, 2, 9, 23, 32, False, seed=5)
        x = synth.make_inputs(w)
        off, n = kshard.shard_range(w.Nk, rank, world)
        O, L = oracle.default().forward(x["q"], x["k"][:, off:off + n], x["v"][:, off:off + n], w.scale, False)
        o_all, l_all = kshard.gather_partials(torch.from_numpy(O), torch.from_numpy(L))
        out[rank] = (o_all.numpy(), l_all.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_reproduces_full_attention():
    import oracle
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    (o0, l0), (o1, l1) = out[0], out[1]
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)      # every rank holds every partial
    # log-sum-exp merge of the stacked partials (the identity the merge kernel applies)
    m = l0.max(axis=0)
    wts = np.exp(l0 - m)                                           # [R, B, Hq, Nq]
    lse = m + np.log(wts.sum(axis=0))
    o = np.einsum("rbhi,rbihd->bihd", wts, o0) / wts.sum(axis=0).transpose(0, 2, 1)[..., None]
    w = synth.Workload("kshard", 77, 1, 4, 2, 9, 23, 32, False, seed=5)
    x = synth.make_inputs(w)
    Oref, Lref = oracle.default().forward(x["q"], x["k"], x["v"], w.scale, False)
    assert np.abs(o - Oref).max() < 1e-12 and np.abs(lse - Lref).max() < 1e-12

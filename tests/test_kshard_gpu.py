"""Key-sharded attention kernels on one GPU: the R shards a multi-GPU run would spread over
R GPUs are computed one after another here (fa_fwd_partial with each shard's offset),
stacked as the all-gather would stack them, and merged (fa_merge_partials); the result must
equal the oracle's forward over all keys, causal included (the mask is taken against the
global key index)."""
import math

import numpy as np
import pytest

import oracle
import synth
from exact_attention_146_b200 import kshard
from tests import _parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_attention_146_b200 import build
    build.build()
    yield


@pytest.mark.parametrize("R", [1, 2, 3, 5])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 4, 2, 300, 1000, 128), (2, 2, 2, 129, 129, 64), (1, 8, 8, 700, 450, 128),
                                   (1, 4, 4, 333, 700, 96)])
def test_sharded_equals_full(orc, R, causal, shape):
    import torch
    import exact_attention_146_b200 as fa
    B, Hq, Hkv, Nq, Nk, d = shape
    w = synth.Workload("ks", 5000 + R + Nk, B, Hq, Hkv, Nq, Nk, d, False, seed=R)
    x = synth.make_inputs(w)
    q, k, v = (_parity.to_device(x[n], torch) for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    o_all = torch.empty((R, B, Nq, Hq, d), dtype=torch.float32, device="cuda")
    l_all = torch.empty((R, B, Hq, Nq), dtype=torch.float32, device="cuda")
    for r in range(R):
        off, n = kshard.shard_range(Nk, r, R)
        fa.fa_fwd_partial(q, k[:, off:off + n].contiguous(), v[:, off:off + n].contiguous(), key_offset=off,
                          nk_total=Nk, causal=causal, scale=scale, o_part=o_all[r], lse_part=l_all[r])
    out, lse = fa.fa_merge_partials(o_all, l_all)
    st, word = fa.device_status()
    assert st == fa.FA_OK, f"device status {st} ({word:#x})"
    torch.cuda.synchronize()
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], scale, causal)
    _parity.compare(_parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), Oref, Lref,
                    f"R={R} causal={causal} {shape}")


def test_empty_shard_is_neutral(orc):
    """A shard with no keys contributes O = 0, LSE = -inf (weight 0)."""
    import torch
    import exact_attention_146_b200 as fa
    w = synth.Workload("ks0", 5900, 1, 2, 1, 50, 80, 64, False, seed=9)
    x = synth.make_inputs(w)
    q, k, v = (_parity.to_device(x[n], torch) for n in ("q", "k", "v"))
    o_all = torch.empty((2, 1, 50, 2, 64), dtype=torch.float32, device="cuda")
    l_all = torch.empty((2, 1, 2, 50), dtype=torch.float32, device="cuda")
    fa.fa_fwd_partial(q, k, v, key_offset=0, nk_total=80, scale=0.125, o_part=o_all[0], lse_part=l_all[0])
    fa.fa_fwd_partial(q, k[:, :0].contiguous(), v[:, :0].contiguous(), key_offset=80, nk_total=80, scale=0.125,
                      o_part=o_all[1], lse_part=l_all[1])
    out, lse = fa.fa_merge_partials(o_all, l_all)
    torch.cuda.synchronize()
    assert torch.isneginf(l_all[1]).all() and (o_all[1] == 0).all()
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 0.125, False)
    _parity.compare(_parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), Oref, Lref, "empty shard")


@pytest.mark.parametrize("R", [2, 3])
def test_row_block_exchange_layout(orc, R):
    """The all-to-all by query rows, emulated on one GPU: each of R shards' partials is cut
    by destination (kshard.send_blocks), every destination stacks what it would receive
    (kshard.received_layout) and merges only its rows; the rows, put back in order, equal
    the oracle's forward over all keys."""
    import torch
    import exact_attention_146_b200 as fa
    B, Hq, Hkv, Nq, Nk, d = 2, 4, 2, 301, 900, 128
    w = synth.Workload("ksrows", 5950 + R, B, Hq, Hkv, Nq, Nk, d, False, seed=R)
    x = synth.make_inputs(w)
    q, k, v = (_parity.to_device(x[n], torch) for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(d)
    sends = []
    for r in range(R):
        off, n = kshard.shard_range(Nk, r, R)
        o_p, l_p = fa.fa_fwd_partial(q, k[:, off:off + n].contiguous(), v[:, off:off + n].contiguous(),
                                     key_offset=off, nk_total=Nk, causal=True, scale=scale)
        sends.append(kshard.send_blocks(o_p, l_p, R))
    outs, lses = [], []
    for s in range(R):
        row0, n = kshard.shard_range(B * Nq, s, R)
        o_recv = torch.cat([o_send[row0:row0 + n] for o_send, _, _ in sends])
        l_recv = torch.cat([l_send[row0:row0 + n] for _, l_send, _ in sends])
        o_parts, l_parts = kshard.received_layout(o_recv, l_recv, R, n, Hq, d)
        o_rows, l_rows = fa.fa_merge_partials(o_parts, l_parts)
        outs.append(o_rows.reshape(n, Hq, d))
        lses.append(l_rows.reshape(Hq, n).t())
    out = torch.cat(outs).view(B, Nq, Hq, d)
    lse = torch.cat(lses).view(B, Nq, Hq).permute(0, 2, 1).contiguous()
    assert fa.device_status()[0] == fa.FA_OK
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], scale, True)
    _parity.compare(_parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), Oref, Lref, f"rows R={R}")

"""Parity of the CUDA path (through the C ABI) with the CPU fp64 oracle, element by
element, on seeded inputs: small shapes that span several tiles with ragged tails for
every head dim, GQA ratios, Nq != Nk, empty rows, the degenerate sizes, and every
workload of the table at its full size (rows sampled from the very launch the benchmark
times, checked one by one against the oracle)."""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import _parity

pytestmark = pytest.mark.gpu

HEAD_DIMS = (32, 64, 80, 96, 128, 192, 256)


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


def tiny(B, Hq, Hkv, Nq, Nk, d, seed, **kw):
    w = synth.Workload("t", 500 + seed, B, Hq, Hkv, Nq, Nk, d, False, seed=seed, **kw)
    return synth.make_inputs(w)


def check_full(orc, x, scale, causal, what, dtype="bf16"):
    O, L = _parity.run_cuda(x, scale, causal, dtype=dtype)
    if dtype == "e4m3":
        return _parity.compare_fp8(orc, x, O, L, scale, causal, what=what)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], scale, causal, dtype=dtype)
    return _parity.compare(O, L, Oref, Lref, what)


@pytest.mark.parametrize("d", HEAD_DIMS)
@pytest.mark.parametrize("N", [1, 17, 128, 129, 300, 600])
@pytest.mark.parametrize("causal", [False, True])
def test_small_shapes(orc, d, N, causal):
    x = tiny(1, 2, 1, N, N, d, seed=N + d)
    check_full(orc, x, 1.0 / math.sqrt(d), causal, f"d={d} N={N} causal={causal}")


@pytest.mark.parametrize("Hkv", [1, 2, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_ratios(orc, Hkv, causal):
    x = tiny(2, 8, Hkv, 200, 200, 128, seed=40 + Hkv)
    check_full(orc, x, 1.0 / math.sqrt(128), causal, f"GQA 8/{Hkv}")


def test_gqa_32_query_heads_per_kv_head(orc):
    x = tiny(1, 32, 1, 130, 130, 64, seed=49)
    check_full(orc, x, 0.125, True, "GQA 32/1")


@pytest.mark.parametrize("Nq,Nk", [(100, 300), (300, 100), (1, 700), (257, 256), (600, 5)])
@pytest.mark.parametrize("causal", [False, True])
def test_unequal_lengths(orc, Nq, Nk, causal):
    """Bottom-right aligned causal mask; Nq > Nk leaves the first rows without a key."""
    x = tiny(1, 4, 2, Nq, Nk, 64, seed=Nq * 7 + Nk)
    check_full(orc, x, 0.125, causal, f"Nq={Nq} Nk={Nk}")


@pytest.mark.parametrize("d", [64, 128])
def test_large_logits_rescale_path(orc, d):
    """Q x 8 (exact in bf16): logits of tens, row maxima keep growing along the row."""
    x = tiny(2, 4, 4, 700, 700, d, seed=60 + d, q_mult=8.0)
    check_full(orc, x, 1.0 / math.sqrt(d), False, "qx8")
    check_full(orc, x, 1.0 / math.sqrt(d), True, "qx8 causal")


def test_increasing_logits_force_rescales(orc):
    """Keys whose logits grow tile after tile, so the running max rises past the lazy
    rescale threshold many times."""
    x = tiny(1, 2, 2, 256, 1024, 128, seed=70)
    q = synth.bf16_bits_to_f32(x["q"]).copy()
    k = synth.bf16_bits_to_f32(x["k"]).copy()
    q[..., :] = np.abs(q)
    ramp = np.linspace(0.0, 6.0, 1024, dtype=np.float32)[None, :, None, None]
    k = np.abs(k) * ramp
    x = {"q": synth.f32_to_bf16_bits(q), "k": synth.f32_to_bf16_bits(k), "v": x["v"]}
    check_full(orc, x, 1.0 / math.sqrt(128), False, "ramp")
    check_full(orc, x, 1.0 / math.sqrt(128), True, "ramp causal")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [129, 300, 700])
@pytest.mark.parametrize("W", [1, 17, 128, 129, 250, 1000])
def test_sliding_window(orc, d, N, W):
    x = tiny(1, 2, 1, N, N, d, seed=N + W + d)
    O, L = _parity.run_cuda(x, 1.0 / math.sqrt(d), True, window=W)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 1.0 / math.sqrt(d), True, window=W)
    _parity.compare(O, L, Oref, Lref, f"window d={d} N={N} W={W}")


@pytest.mark.parametrize("Nq,Nk,W", [(100, 300, 64), (300, 100, 40), (257, 700, 300), (1, 500, 130)])
def test_sliding_window_unequal_lengths(orc, Nq, Nk, W):
    x = tiny(2, 4, 2, Nq, Nk, 64, seed=Nq + Nk + W)
    O, L = _parity.run_cuda(x, 0.125, True, window=W)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 0.125, True, window=W)
    _parity.compare(O, L, Oref, Lref, f"window Nq={Nq} Nk={Nk} W={W}")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("Nq,Nk", [(1, 1000), (16, 2049), (130, 700)])
@pytest.mark.parametrize("splits", [2, 3, 7, 40])
@pytest.mark.parametrize("causal", [False, True])
def test_splitkv(orc, d, Nq, Nk, splits, causal):
    """Split-KV (40 splits leaves some slices without a key tile) equals the oracle."""
    x = tiny(1, 4, 2, Nq, Nk, d, seed=Nq + Nk + splits + d)
    O, L = _parity.run_cuda(x, 1.0 / math.sqrt(d), causal, num_splits=splits)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 1.0 / math.sqrt(d), causal)
    _parity.compare(O, L, Oref, Lref, f"splitkv d={d} Nq={Nq} Nk={Nk} S={splits} causal={causal}")


# The head dims whose two query tiles take turns in one TMEM S buffer (P in columns of its
# own); d = 128 is covered by the tests above and the full-size workloads.
SHARED_S_DIMS = (80, 96, 192)


@pytest.mark.parametrize("d", SHARED_S_DIMS)
@pytest.mark.parametrize("N,W", [(300, 1), (300, 129), (700, 250), (700, 1000)])
def test_shared_s_sliding_window(orc, d, N, W):
    x = tiny(1, 2, 1, N, N, d, seed=N + W + d + 1)
    O, L = _parity.run_cuda(x, 1.0 / math.sqrt(d), True, window=W)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 1.0 / math.sqrt(d), True, window=W)
    _parity.compare(O, L, Oref, Lref, f"window d={d} N={N} W={W}")


@pytest.mark.parametrize("d", SHARED_S_DIMS)
@pytest.mark.parametrize("Nq,Nk,splits,causal", [(1, 1000, 3, False), (16, 2049, 7, True), (130, 700, 2, True),
                                                 (130, 700, 40, False)])
def test_shared_s_splitkv(orc, d, Nq, Nk, splits, causal):
    x = tiny(1, 4, 2, Nq, Nk, d, seed=Nq + Nk + splits + d + 1)
    O, L = _parity.run_cuda(x, 1.0 / math.sqrt(d), causal, num_splits=splits)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 1.0 / math.sqrt(d), causal)
    _parity.compare(O, L, Oref, Lref, f"splitkv d={d} Nq={Nq} Nk={Nk} S={splits} causal={causal}")


@pytest.mark.parametrize("d", SHARED_S_DIMS)
def test_shared_s_rescale_path(orc, d):
    """Q x 8: the row maxima keep growing, so O is rescaled between P V products."""
    x = tiny(2, 4, 4, 700, 700, d, seed=61 + d, q_mult=8.0)
    check_full(orc, x, 1.0 / math.sqrt(d), False, f"qx8 d={d}")
    check_full(orc, x, 1.0 / math.sqrt(d), True, f"qx8 causal d={d}")


@pytest.mark.parametrize("d", SHARED_S_DIMS)
@pytest.mark.parametrize("Hkv", [1, 4])
def test_shared_s_causal_tile_ranges(orc, d, Hkv):
    """Causal with Hq == Hkv: the unit's two query tiles see different numbers of key tiles
    (the second one more), so the shared buffer's turns are uneven; Hkv = 1: the causal GQA
    units pair two query heads over the same rows."""
    x = tiny(1, 4, Hkv, 600, 600, d, seed=80 + d + Hkv)
    check_full(orc, x, 1.0 / math.sqrt(d), True, f"causal d={d} Hkv={Hkv}")


@pytest.mark.parametrize("n_rep", [2, 4, 8, 16, 32])
@pytest.mark.parametrize("Nq", [1, 5, 16, 33, 127])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_packed_rows(orc, n_rep, Nq, causal):
    """Nq < 128 with n_rep | 128: the n_rep heads of a KV head share a tile (flat rows
    i * n_rep + r); two batches and two KV heads exercise the group indexing."""
    Hkv = 2
    d = 64 if n_rep >= 16 else 128
    x = tiny(2, Hkv * n_rep, Hkv, Nq, 700, d, seed=n_rep * 100 + Nq)
    check_full(orc, x, 1.0 / math.sqrt(d), causal, f"packed n_rep={n_rep} Nq={Nq} causal={causal}")


@pytest.mark.parametrize("n_rep,Nq", [(3, 16), (4, 128), (64, 2)])
def test_gqa_unpacked_and_edge(orc, n_rep, Nq):
    """n_rep = 3 (does not divide 128) and Nq = 128 run unpacked; n_rep = 64 packs 2 rows per head."""
    x = tiny(1, n_rep * 2, 2, Nq, 900, 64, seed=n_rep + Nq)
    check_full(orc, x, 0.125, True, f"n_rep={n_rep} Nq={Nq}")


@pytest.mark.parametrize("splits", [3, 9])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_packed_splitkv(orc, splits, causal):
    x = tiny(2, 32, 8, 16, 5000, 128, seed=splits + 40)
    O, L = _parity.run_cuda(x, 0.088, causal, num_splits=splits)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 0.088, causal)
    _parity.compare(O, L, Oref, Lref, f"packed split-KV S={splits} causal={causal}")


@pytest.mark.parametrize("W", [1, 100, 1000])
def test_gqa_packed_window(orc, W):
    x = tiny(1, 16, 2, 40, 1200, 128, seed=W)
    O, L = _parity.run_cuda(x, 0.088, True, window=W)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 0.088, True, window=W)
    _parity.compare(O, L, Oref, Lref, f"packed window W={W}")


@pytest.mark.parametrize("d", HEAD_DIMS)
@pytest.mark.parametrize("N", [17, 300])
@pytest.mark.parametrize("causal", [False, True])
def test_f16_small_shapes(orc, d, N, causal):
    """fp16 inputs (fa_fwd_f16) against the oracle reading the same half bit patterns."""
    x = tiny(1, 2, 1, N, N, d, seed=N + d + 7, dtype="f16")
    check_full(orc, x, 1.0 / math.sqrt(d), causal, f"f16 d={d} N={N} causal={causal}", dtype="f16")


@pytest.mark.parametrize("case", [(2, 8, 2, 200, 700, 128, True), (1, 32, 8, 16, 3000, 128, False),
                                  (1, 4, 4, 1, 1, 64, False), (2, 6, 3, 130, 129, 96, True)])
def test_f16_gqa_ragged(orc, case):
    B, Hq, Hkv, Nq, Nk, d, causal = case
    x = tiny(B, Hq, Hkv, Nq, Nk, d, seed=Nq + Nk, q_mult=8.0, dtype="f16")
    check_full(orc, x, 1.0 / math.sqrt(d), causal, f"f16 {case}", dtype="f16")


def test_f16_is_not_read_as_bf16(orc):
    """The same bits read as bf16 give a different answer: fa_fwd_f16 must match the fp16
    reading, not the bf16 one."""
    x = tiny(1, 2, 1, 64, 64, 64, seed=3, dtype="f16")
    O, L = _parity.run_cuda(x, 0.125, False, dtype="f16")
    Of, _ = orc.forward(x["q"], x["k"], x["v"], 0.125, False, dtype="f16")
    Ob, _ = orc.forward(x["q"], x["k"], x["v"], 0.125, False, dtype="bf16")
    assert np.abs(O - Of).max() <= _parity.TOL_O_MAX < np.abs(O - Ob).max()


@pytest.mark.parametrize("N", [1, 17, 128, 129, 300, 600])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_small_shapes(orc, N, causal):
    """E4M3 inputs (fa_fwd_fp8, d = 128) against the oracle reading the same bytes."""
    x = tiny(1, 2, 1, N, N, 128, seed=N + 11, dtype="e4m3")
    check_full(orc, x, 1.0 / math.sqrt(128), causal, f"fp8 N={N} causal={causal}", dtype="e4m3")


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("N", [1, 17, 129, 300, 600])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_head_dims(orc, d, N, causal):
    """fa_fwd_fp8 at the other FP8 head dims (64-byte rows at d = 64; one query tile and two
    S buffers at d = 256), several key tiles and a ragged tail, against the oracle."""
    x = tiny(1, 2, 1, N, N, d, seed=N + d, dtype="e4m3")
    check_full(orc, x, 1.0 / math.sqrt(d), causal, f"fp8 d={d} N={N} causal={causal}", dtype="e4m3")


@pytest.mark.parametrize("d", [64, 256])
def test_fp8_head_dims_gqa_descales(orc, d):
    B, Hq, Hkv, Nq, Nk, causal, ds = 2, 8, 2, 200, 700, True, (0.5, 2.0, 0.25)
    x = tiny(B, Hq, Hkv, Nq, Nk, d, seed=Nq + d, q_mult=4.0, dtype="e4m3")
    scale = 1.0 / math.sqrt(d)
    O, L = _parity.run_cuda_fp8(x, scale, causal, descale=ds)
    _parity.compare_fp8(orc, x, O, L, scale, causal, descale=ds, what=f"fp8 d={d} gqa descales")


@pytest.mark.parametrize("case", [(2, 8, 2, 200, 700, True, (0.5, 2.0, 0.25)), (1, 32, 8, 16, 3000, False, (1.0, 1.0, 4.0)),
                                  (2, 6, 3, 130, 129, True, (0.125, 0.75, 1.5)), (1, 4, 4, 1000, 1000, False, (2.0, 2.0, 0.5))])
def test_fp8_gqa_descales(orc, case):
    """GQA, ragged lengths, GQA-packed decode rows and non-unit dequantisation factors."""
    B, Hq, Hkv, Nq, Nk, causal, ds = case
    x = tiny(B, Hq, Hkv, Nq, Nk, 128, seed=Nq + Nk, q_mult=4.0, dtype="e4m3")
    scale = 1.0 / math.sqrt(128)
    O, L = _parity.run_cuda_fp8(x, scale, causal, descale=ds)
    _parity.compare_fp8(orc, x, O, L, scale, causal, descale=ds, what=f"fp8 {case}")


def test_splitkv_matches_plain_forward():
    x = tiny(2, 8, 2, 64, 4096, 128, seed=99)
    O1, L1 = _parity.run_cuda(x, 0.08, False)
    O2, L2 = _parity.run_cuda(x, 0.08, False, num_splits=5)
    assert np.abs(O1 - O2).max() < 1e-2 and np.abs(L1 - L2).max() < 1e-4


def test_lse_optional(orc):
    x = tiny(1, 2, 1, 200, 200, 64, seed=80)
    O, L = _parity.run_cuda(x, 0.125, True, with_lse=False)
    Oref, _ = orc.forward(x["q"], x["k"], x["v"], 0.125, True)
    _parity.compare(O, None, Oref, None, "no lse")


def test_no_keys():
    """Nk = 0: O = 0, LSE = -inf."""
    x = tiny(2, 2, 1, 50, 0, 64, seed=81)
    O, L = _parity.run_cuda(x, 0.125, False)
    assert (O == 0).all() and np.isneginf(L).all()


def test_empty_problems():
    """B = 0 or Nq = 0: nothing to compute, FA_OK, nothing launched."""
    import torch
    import exact_attention_146_b200 as fa
    kv = torch.zeros((1, 16, 2, 64), dtype=torch.bfloat16, device="cuda")
    q0 = torch.zeros((0, 16, 2, 64), dtype=torch.bfloat16, device="cuda")
    out, lse = fa.fa_fwd(q0, kv[:0], kv[:0])
    assert out.shape == q0.shape and lse.shape == (0, 2, 16)
    q1 = torch.zeros((1, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    out, lse = fa.fa_fwd(q1, kv, kv)
    assert out.numel() == 0 and lse.numel() == 0
    assert fa.device_status()[0] == fa.FA_OK


def test_rejects_host_memory():
    import torch
    import exact_attention_146_b200 as fa
    qh = torch.zeros((1, 64, 2, 64), dtype=torch.int16).view(torch.bfloat16)
    qd = torch.zeros((1, 64, 2, 64), dtype=torch.bfloat16, device="cuda")
    od = torch.empty_like(qd)
    rc = fa.fa_fwd_raw(qh.data_ptr(), qd.data_ptr(), qd.data_ptr(), od.data_ptr(), None,
                       1, 2, 2, 64, 64, 64, 0.125, 0, 0)
    assert rc == fa.FA_ERR_NOT_DEVICE_MEMORY
    assert fa.device_status()[0] == fa.FA_OK


def _cudart():
    try:
        from cuda.bindings import runtime as rt
    except ImportError:
        try:
            from cuda import cudart as rt
        except ImportError:
            pytest.skip("cuda-python not available")
    return rt


def test_rejects_buffer_shorter_than_sizes():
    """A K/V buffer shorter than B*Nk*Hkv*d elements is refused before any launch."""
    import torch
    import exact_attention_146_b200 as fa
    rt = _cudart()
    err, kbuf = rt.cudaMalloc(1 << 20)
    assert int(err) == 0
    try:
        q = torch.zeros((1, 64, 2, 64), dtype=torch.bfloat16, device="cuda")
        out = torch.empty_like(q)
        Nk = 1 << 16                          # claims 16 MiB of K and of V
        lo, hi = int(kbuf), int(kbuf) + Nk * 2 * 64 * 2
        for t in (q, out):
            if lo < t.data_ptr() + t.numel() * 2 and t.data_ptr() < hi:
                pytest.skip("allocator placed the tensors inside the claimed range")
        rc = fa.fa_fwd_raw(q.data_ptr(), int(kbuf), int(kbuf), out.data_ptr(), None,
                           1, 2, 2, 64, Nk, 64, 0.125, 0, 0)
        assert rc == fa.FA_ERR_NOT_DEVICE_MEMORY
    finally:
        rt.cudaFree(kbuf)
    assert fa.device_status()[0] == fa.FA_OK


def test_deterministic(orc):
    x = tiny(2, 4, 2, 333, 333, 128, seed=90)
    O1, L1 = _parity.run_cuda(x, 0.1, True)
    O2, L2 = _parity.run_cuda(x, 0.1, True)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


# ------------------------------------------------------------------ workload table

SMALL_FULL = ["yolo20x20_b1_h4_d64", "yolo20x20_b1_h4_d64_qx8", "yolo20x20_b32_h16_d64"]
LARGE_SAMPLED = [n for n in synth.WORKLOADS if n not in SMALL_FULL]


@pytest.mark.parametrize("name", SMALL_FULL)
def test_workload_full(orc, name):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    res = check_full(orc, x, w.scale, w.causal, name, dtype=w.dtype)
    print(name, res)


@pytest.mark.parametrize("name", LARGE_SAMPLED)
def test_workload_sampled_rows(orc, name):
    """Full-size launch (the one the benchmark times); sampled rows checked against the
    oracle one by one, and every output row checked to be written and finite."""
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    if w.dtype == "e4m3":
        O, L = _parity.run_cuda_fp8(x, w.scale, w.causal)
        assert np.isfinite(O).all() and np.isfinite(L).all()
        _parity.compare_fp8(orc, x, O, L, w.scale, w.causal, what=name, rows=_parity.sample_rows(w, 64))
        return
    O, L = _parity.run_cuda(x, w.scale, w.causal, window=w.window or None, num_splits=_parity.workload_splits(w),
                            dtype=w.dtype)
    assert np.isfinite(O).all() and np.isfinite(L).all()
    rows = _parity.sample_rows(w, 192, seed=w.wid)
    Oref, Lref = orc.rows(x["q"], x["k"], x["v"], rows, w.scale, w.causal, window=w.window, dtype=w.dtype)
    Os = O[rows[:, 0], rows[:, 2], rows[:, 1], :]
    Ls = L[rows[:, 0], rows[:, 1], rows[:, 2]]
    res = _parity.compare(Os, Ls, Oref, Lref, name)
    print(name, len(rows), res)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("window", [1, 77, 300])
def test_f16_sliding_window(orc, d, window):
    """fp16 inputs with the sliding-window mask (fa_fwd_window_f16), Nq != Nk, GQA."""
    x = tiny(2, 4, 2, 333, 517, d, seed=window + d, dtype="f16")
    O, L = _parity.run_cuda(x, 1.0 / math.sqrt(d), True, window=window, dtype="f16")
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 1.0 / math.sqrt(d), True, window=window, dtype="f16")
    _parity.compare(O, L, Oref, Lref, f"f16 window={window} d={d}")


@pytest.mark.parametrize("splits", [2, 7])
@pytest.mark.parametrize("causal", [False, True])
def test_f16_splitkv(orc, splits, causal):
    """fp16 inputs through split-KV (fa_fwd_splitkv_f16): decode-shaped GQA rows, fp16 merge."""
    x = tiny(2, 8, 2, 16, 2500, 128, seed=splits + 40, dtype="f16")
    O, L = _parity.run_cuda(x, 0.09, causal, num_splits=splits, dtype="f16")
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 0.09, causal, dtype="f16")
    _parity.compare(O, L, Oref, Lref, f"f16 splitkv S={splits} causal={causal}")

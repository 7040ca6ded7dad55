"""Host-only checks of the C ABI (no GPU needed): the library builds and loads, exports
every symbol include/fa.h declares, reports the tiling per head dim, and rejects bad
arguments synchronously, before touching any device (fake pointers are never
dereferenced: validation runs first)."""
import ctypes
import json
import re
from pathlib import Path

import pytest

import exact_attention_146_b200 as fa
from exact_attention_146_b200 import build as fa_build

ROOT = Path(__file__).resolve().parent.parent
GOLDEN = json.loads((ROOT / "tests" / "golden" / "pages_facts.json").read_text())


@pytest.fixture(scope="module")
def L():
    fa_build.build()
    return fa.lib()


def header_functions():
    text = (ROOT / "include" / "fa.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_header_symbols_exported(L):
    names = header_functions()
    assert set(names) == set(fa.EXPORTED)
    for n in names:
        assert hasattr(L, n), n


def test_version(L):
    assert L.fa_version() == 100


def test_head_dims_from_pages(L):
    supported = GOLDEN["head_dims_listed"]["value"] + GOLDEN["head_dims_added"]["value"]
    assert sorted(supported) == sorted(fa.SUPPORTED_HEAD_DIMS)
    for d in supported:
        cfg = fa.tile_config(d)
        assert cfg["block_q"] == 128 and cfg["block_k"] in (64, 128)
        assert cfg["q_tiles_per_unit"] in (1, 2) and cfg["kv_slots"] >= 2
    for d in GOLDEN["head_dims_rejected_examples"]["value"]:
        assert L.fa_tile_config(d, None, None, None, None) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM
    msg = fa.status_string(fa.FA_ERR_UNSUPPORTED_HEAD_DIM)
    for d in supported:
        assert str(d) in msg


FAKE = 1 << 40  # never dereferenced: every case below fails validation first


def call(L, q=FAKE, k=FAKE + (1 << 30), v=FAKE + (2 << 30), out=FAKE + (3 << 30), lse=FAKE + (4 << 30),
         B=1, Hq=2, Hkv=1, Nq=16, Nk=16, d=64, scale=0.125, causal=0):
    return L.fa_fwd(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), fa.FA_ERR_INVALID_ARG),
    (dict(Hq=0), fa.FA_ERR_INVALID_ARG),
    (dict(Hkv=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=-3), fa.FA_ERR_INVALID_ARG),
    (dict(Nk=-1), fa.FA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), fa.FA_ERR_INVALID_ARG),
    (dict(causal=2), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=-0.5), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(d=48), fa.FA_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(d=512), fa.FA_ERR_UNSUPPORTED_HEAD_DIM),
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(out=None), fa.FA_ERR_INVALID_ARG),
    (dict(k=None), fa.FA_ERR_INVALID_ARG),
    (dict(v=None), fa.FA_ERR_INVALID_ARG),
    (dict(q=FAKE + 8), fa.FA_ERR_MISALIGNED),
    (dict(out=FAKE + (3 << 30) + 2), fa.FA_ERR_MISALIGNED),
    (dict(lse=FAKE + (4 << 30) + 2), fa.FA_ERR_MISALIGNED),
    (dict(out=FAKE + 64), fa.FA_ERR_OVERLAP),                 # out inside q
    (dict(lse=FAKE + (3 << 30) + 128), fa.FA_ERR_OVERLAP),    # lse inside out
    (dict(lse=FAKE + (1 << 30)), fa.FA_ERR_OVERLAP),          # lse on k
])
def test_validation_rejects(L, kw, code):
    assert call(L, **kw) == code


@pytest.mark.parametrize("window", [0, -1, -100])
def test_window_must_be_positive(L, window):
    assert L.fa_fwd_window(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), None,
                           1, 2, 1, 16, 16, 64, 0.125, window, None) == fa.FA_ERR_INVALID_ARG


def test_splitkv_workspace_and_default_splits(L):
    assert fa.splitkv_workspace_bytes(2, 4, 100, 128, 1) == 0
    o = 3 * 2 * 100 * 4 * 128 * 4
    assert fa.splitkv_workspace_bytes(2, 4, 100, 128, 3) == ((o + 255) // 256) * 256 + 3 * 2 * 4 * 100 * 4
    assert fa.splitkv_workspace_bytes(2, 4, 100, 128, 0) == 0 and fa.splitkv_workspace_bytes(2, 4, 100, 128, 999) == 0
    assert fa.splitkv_default_splits(8, 32, 32, 4096, 4096, 128, 148) == 1   # already fills the GPU
    bk = fa.tile_config(128)["block_k"]
    # GQA-packed decode: 4 x 8 units of 64 rows; the split minimising waves x (tiles per split + 1)
    assert fa.splitkv_default_splits(4, 32, 8, 16, 32768, 128, 148) == _split_model(4, 32, 8, 16, 32768, 148, bk)
    # one unit: as many splits as keep >= 4 key tiles each, within one wave
    assert fa.splitkv_default_splits(1, 1, 1, 1, 65536, 128, 148) == min(147, 65536 // bk // 4, 256) or \
        fa.splitkv_default_splits(1, 1, 1, 1, 65536, 128, 148) == _split_model(1, 1, 1, 1, 65536, 148, bk)
    assert fa.splitkv_default_splits(1, 1, 1, 1, 300, 64, 148) == 1          # too few key tiles
    assert fa.splitkv_default_splits(1, 6, 2, 1, 4096, 64, 148) >= 1         # n_rep = 3: not packed


def _split_model(B, Hq, Hkv, Nq, Nk, sms, bk=128):
    """The documented choice: fewest (waves x (tiles per split + 1)), >= 4 tiles per split."""
    n_rep = Hq // Hkv
    g = n_rep if (n_rep > 1 and 128 % n_rep == 0 and Nq < 128) else 1
    units = B * (Hq // g) * -(-(Nq * g) // 256)
    if units >= sms:
        return 1
    nkv = -(-Nk // bk)
    costs = [(-(-units * s // sms) * (-(-nkv // s) + 1), s) for s in range(1, 257) if s == 1 or nkv // s >= 4]
    return min(costs)[1]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk", [(4, 32, 32, 16, 32768), (1, 8, 1, 1, 8192), (2, 16, 2, 64, 100000),
                                            (1, 32, 8, 1, 1000), (3, 12, 4, 100, 50000)])
def test_splitkv_default_splits_model(L, B, Hq, Hkv, Nq, Nk):
    bk = fa.tile_config(128)["block_k"]
    assert fa.splitkv_default_splits(B, Hq, Hkv, Nq, Nk, 128, 148) == _split_model(B, Hq, Hkv, Nq, Nk, 148, bk)


def _splitkv(L, splits=4, ws=FAKE + (5 << 30), ws_bytes=1 << 30, out=FAKE + (3 << 30)):
    return L.fa_fwd_splitkv(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), out, FAKE + (4 << 30),
                            1, 2, 1, 16, 4096, 64, 0.125, 0, splits, ws, ws_bytes, None)


def test_splitkv_validation(L):
    assert _splitkv(L, splits=0) == fa.FA_ERR_INVALID_ARG
    assert _splitkv(L, splits=257) == fa.FA_ERR_INVALID_ARG
    assert _splitkv(L, ws=None) == fa.FA_ERR_INVALID_ARG
    assert _splitkv(L, ws_bytes=100) == fa.FA_ERR_INVALID_ARG
    assert _splitkv(L, ws=FAKE + (5 << 30) + 16) == fa.FA_ERR_MISALIGNED
    assert _splitkv(L, ws=FAKE + (3 << 30)) == fa.FA_ERR_OVERLAP            # workspace on out
    assert _splitkv(L) in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)


def _bwd(L, d=128, ws=FAKE + (12 << 30), ws_bytes=1 << 30, dq=FAKE + (5 << 30), causal=0, lse=FAKE + (4 << 30)):
    return L.fa_bwd(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (6 << 30), lse, dq,
                    FAKE + (7 << 30), FAKE + (8 << 30), 1, 2, 1, 64, 64, d, 0.125, causal, ws, ws_bytes, None)


def test_bwd_validation(L):
    assert fa.bwd_workspace_bytes(2, 4, 100, 128) == ((2 * 100 * 4 * 128 * 4 + 255) // 256) * 256 + 2 * 4 * 100 * 4
    assert _bwd(L, d=192) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM and _bwd(L, d=48) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM
    assert _bwd(L, causal=2) == fa.FA_ERR_INVALID_ARG
    assert _bwd(L, lse=None) == fa.FA_ERR_INVALID_ARG
    assert _bwd(L, ws=None) == fa.FA_ERR_INVALID_ARG
    assert _bwd(L, ws_bytes=10) == fa.FA_ERR_INVALID_ARG
    assert _bwd(L, ws=FAKE + (12 << 30) + 16) == fa.FA_ERR_MISALIGNED
    assert _bwd(L, dq=FAKE + (5 << 30) + 2) == fa.FA_ERR_MISALIGNED
    assert _bwd(L, dq=FAKE) == fa.FA_ERR_OVERLAP                       # dq over q
    assert _bwd(L, ws=FAKE + (7 << 30)) == fa.FA_ERR_OVERLAP           # workspace over dk
    assert _bwd(L) in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)
    assert L.fa_bwd_window(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (6 << 30),
                           FAKE + (4 << 30), FAKE + (5 << 30), FAKE + (7 << 30), FAKE + (8 << 30), 1, 2, 1, 64, 64,
                           128, 0.125, 0, FAKE + (12 << 30), 1 << 30, None) == fa.FA_ERR_INVALID_ARG   # W = 0


def test_fp8_validation(L):
    def call(d=128, ds=(1.0, 1.0, 1.0)):
        return L.fa_fwd_fp8(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (4 << 30),
                            1, 2, 1, 64, 64, d, 0.125, ds[0], ds[1], ds[2], 0, None)
    assert call(d=80) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM and call(d=96) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM
    assert call(d=64) in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)
    assert call(d=256) in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)
    assert call(ds=(0.0, 1.0, 1.0)) == fa.FA_ERR_INVALID_ARG
    assert call(ds=(1.0, float("inf"), 1.0)) == fa.FA_ERR_INVALID_ARG
    assert call(ds=(1.0, 1.0, -2.0)) == fa.FA_ERR_INVALID_ARG
    assert call() in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)


def test_partial_and_merge_validation(L):
    """Key-shard partial: 0 <= key_offset, key_offset + Nk <= Nk_total; merge: R >= 1."""
    def partial(key_offset=0, nk_total=64, Nk=64, d=128, o_part=FAKE + (3 << 30)):
        return L.fa_fwd_partial(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), o_part, FAKE + (4 << 30),
                                1, 2, 1, 16, Nk, d, 0.125, 1, key_offset, nk_total, None)
    assert partial(key_offset=-1) == fa.FA_ERR_INVALID_ARG
    assert partial(key_offset=1, nk_total=64) == fa.FA_ERR_INVALID_ARG        # shard runs past the end
    assert partial(d=48) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM
    assert partial(o_part=FAKE + (3 << 30) + 4) == fa.FA_ERR_MISALIGNED       # fp32 partial needs 16 bytes
    assert partial(o_part=FAKE) == fa.FA_ERR_OVERLAP                           # partial over q
    assert partial() in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)

    def merge(R=2, out=FAKE + (6 << 30), d=128):
        return L.fa_merge_partials(FAKE, FAKE + (2 << 30), R, out, FAKE + (7 << 30), 1, 2, 16, d, None)
    assert merge(R=0) == fa.FA_ERR_INVALID_ARG
    assert merge(d=100) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM
    assert merge(out=FAKE + 64) == fa.FA_ERR_OVERLAP                          # out over the partials
    assert merge() in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)


def test_withheld_load_validation(L):
    """The failure-path test entry: index >= 0, limit in 1 .. 10^6 us, then fa_fwd's checks."""
    def call(load=1, limit=20000, scale=0.125):
        return L.fa_test_withheld_load(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (4 << 30),
                                       1, 1, 1, 256, 256, scale, 0, load, limit, None)
    assert call(load=-1) == fa.FA_ERR_INVALID_ARG
    assert call(limit=0) == fa.FA_ERR_INVALID_ARG
    assert call(limit=2000000) == fa.FA_ERR_INVALID_ARG
    assert call(scale=-1.0) == fa.FA_ERR_INVALID_ARG
    assert call() in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)


def test_f16_entry_validates_like_bf16(L):
    args = (FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (4 << 30), 1, 2, 1, 64, 64)
    assert L.fa_fwd_f16(*args, 48, 0.125, 0, None) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM
    assert L.fa_fwd_f16(*args, 128, -1.0, 0, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd_f16(*args, 128, 0.125, 3, None) == fa.FA_ERR_INVALID_ARG
    assert L.fa_fwd_f16(*args, 128, 0.125, 1, None) in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)
    assert L.fa_bwd_f16(FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (6 << 30), FAKE + (4 << 30),
                        FAKE + (5 << 30), FAKE + (7 << 30), FAKE + (8 << 30), 1, 2, 1, 64, 64, 192, 0.125, 0,
                        FAKE + (12 << 30), 1 << 30, None) == fa.FA_ERR_UNSUPPORTED_HEAD_DIM


def test_empty_problems_are_noops(L):
    # no output rows: nothing to validate against the device, nothing launched
    assert call(L, B=0, q=None, k=None, v=None, out=None, lse=None) == fa.FA_OK
    assert call(L, Nq=0, q=None, out=None, lse=None) == fa.FA_OK


def test_valid_args_without_usable_device(L):
    """Arguments pass validation; the library must then refuse (no device here, or the
    fake pointers are not device memory on a GPU machine) instead of launching."""
    assert call(L) in (fa.FA_ERR_UNSUPPORTED_DEVICE, fa.FA_ERR_NOT_DEVICE_MEMORY)


def test_status_strings(L):
    for c in range(0, 9):
        s = fa.status_string(c)
        assert s and s != "unknown status"
    assert fa.status_string(99) == "unknown status"

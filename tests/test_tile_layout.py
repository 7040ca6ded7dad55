"""Host-side check of the forward kernel's on-chip layouts (no GPU): for every tiling that
fa_fwd.cu instantiates, a small host program built with nvcc from fa_kernel.cuh prints the
TMEM column ranges (S buffers, O tiles, P tiles) and the shared-memory regions, and this test
checks that they are disjoint, inside the 512 TMEM columns and the 227 KB a CTA may use,
aligned as TMA and the UMMA descriptors require, and that the register split fits the
launch budget.  The tilings are read from fa_fwd.cu itself, so a new one is covered."""
import re
import shutil
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
CSRC = ROOT / "exact_attention_146_b200" / "csrc"
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

TMEM_COLS = 512
SMEM_LIMIT = 232448          # 227 KB of opt-in shared memory per CTA on sm_100


def tilings():
    """(name, TileCfg argument list) for every `using CfgX = TileCfg<...>` of fa_fwd.cu; the
    templated ones once with bf16 and once with fp16 elements."""
    src = (CSRC / "fa_fwd.cu").read_text()
    out = []
    for m in re.finditer(r"^(template <bool H> )?using (Cfg\w+) = TileCfg<([^;]*)>;", src, re.M):
        args = m.group(3)
        if m.group(1):
            out.append((m.group(2) + "_bf16", args.replace("H", "false")))
            out.append((m.group(2) + "_f16", args.replace("H", "true")))
        else:
            out.append((m.group(2), args))
    return out


PROGRAM_HEAD = r'''
#include "fa_kernel.cuh"
#include <cstdio>
using namespace fa;
template <class C> void dump(const char *name) {
    printf("cfg %s D=%d BC=%d NQT=%d NS=%d NQB=%d SB=%d PSEP=%d SSHARE=%d FP8=%d PSPLIT=%d\n", name, C::D, C::BC,
           C::NQT, C::NS, C::NQB, C::SB, int(C::PSEP), int(C::SSHARE), int(C::FP8), int(C::PSPLIT));
    // TMEM: S buffers, O tiles, P tiles (columns [lo, hi))
    const int nS = C::SSHARE ? 1 : C::NQT * C::SB;
    for (int i = 0; i < nS; ++i) printf("tmem S%d %d %d\n", i, i * C::BC, (i + 1) * C::BC);
    for (int t = 0; t < C::NQT; ++t)
        printf("tmem O%d %d %d\n", t, C::O_COL0 + t * C::OST, C::O_COL0 + t * C::OST + ((C::D + 31) / 32) * 32);
    if (C::PSEP)
        for (int t = 0; t < C::NQT; ++t)
            printf("tmem P%d %d %d\n", t, C::P_COL0 + t * C::PCOLS, C::P_COL0 + (t + 1) * C::PCOLS);
    // shared memory (offsets from the 1024-aligned base) and the allocation
    printf("smem Q %d %d\n", C::SMEM_Q, C::SMEM_Q + C::NQT * C::NQB * C::Q_TILE);
    printf("smem KV %d %d\n", C::SMEM_KV, C::SMEM_KV + C::NS * C::KV_TILE);
    printf("smem BAR %d %d\n", C::SMEM_BAR, C::SMEM_BAR + C::NUM_BARS * 8);
    printf("smem MISC %d %d\n", C::SMEM_MISC, C::SMEM_MISC + 16);
    if (C::OSTAGE) printf("smem OST %d %d\n", C::SMEM_OST, C::SMEM_OST + 4 * C::NQT * C::OST_BYTES);
    printf("alloc %d %d\n", C::SMEM_BYTES, C::SMEM_NEEDED);
    printf("tiles %d %d %d\n", C::Q_TILE, C::KV_TILE, C::OST_BYTES);
    printf("bars %d %d\n", C::B_SEMPTY, C::NUM_BARS);
    printf("regs %d %d %d %d %d\n", int(C::REALLOC_REGS), C::SOFTMAX_REGS, C::CONTROL_REGS, C::LAUNCH_REGS, C::THREADS);
}
int main() {
'''


@pytest.fixture(scope="module")
def layouts(tmp_path_factory):
    if not Path(NVCC).exists():
        pytest.skip("nvcc not available")
    cfgs = tilings()
    assert len(cfgs) >= 10, cfgs
    body = "".join(f'    dump<TileCfg<{args}>>("{name}");\n' for name, args in cfgs)
    d = tmp_path_factory.mktemp("layout")
    src = d / "layout.cu"
    src.write_text(PROGRAM_HEAD + body + "    return 0;\n}\n")
    exe = d / "layout"
    res = subprocess.run([NVCC, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", f"-I{CSRC}", str(src),
                          "-o", str(exe)], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-3000:]
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    parsed = {}
    cur = None
    for line in out.splitlines():
        f = line.split()
        if f[0] == "cfg":
            cur = {"name": f[1], **{k: int(v) for k, v in (x.split("=") for x in f[2:])}, "tmem": {}, "smem": {}}
            parsed[f[1]] = cur
        elif f[0] in ("tmem", "smem"):
            cur[f[0]][f[1]] = (int(f[2]), int(f[3]))
        else:
            cur[f[0]] = tuple(int(x) for x in f[1:])
    assert set(parsed) == {n for n, _ in cfgs}
    return parsed


def disjoint(ranges):
    rs = sorted(ranges.items(), key=lambda kv: kv[1])
    for (na, (a0, a1)), (nb, (b0, b1)) in zip(rs, rs[1:]):
        assert a1 <= b0, f"{na} [{a0}, {a1}) overlaps {nb} [{b0}, {b1})"


def test_tmem_regions_disjoint_and_in_budget(layouts):
    for name, c in layouts.items():
        tm = c["tmem"]
        disjoint(tm)
        assert all(0 <= lo < hi <= TMEM_COLS for lo, hi in tm.values()), (name, tm)
        # the softmax reads a whole S row of BC columns and O in 32-column chunks
        assert all(lo % 32 == 0 for lo in (r[0] for r in tm.values())), (name, tm)
        n_s = sum(1 for k in tm if k.startswith("S"))
        if c["SSHARE"]:
            assert n_s == 1 and c["SB"] == 1 and c["NQT"] == 2 and c["PSEP"], name
            assert c["PSPLIT"] == 0, name
        else:
            assert n_s == c["NQT"] * c["SB"], name
        if c["PSEP"]:
            # one row of P: BC keys of 2 bytes (bf16 / fp16) or 1 byte (E4M3) per 32-bit column
            width = c["BC"] // (4 if c["FP8"] else 2)
            assert all(hi - lo == width for k, (lo, hi) in tm.items() if k.startswith("P")), (name, tm)


def test_shared_memory_regions(layouts):
    for name, c in layouts.items():
        sm = c["smem"]
        disjoint(sm)
        alloc, needed = c["alloc"]
        q_tile, kv_tile, ost_bytes = c["tiles"]
        assert needed <= alloc <= SMEM_LIMIT, (name, alloc)
        # 1024 bytes of slack are requested so the kernel can align its base to 1024
        assert max(hi for _, hi in sm.values()) + 1024 <= alloc, (name, sm, alloc)
        # TMA boxes and 128-byte-swizzled UMMA operands start on 1024-byte boundaries
        assert sm["Q"][0] % 1024 == 0 and sm["KV"][0] % 1024 == 0 and q_tile % 1024 == 0 and kv_tile % 1024 == 0
        if "OST" in sm:
            assert sm["OST"][0] % 1024 == 0 and ost_bytes % 1024 == 0, name
        assert sm["BAR"][0] % 8 == 0, name
        # one CTA per SM: each CTA allocates all 512 TMEM columns
        assert alloc >= 120 * 1024, name
        # the SEMPTY barrier (last index) lies inside the barrier block
        b_sempty, num_bars = c["bars"]
        assert b_sempty == num_bars - 1, name


def test_register_split_fits_launch(layouts):
    for name, c in layouts.items():
        realloc, soft, ctrl, launch, threads = c["regs"]
        assert launch * threads <= 65536, name
        if realloc:
            softmax_threads = threads - 128
            assert soft * softmax_threads + ctrl * 128 <= launch * threads, name
            assert soft % 8 == 0 and ctrl % 8 == 0 and 24 <= ctrl <= soft <= 256, name


def test_shared_s_tilings_are_the_ones_documented(layouts):
    """The head dims whose two query tiles share one S buffer (P in columns of its own)."""
    shared = sorted({(c["D"], bool(c["FP8"])) for c in layouts.values() if c["SSHARE"]})
    assert shared == [(64, True), (80, False), (96, False), (128, False), (128, True), (192, False)], shared

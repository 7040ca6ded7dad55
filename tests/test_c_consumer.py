"""The C ABI from plain C: a C99 program that includes include/fa.h, links libfa.so and calls
the host-only entry points (no GPU needed): version, status strings, tiling, the split-KV
and backward size helpers, and argument validation."""
import subprocess
import tempfile
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fa.h"

int main(void) {
    int bq = 0, bk = 0, nqt = 0, ns = 0;
    if (fa_version() != 100) return 1;
    if (fa_tile_config(128, &bq, &bk, &nqt, &ns) != FA_OK || bq != 128 || bk < 64 || bk % 64 != 0) return 2;
    if (fa_tile_config(100, NULL, NULL, NULL, NULL) != FA_ERR_UNSUPPORTED_HEAD_DIM) return 3;
    if (strlen(fa_status_string(FA_ERR_OVERLAP)) == 0) return 4;
    if (fa_splitkv_workspace_bytes(1, 2, 16, 128, 1) != 0) return 5;
    if (fa_bwd_workspace_bytes(1, 2, 16, 64) == 0) return 6;
    /* invalid arguments are rejected before any CUDA call */
    if (fa_fwd((void *)16, (void *)16, (void *)16, (void *)16, NULL, 1, 3, 2, 4, 4, 128, 0.1f, 0, NULL)
        != FA_ERR_INVALID_ARG) return 7;          /* Hq not a multiple of Hkv */
    if (fa_fwd_window((void *)16, (void *)16, (void *)16, (void *)16, NULL, 1, 2, 1, 4, 4, 128, 0.1f, 0, NULL)
        != FA_ERR_INVALID_ARG) return 8;          /* window < 1 */
    if (fa_fwd(NULL, NULL, NULL, NULL, NULL, 0, 1, 1, 0, 0, 128, 0.1f, 0, NULL) != FA_OK) return 9;  /* empty */
    printf("ok %d\n", FA_SPLITKV_STATIC_SCRATCH_BYTES > 0);
    return 0;
}
"""


def test_c_program_against_header_and_library():
    lib = ROOT / "exact_attention_146_b200" / "libfa.so"
    if not lib.exists():
        from exact_attention_146_b200 import build
        build.build()
    with tempfile.TemporaryDirectory() as td:
        src = Path(td) / "consumer.c"
        exe = Path(td) / "consumer"
        src.write_text(PROGRAM)
        cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", f"-I{ROOT / 'include'}", str(src),
                             f"-L{lib.parent}", "-lfa", f"-Wl,-rpath,{lib.parent}", "-o", str(exe)],
                            capture_output=True, text=True)
        assert cc.returncode == 0, cc.stderr
        run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
        assert run.returncode == 0, f"check {run.returncode} failed: {run.stdout} {run.stderr}"
        assert run.stdout.strip() == "ok 1"

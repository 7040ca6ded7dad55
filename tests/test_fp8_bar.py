"""The FP8 parity bar (tests/_fp8_bar.py) on the CPU: a model of the FP8 kernel's own
rounding passes it, and plausible kernel mistakes, built from the oracle, fail it.

The model follows the kernel's arithmetic in fp64 except for the roundings the bar is
derived from: keys in tiles of 128, a reference maximum that is raised (and O, l rescaled)
only when a tile's maximum exceeds it by more than 2^8, each weight 2^(x - m) rounded to
E4M3 (torch's round-to-nearest-even cast) before it multiplies V, the row sum over the
unrounded weights, and O / l rounded to bf16."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import _fp8_bar

SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


def inputs(B, Hq, Hkv, N, seed, q_mult=1.0):
    w = synth.Workload("fp8bar", 7000 + seed, B, Hq, Hkv, N, N, 128, False, q_mult=q_mult, seed=seed, dtype="e4m3")
    return synth.make_inputs(w)


def kernel_model(x, rows, scale, causal, descale, skip_tile=None):
    """The FP8 kernel's rounding, row by row (see the module docstring)."""
    q = _fp8_bar.e4m3_values(x["q"]) * descale[0]
    k = _fp8_bar.e4m3_values(x["k"]) * descale[1]
    v8 = _fp8_bar.e4m3_values(x["v"])
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    out = np.zeros((len(rows), d))
    for r, (b, hq, i) in enumerate(rows):
        g = hq // (Hq // Hkv)
        last = min(Nk - 1, i + Nk - Nq) if causal else Nk - 1
        x2 = (k[b, :last + 1, g] @ q[b, i, hq]) * scale * math.log2(math.e)
        m, l, o = -math.inf, 0.0, np.zeros(d)
        for j0 in range(0, last + 1, 128):
            if skip_tile is not None and j0 // 128 == skip_tile:
                continue
            xt = x2[j0:j0 + 128]
            mx = float(xt.max())
            if m == -math.inf:
                m = mx
            elif mx > m + 8.0:
                a = 2.0 ** (m - mx)
                o, l, m = o * a, l * a, mx
            p = np.exp2(xt - m)
            p8 = torch.from_numpy(p).to(torch.float8_e4m3fn).to(torch.float64).numpy()
            o = o + p8 @ v8[b, j0:j0 + len(xt), g]
            l += float(p.sum())
        res = descale[2] * o / l if l > 0 else o
        out[r] = torch.from_numpy(res).to(torch.bfloat16).to(torch.float64).numpy()
    return out


def all_rows(B, Hq, Nq):
    return np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in range(Nq)], dtype=np.int32)


def bar_rejects(O, Oref, tol, rel_bound):
    try:
        _fp8_bar.check_fp8(O, None, Oref, None, tol, rel_bound)
        return False
    except AssertionError:
        return True


CASES = [
    # (B, Hq, Hkv, N, causal, q_mult, descale)
    (1, 2, 1, 300, False, 1.0, (1.0, 1.0, 1.0)),
    (1, 2, 1, 300, True, 1.0, (1.0, 1.0, 1.0)),
    (1, 2, 2, 600, False, 4.0, (1.0, 1.0, 1.0)),   # large logits: the lazy rescale runs
    (2, 4, 2, 260, True, 4.0, (0.5, 2.0, 0.25)),   # GQA and non-unit factors
]


@pytest.mark.parametrize("case", CASES)
def test_kernel_model_passes(orc, case):
    B, Hq, Hkv, N, causal, qm, ds = case
    x = inputs(B, Hq, Hkv, N, seed=N + Hq, q_mult=qm)
    rows = all_rows(B, Hq, N)
    Oref, _ = orc.rows_fp8(x["q"], x["k"], x["v"], rows, SCALE, causal, descale=ds)
    tol, rel_bound = _fp8_bar.fp8_bar(orc, x, rows, SCALE, causal, ds, Oref)
    Om = kernel_model(x, rows, SCALE, causal, ds)
    res = _fp8_bar.check_fp8(Om, None, Oref, None, tol, rel_bound, f"model {case}")
    # the bar is not loose against the model: the model's error uses a fair share of it
    assert res["rel_l2_O"] > 0.05 * rel_bound, res
    print(case, res)


@pytest.mark.parametrize("case", [c for c in CASES if not c[4]])
def test_bar_rejects_mistakes(orc, case):
    """Mistakes a kernel could make, each built from the oracle: a 128-key tile left out,
    the V factor applied twice, the Q and K factors applied twice."""
    B, Hq, Hkv, N, causal, qm, _ = case
    ds = (0.75, 1.5, 0.5)
    x = inputs(B, Hq, Hkv, N, seed=N + Hq, q_mult=qm)
    rows = all_rows(B, Hq, N)
    Oref, _ = orc.rows_fp8(x["q"], x["k"], x["v"], rows, SCALE, causal, descale=ds)
    tol, rel_bound = _fp8_bar.fp8_bar(orc, x, rows, SCALE, causal, ds, Oref)
    assert not bar_rejects(kernel_model(x, rows, SCALE, causal, ds), Oref, tol, rel_bound)
    keep = np.r_[0:128, 256:N]
    O_drop, _ = orc.rows_fp8(x["q"], np.ascontiguousarray(x["k"][:, keep]), np.ascontiguousarray(x["v"][:, keep]),
                             rows, SCALE, causal, descale=ds)
    assert bar_rejects(O_drop, Oref, tol, rel_bound), "dropped key tile passed"
    O_v, _ = orc.rows_fp8(x["q"], x["k"], x["v"], rows, SCALE, causal, descale=(ds[0], ds[1], ds[2] ** 2))
    assert bar_rejects(O_v, Oref, tol, rel_bound), "V factor twice passed"
    O_qk, _ = orc.rows_fp8(x["q"], x["k"], x["v"], rows, SCALE, causal, descale=(ds[0] ** 2, ds[1] ** 2, ds[2]))
    assert bar_rejects(O_qk, Oref, tol, rel_bound), "Q and K factors twice passed"
    # one output row stored in its neighbour's place (an epilogue indexing slip)
    r = len(rows) // 2
    b, h, i = (int(c) for c in rows[r])
    O_nb, _ = orc.rows_fp8(x["q"], x["k"], x["v"], np.array([(b, h, (i + 1) % N)], dtype=np.int32), SCALE, causal,
                           descale=ds)
    O_row = Oref.copy()
    O_row[r] = O_nb[0]
    assert bar_rejects(O_row, Oref, tol, rel_bound), "misplaced row passed"
    # the last key masked out (a tail-mask slip): the element bar catches it at N = 300,
    # where the previous bar (2^-4 max|V| and 2^-4 relative L2) let it pass
    O_key, _ = orc.rows_fp8(x["q"], np.ascontiguousarray(x["k"][:, :N - 1]), np.ascontiguousarray(x["v"][:, :N - 1]),
                            rows, SCALE, causal, descale=ds)
    assert bar_rejects(O_key, Oref, tol, rel_bound), "one key dropped passed"


def test_full_size_rows(orc):
    """At the benchmark's size (N = 4096, d = 128) on sampled rows: the kernel model
    passes; one dropped key tile (1 of 32) and one misplaced row fail."""
    B, Hq, N = 1, 2, 4096
    x = inputs(B, Hq, Hq, N, seed=5)
    rng = np.random.default_rng(1)
    rows = np.array([(0, int(rng.integers(Hq)), int(rng.integers(N))) for _ in range(24)], dtype=np.int32)
    ds = (1.0, 1.0, 1.0)
    Oref, _ = orc.rows_fp8(x["q"], x["k"], x["v"], rows, SCALE, False, descale=ds)
    tol, rel_bound = _fp8_bar.fp8_bar(orc, x, rows, SCALE, False, ds, Oref)
    Om = kernel_model(x, rows, SCALE, False, ds)
    res = _fp8_bar.check_fp8(Om, None, Oref, None, tol, rel_bound, "model full size")
    keep = np.r_[0:1024, 1152:N]
    O_drop, _ = orc.rows_fp8(x["q"], np.ascontiguousarray(x["k"][:, keep]), np.ascontiguousarray(x["v"][:, keep]),
                             rows, SCALE, False, descale=ds)
    assert bar_rejects(O_drop, Oref, tol, rel_bound), "dropped key tile passed at full size"
    b, h, i = (int(c) for c in rows[7])
    O_nb, _ = orc.rows_fp8(x["q"], x["k"], x["v"], np.array([(b, h, (i + 1) % N)], dtype=np.int32), SCALE, False,
                           descale=ds)
    O_row = Oref.copy()
    O_row[7] = O_nb[0]
    assert bar_rejects(O_row, Oref, tol, rel_bound), "misplaced row passed at full size"
    print("full size", res)

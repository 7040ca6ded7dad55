"""Shared parity machinery: run the CUDA path through the C ABI on seeded inputs and
compare with the CPU oracle element by element.

Acceptance (the stated target for bf16 O against the fp64 oracle):
    max |dO| <= 2e-2,  ||dO||_2 / ||O||_2 <= 5e-3,  max |dLSE| <= 1e-3
with -inf LSE (rows without a visible key) required to match exactly."""
from __future__ import annotations

import numpy as np

import synth

TOL_O_MAX = 2e-2
TOL_O_REL_L2 = 5e-3
TOL_LSE = 1e-3
# FP8 (E4M3) inputs: the bar is derived from the E4M3 rounding of P (tests/_fp8_bar.py).


def to_device(bits, torch, dtype="bf16"):
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(tdt).cuda()


def bf16_to_f64(t):
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def run_cuda_fp8(x, scale, causal, descale=(1.0, 1.0, 1.0)):
    """fa_fwd_fp8 through the C ABI on E4M3 bytes; out/lse pre-filled with NaN."""
    import torch
    import exact_attention_146_b200 as fa
    q, k, v = (torch.from_numpy(np.ascontiguousarray(x[n], dtype=np.uint8)).cuda() for n in ("q", "k", "v"))
    B, Nq, Hq, d = q.shape
    out = torch.full((B, Nq, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, Nq), float("nan"), dtype=torch.float32, device="cuda")
    fa.fa_fwd_fp8(q, k, v, descale=descale, causal=causal, scale=scale, out=out, lse=lse)
    st, word = fa.device_status()
    assert st == fa.FA_OK, f"device status {st} (word {word:#x})"
    torch.cuda.synchronize()
    return bf16_to_f64(out), lse.cpu().numpy().astype(np.float64)


def compare_fp8(orc, x, O, L, scale, causal, descale=(1.0, 1.0, 1.0), what="", rows=None):
    """The FP8 bar (tests/_fp8_bar.py) on the listed (b, hq, i) rows (all rows if None) of a
    full-size output O [B, Nq, Hq, d] and L [B, Hq, Nq]; returns and prints the observed errors."""
    from tests import _fp8_bar
    if rows is None:
        B, Nq, Hq, _ = O.shape
        rows = np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in range(Nq)], dtype=np.int32)
    Oref, Lref = orc.rows_fp8(x["q"], x["k"], x["v"], rows, scale, causal, descale=descale)
    Og = O[rows[:, 0], rows[:, 2], rows[:, 1], :]
    Lg = L[rows[:, 0], rows[:, 1], rows[:, 2]]
    tol, rel_bound = _fp8_bar.fp8_bar(orc, x, rows, scale, causal, descale, Oref)
    res = _fp8_bar.check_fp8(Og, Lg, Oref, Lref, tol, rel_bound, what)
    print("fp8", what, res)
    return res


def run_cuda(x, scale, causal, with_lse=True, canary=True, window=None, num_splits=None, dtype="bf16"):
    """fa_fwd (fa_fwd_f16 for dtype "f16") through the C ABI; out/lse pre-filled with NaN
    so unwritten rows show up."""
    import torch
    import exact_attention_146_b200 as fa
    if dtype == "e4m3":
        assert window is None and num_splits is None and with_lse
        return run_cuda_fp8(x, scale, causal)
    q, k, v = (to_device(x[n], torch, dtype) for n in ("q", "k", "v"))
    out = torch.full_like(q, float("nan")) if canary else torch.empty_like(q)
    B, Nq, Hq, d = q.shape
    lse = torch.full((B, Hq, Nq), float("nan"), dtype=torch.float32, device="cuda") if with_lse else None
    fa.fa_fwd(q, k, v, causal=causal, scale=scale, out=out, lse=lse, return_lse=with_lse, window=window,
              num_splits=num_splits)
    st, word = fa.device_status()
    assert st == fa.FA_OK, f"device status {st} (word {word:#x})"
    torch.cuda.synchronize()
    return bf16_to_f64(out), (lse.cpu().numpy().astype(np.float64) if with_lse else None)


def compare(O, L, Oref, Lref, what="", tol_o_max=TOL_O_MAX, tol_rel=TOL_O_REL_L2):
    """Apply the acceptance bar; returns the error figures."""
    assert O.shape == Oref.shape, (O.shape, Oref.shape)
    assert np.isfinite(O).all(), f"{what}: non-finite O (unwritten or overflowed rows)"
    dO = np.abs(O - Oref)
    max_o = float(dO.max()) if dO.size else 0.0
    nrm = float(np.linalg.norm(Oref))
    rel = float(np.linalg.norm(O - Oref) / nrm) if nrm > 0 else float(np.linalg.norm(O))
    res = {"max_abs_O": max_o, "rel_l2_O": rel}
    if L is not None:
        fin = np.isfinite(Lref)
        assert np.array_equal(np.isfinite(L), fin), f"{what}: LSE finiteness differs"
        assert np.array_equal(L[~fin], Lref[~fin]), f"{what}: LSE infinities differ"
        res["max_abs_LSE"] = float(np.abs(L[fin] - Lref[fin]).max()) if fin.any() else 0.0
    assert max_o <= tol_o_max, f"{what}: max|dO| = {max_o:.3e}"
    assert rel <= tol_rel or nrm == 0, f"{what}: rel L2 = {rel:.3e}"
    if L is not None:
        assert res["max_abs_LSE"] <= TOL_LSE, f"{what}: max|dLSE| = {res['max_abs_LSE']:.3e}"
    return res


def workload_splits(w: synth.Workload) -> int | None:
    """The split count a workload runs with (the library's default for split-KV ones)."""
    if not w.splitkv:
        return None
    import exact_attention_146_b200 as fa
    return fa.splitkv_default_splits(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, 148)


def sample_rows(w: synth.Workload, n: int, seed: int = 0):
    """Seeded (b, hq, i) triples: random rows plus every 128-row tile boundary and the
    ragged tail of a few heads."""
    rng = np.random.default_rng(seed)
    rows = set()
    for _ in range(n):
        rows.add((int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.Nq))))
    for (b, h) in [(0, 0), (w.B - 1, w.Hq - 1)]:
        for i in list(range(0, w.Nq, 128)) + [min(w.Nq - 1, i + 127) for i in range(0, w.Nq, 128)] + [w.Nq - 1]:
            rows.add((b, h, i))
    return np.array(sorted(rows), dtype=np.int32)

"""The parity bar of the FP8 (E4M3) forward, derived from the arithmetic the kernel does.

The FP8 forward (the FlashAttention-3 e4m3 forward the datacanvas.csdn.net head-dim page
names) differs from the definition in one rounding that matters: every unnormalised weight
p_ij = 2^(x_ij - m) is rounded to E4M3 (round to nearest even) before P V, while the row
sum l_i uses the unrounded p (as the LSE does).  The reference m is the kernel's running
maximum, which lags the true row maximum by at most 2^8 (the lazy-rescale threshold), so
p <= 256 < 448 (no saturation) and l_i >= 1.  Per weight, in units of the normalised
probability w_ij = p_ij / l_i of the oracle:

  * normal E4M3 (p >= 2^-6): |p^ - p| <= 2^-4 p          -> error <= 2^-4 w_ij
  * subnormal (spacing 2^-9): |p^ - p| <= 2^-10           -> error <= 2^-10 / l_i <= 2^-10 w_max,i
    (the kernel's reference max is at most the true one, so 1 / l_i <= 1 / Z_i = w_max,i)
  * p < 2^-10 flushes to zero: error = w_ij, which only happens where
    w_ij < 2^-10 w_max,i; those errors are one-signed and counted deterministically (D).

So with e_ij = max(2^-4 w_ij, 2^-10 w_max,i), the rounding part of the output error is
R_ic = sum_j eps_ij V_jc with |eps_ij| <= e_ij.  On top come the bf16 rounding of O
(<= 2^-9 |O|) and fp32 accumulation (<= 2^-12 sum_j w_ij |V_jc| over a few thousand keys).

Two bars follow:
  * per element: |dO_ic| <= min(sum_j e_ij |V_jc|, sqrt(2 ln(2n/delta) sum_j e_ij^2 V_jc^2))
                            + D_ic + 2^-9 |O_ic| + 2^-12 A_ic + 1e-6,
    the worst case and, for independent zero-mean rounding errors (the probabilistic
    rounding-error model of Higham and Mary, SIAM J. Sci. Comput. 2019), Hoeffding's
    inequality with a union bound over the n elements (delta = 1e-6);
  * relative L2: ||dO|| <= 2 sqrt(sum_ic sum_j e_ij^2 V_jc^2 / 3) + ||D|| + ||small terms||,
    divided by ||O||: under the same model an error uniform in +-e has variance e^2 / 3,
    so the expected ||R||^2 is at most sum e^2 V^2 / 3, and the bar allows twice that norm.
The LSE bar stays 1e-3 (the LSE uses the unrounded exponentials).

The bar is computed from the oracle's own probabilities: E4M3 values are exactly bf16
values, so the oracle's pinned bf16 `probs` entry point, on the bf16 encoding of the
dequantised Q, K and the logit scale times the Q and K factors, gives w exactly.
"""
from __future__ import annotations

import math

import numpy as np

U_E4M3 = 2.0 ** -4        # unit roundoff of E4M3 (3 mantissa bits)
SUB_HALF = 2.0 ** -10     # half the E4M3 subnormal spacing 2^-9
U_BF16 = 2.0 ** -9        # unit roundoff of bf16 (7 mantissa bits), the output rounding
ACC = 2.0 ** -12          # fp32 accumulation over a few thousand terms, generously
DELTA = 1e-6              # failure probability of the Hoeffding union bound


def e4m3_values(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def bf16_bits(values):
    """Exact bf16 bit patterns of values that are representable in bf16 (E4M3 values are)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float64)).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float64).numpy(), values), "value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def _head_inputs(x, b, hq, descale):
    q8, k8 = x["q"], x["k"]
    Hq, Hkv = q8.shape[2], k8.shape[2]
    g = hq // (Hq // Hkv)
    return e4m3_values(q8[b:b + 1, :, hq:hq + 1]), e4m3_values(k8[b:b + 1, :, g:g + 1])


def head_weights(orc, x, b, hq, scale, causal, descale):
    """P [Nq, Nk] of one (b, hq) head: the oracle's probabilities on the bf16 encoding of
    the E4M3 values, with the Q and K factors folded into the logit scale."""
    qv, kv = _head_inputs(x, b, hq, descale)
    vz = np.zeros_like(kv)
    _, _, P = orc.probs(bf16_bits(qv), bf16_bits(kv), bf16_bits(vz), scale * descale[0] * descale[1], causal)
    return P[0, 0]


def row_weights(orc, x, b, hq, i, scale, causal, descale):
    """w over the keys one output row sees, as a one-query problem (a causal row is unmasked
    attention over its prefix of keys 0 .. i + Nk - Nq)."""
    Nq, Nk = x["q"].shape[1], x["k"].shape[1]
    last = min(Nk - 1, i + Nk - Nq) if causal else Nk - 1
    if last < 0:
        return np.zeros(0)
    qv, kv = _head_inputs(x, b, hq, descale)
    qv, kv = qv[:, i:i + 1], kv[:, :last + 1]
    _, _, P = orc.probs(bf16_bits(qv), bf16_bits(kv), bf16_bits(np.zeros_like(kv)), scale * descale[0] * descale[1],
                        False)
    return P[0, 0, 0]


def fp8_bar(orc, x, rows, scale, causal, descale, Oref):
    """(tol_abs [n, d], rel_bound) for the listed (b, hq, i) rows whose oracle outputs are
    Oref [n, d]."""
    v_all = descale[2] * e4m3_values(x["v"])
    Hq, Hkv = x["q"].shape[2], x["k"].shape[2]
    n_rep = Hq // Hkv
    n_el = max(1, Oref.size)
    z = math.sqrt(2.0 * math.log(2.0 * n_el / DELTA))
    tol = np.zeros_like(Oref)
    s2_total = 0.0
    det_sq = 0.0
    Nq, Nk = x["q"].shape[1], x["k"].shape[1]
    heads = {}
    for r, (b, hq, i) in enumerate(rows):
        heads.setdefault((int(b), int(hq)), []).append((r, int(i)))
    for (b, hq), members in heads.items():
        # a whole head in one oracle call when many of its rows are asked for
        P = head_weights(orc, x, b, hq, scale, causal, descale) if 4 * len(members) >= Nq else None
        V_head = v_all[b, :, hq // n_rep, :]
        idx = np.array([r for r, _ in members])
        qi = np.array([i for _, i in members])
        if P is not None:
            W = P[qi]
        else:
            W = np.zeros((len(members), Nk))
            for n, i in enumerate(qi):
                w = row_weights(orc, x, b, hq, int(i), scale, causal, descale)
                W[n, :len(w)] = w
        # keys each row sees (the rest carry no weight and no rounding)
        nk = np.clip(qi + Nk - Nq + 1, 0, Nk) if causal else np.full(len(qi), Nk)
        seen = np.arange(Nk)[None, :] < nk[:, None]
        aV = np.abs(V_head)
        wmax = W.max(axis=1, keepdims=True)
        E = np.where(seen, np.maximum(U_E4M3 * W, SUB_HALF * wmax), 0.0)
        flush = np.where(seen & (W < SUB_HALF * wmax), W, 0.0)
        A = W @ aV
        D = flush @ aV
        S2 = (E * E) @ (V_head * V_head)
        small = U_BF16 * np.abs(Oref[idx]) + ACC * A + 1e-6
        worst = E @ aV
        t = np.minimum(worst, z * np.sqrt(S2)) + D + small
        t[nk == 0] = 1e-6
        tol[idx] = t
        s2_total += float(S2.sum())
        det_sq += float(((D + small) ** 2).sum())
    nrm = float(np.linalg.norm(Oref))
    rel = (2.0 * math.sqrt(s2_total / 3.0) + math.sqrt(det_sq)) / nrm if nrm > 0 else 0.0
    return tol, rel


def check_fp8(O, L, Oref, Lref, tol, rel_bound, what=""):
    """Apply the derived FP8 bar; returns the observed error figures and the bar."""
    assert O.shape == Oref.shape, (O.shape, Oref.shape)
    assert np.isfinite(O).all(), f"{what}: non-finite O"
    dO = np.abs(O - Oref)
    nrm = float(np.linalg.norm(Oref))
    rel = float(np.linalg.norm(O - Oref) / nrm) if nrm > 0 else float(np.linalg.norm(O))
    worst_ratio = float((dO / tol).max()) if dO.size else 0.0
    res = {"max_abs_O": float(dO.max()) if dO.size else 0.0, "rel_l2_O": rel, "rel_bar": rel_bound,
           "max_err_over_elementwise_bar": worst_ratio}
    if L is not None:
        fin = np.isfinite(Lref)
        assert np.array_equal(np.isfinite(L), fin), f"{what}: LSE finiteness differs"
        assert np.array_equal(L[~fin], Lref[~fin]), f"{what}: LSE infinities differ"
        res["max_abs_LSE"] = float(np.abs(L[fin] - Lref[fin]).max()) if fin.any() else 0.0
        assert res["max_abs_LSE"] <= 1e-3, f"{what}: max|dLSE| = {res['max_abs_LSE']:.3e}"
    assert worst_ratio <= 1.0, f"{what}: |dO| above the element bar (worst ratio {worst_ratio:.3f})"
    assert rel <= rel_bound or nrm == 0, f"{what}: rel L2 = {rel:.3e} > bar {rel_bound:.3e}"
    return res

"""Independent checks ("pins") of the CPU oracle.  None of them calls back into the
oracle's own arithmetic; each states a fact the pages or plain mathematics fix:

* brute force in 40-digit decimal arithmetic, straight from softmax(x_i) = e^{x_i} /
  sum_j e^{x_j} (no max subtraction needed at that precision);
* closed forms of special cases (one key, constant V, zero Q, causal row 0);
* invariants (P rows sum to one, GQA equals MHA with K/V repeated per the
  repeat_interleave expansion, key permutation invariance, causal = non-causal on
  the visible prefix);
* a second statement of the method: the block-wise online-softmax recurrence of the
  hwcomputing.csdn.net FlashAttention article (section "online softmax"), with the
  scale applied, run in fp64 at several block sizes.

Each pin is a function taking an oracle object and raising AssertionError on a
mismatch, so the mutation test can run every pin against deliberately broken builds.
"""
from __future__ import annotations

import math
from decimal import Decimal, getcontext

import numpy as np

import synth

TOL = 1e-12


def bits_f64(bits, dtype="bf16"):
    if dtype == "f16":   # numpy's own IEEE half, widened (exact)
        return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def tiny_inputs(B, Hq, Hkv, Nq, Nk, d, seed, q_mult=1.0, dtype="bf16"):
    w = synth.Workload("tiny", 1000 + seed, B, Hq, Hkv, Nq, Nk, d, False, q_mult=q_mult, seed=seed, dtype=dtype)
    return synth.make_inputs(w)


def visible(i, j, Nq, Nk, causal, window=0):
    """Causal reading: keep the diagonal, align bottom-right (j <= i + Nk - Nq); a window
    of W keys ends at that diagonal (i + Nk - Nq - W < j)."""
    diag = i + (Nk - Nq)
    if window and j <= diag - window:
        return False
    return (not causal and not window) or j <= diag


# ---------------------------------------------------------------- brute force

def e4m3_f64(bits):
    """OCP E4M3 bytes widened by torch's own float8_e4m3fn type (exact)."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def brute_force_decimal(x, scale, causal, prec=40, window=0, dtype="bf16"):
    """O and LSE by the definition in `prec`-digit decimal arithmetic (tiny inputs)."""
    return brute_force_values(*(bits_f64(x[n], dtype) for n in ("q", "k", "v")), scale, causal, prec, window)


def brute_force_values(q, k, v, scale, causal, prec=40, window=0):
    """The same on already-decoded float64 arrays q, k, v."""
    getcontext().prec = prec
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    rep = Hq // Hkv
    D = Decimal
    sc = D(float(scale))
    O = np.zeros((B, Nq, Hq, d))
    L = np.zeros((B, Hq, Nq))
    kd = [[[[D(float(k[b, j, g, c])) for c in range(d)] for g in range(Hkv)] for j in range(Nk)] for b in range(B)]
    vd = [[[[D(float(v[b, j, g, c])) for c in range(d)] for g in range(Hkv)] for j in range(Nk)] for b in range(B)]
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            for i in range(Nq):
                qi = [D(float(q[b, i, h, c])) for c in range(d)]
                num = [D(0)] * d
                Z = D(0)
                for j in range(Nk):
                    if not visible(i, j, Nq, Nk, causal, window):
                        continue
                    s = sc * sum(qi[c] * kd[b][j][g][c] for c in range(d))
                    e = s.exp()
                    Z += e
                    for c in range(d):
                        num[c] += e * vd[b][j][g][c]
                if Z == 0:
                    O[b, i, h, :] = 0.0
                    L[b, h, i] = -math.inf
                else:
                    O[b, i, h, :] = [float(n / Z) for n in num]
                    L[b, h, i] = float(Z.ln())
    return O, L


# ---------------------------------------------------------------- second statement

def online_softmax_blocks(x, scale, causal, block, window=0):
    """The block-wise recurrence: running row max m, running sum l, output rescaled by
    exp(m_old - m_new) at every block, divided by l at the end (fp64)."""
    q, k, v = (bits_f64(x[n]) for n in ("q", "k", "v"))
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    rep = Hq // Hkv
    O = np.zeros((B, Nq, Hq, d))
    L = np.zeros((B, Hq, Nq))
    ii = np.arange(Nq)[:, None]
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            Q = q[b, :, h, :]
            m = np.full(Nq, -np.inf)
            l = np.zeros(Nq)
            acc = np.zeros((Nq, d))
            for j0 in range(0, Nk, block):
                Kb = k[b, j0:j0 + block, g, :]
                Vb = v[b, j0:j0 + block, g, :]
                s = scale * (Q @ Kb.T)
                if causal or window:
                    jj = np.arange(j0, j0 + Kb.shape[0])[None, :]
                    diag = ii + (Nk - Nq)
                    keep = jj <= diag
                    if window:
                        keep &= jj > diag - window
                    s = np.where(keep, s, -np.inf)
                m_new = np.maximum(m, s.max(axis=1))
                safe = np.where(np.isfinite(m_new), m_new, 0.0)
                corr = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
                p = np.exp(s - safe[:, None])
                acc = acc * corr[:, None] + p @ Vb
                l = l * corr + p.sum(axis=1)
                m = m_new
            nz = l > 0
            O[b, :, h, :] = np.where(nz[:, None], acc / np.where(nz, l, 1.0)[:, None], 0.0)
            L[b, h, :] = np.where(nz, m + np.log(np.where(nz, l, 1.0)), -np.inf)
    return O, L


def assert_close(a, b, tol=TOL, what=""):
    a, b = np.asarray(a), np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin), f"{what}: finiteness differs"
    assert np.array_equal(a[~fin], b[~fin]), f"{what}: infinities differ"
    if fin.any():
        err = np.abs(a[fin] - b[fin]) / np.maximum(1.0, np.abs(b[fin]))
        assert err.max() <= tol, f"{what}: max rel err {err.max():.3e} > {tol}"


# ---------------------------------------------------------------- the pins

BRUTE_CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, seed
    (1, 1, 1, 5, 7, 32, False, 1),
    (1, 2, 1, 6, 6, 64, True, 2),
    (2, 4, 2, 9, 9, 16, True, 3),
    (1, 4, 1, 11, 5, 80, True, 4),     # Nq > Nk: first rows see no key
    (1, 2, 2, 4, 13, 96, True, 5),     # Nq < Nk: bottom-right alignment
    (1, 1, 1, 3, 4, 128, False, 6),
    (1, 3, 3, 3, 3, 192, False, 7),
    (1, 1, 1, 2, 3, 256, True, 8),
]


def pin_brute_force(orc):
    for (B, Hq, Hkv, Nq, Nk, d, causal, seed) in BRUTE_CASES:
        x = tiny_inputs(B, Hq, Hkv, Nq, Nk, d, seed)
        scale = 1.0 / math.sqrt(d)
        O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal)
        Ob, Lb = brute_force_decimal(x, scale, causal)
        assert_close(O, Ob, what=f"O brute {B,Hq,Hkv,Nq,Nk,d,causal}")
        assert_close(L, Lb, what=f"LSE brute {B,Hq,Hkv,Nq,Nk,d,causal}")


def pin_large_logits(orc):
    """Q x 8 (exact in bf16): logits of size ~8-30; must neither overflow nor drift."""
    x = tiny_inputs(1, 2, 1, 7, 9, 64, seed=11, q_mult=8.0)
    scale = 1.0 / 8.0
    for causal in (False, True):
        O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal)
        Ob, Lb = brute_force_decimal(x, scale, causal)
        assert np.isfinite(O).all()
        assert_close(O, Ob, what="O qx8")
        assert_close(L, Lb, what="LSE qx8")


def pin_probs_rows_sum_to_one(orc):
    x = tiny_inputs(1, 2, 2, 9, 12, 32, seed=12)
    for causal in (False, True):
        _, _, P = orc.probs(x["q"], x["k"], x["v"], 0.3, causal)
        assert (P >= 0).all()
        assert np.abs(P.sum(axis=-1) - 1.0).max() < TOL
        if causal:
            i = np.arange(9)[:, None]
            j = np.arange(12)[None, :]
            hidden = j > i + 3          # Nk - Nq = 3
            assert (P[..., hidden] == 0).all()


def pin_one_key(orc):
    """Nk = 1: every row attends to its single key: O = v_0, LSE = scale * q . k_0."""
    x = tiny_inputs(2, 4, 2, 5, 1, 64, seed=13)
    scale = 0.125
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, False)
    q, k, v = (bits_f64(x[n]) for n in ("q", "k", "v"))
    for b in range(2):
        for h in range(4):
            g = h // 2
            assert_close(O[b, :, h, :], np.broadcast_to(v[b, 0, g, :], (5, 64)), what="O one key")
            assert_close(L[b, h, :], scale * (q[b, :, h, :] @ k[b, 0, g, :]), what="LSE one key")


def pin_constant_v(orc):
    """Every key carries the same value row -> every output row equals it."""
    x = tiny_inputs(1, 2, 2, 8, 10, 32, seed=14)
    v = x["v"].copy()
    v[:] = v[:, :1]
    for causal in (False, True):
        O, _ = orc.forward(x["q"], x["k"], v, 0.2, causal)
        vf = bits_f64(v)
        for h in range(2):
            assert_close(O[0, :, h, :], np.broadcast_to(vf[0, 0, h, :], (8, 32)), what="O const V")


def pin_zero_q(orc):
    """Q = 0: all logits equal -> O = mean of the visible V rows, LSE = ln(#visible)."""
    x = tiny_inputs(1, 2, 1, 6, 6, 32, seed=15)
    q = np.zeros_like(x["q"])
    vf = bits_f64(x["v"])
    for causal in (False, True):
        O, L = orc.forward(q, x["k"], x["v"], 0.5, causal)
        for i in range(6):
            n = i + 1 if causal else 6
            for h in range(2):
                assert_close(O[0, i, h, :], vf[0, :n, 0, :].mean(axis=0), what="O zero Q")
                assert_close(L[0, h, i], math.log(n), what="LSE zero Q")


def pin_causal_row0(orc):
    """Causal, Nq = Nk: row 0 sees only key 0 -> O_0 = v_0, LSE_0 = s_00."""
    x = tiny_inputs(1, 2, 2, 7, 7, 64, seed=16)
    scale = 0.125
    O, L = orc.forward(x["q"], x["k"], x["v"], scale, True)
    q, k, v = (bits_f64(x[n]) for n in ("q", "k", "v"))
    for h in range(2):
        assert_close(O[0, 0, h, :], v[0, 0, h, :], what="O causal row 0")
        assert_close(L[0, h, 0], scale * float(q[0, 0, h, :] @ k[0, 0, h, :]), what="LSE causal row 0")


def pin_gqa_equals_repeated_mha(orc):
    """GQA result == MHA with K/V repeated n_rep times per head (repeat_interleave)."""
    x = tiny_inputs(2, 8, 2, 6, 9, 32, seed=17)
    kr = np.repeat(x["k"], 4, axis=2)
    vr = np.repeat(x["v"], 4, axis=2)
    for causal in (False, True):
        O1, L1 = orc.forward(x["q"], x["k"], x["v"], 0.3, causal)
        O2, L2 = orc.forward(x["q"], kr, vr, 0.3, causal)
        assert_close(O1, O2, what="GQA vs MHA O")
        assert_close(L1, L2, what="GQA vs MHA LSE")


def pin_key_permutation(orc):
    """Without a mask the result does not depend on the order of the (key, value) pairs."""
    x = tiny_inputs(1, 2, 2, 5, 11, 32, seed=18)
    perm = np.random.default_rng(0).permutation(11)
    O1, L1 = orc.forward(x["q"], x["k"], x["v"], 0.3, False)
    O2, L2 = orc.forward(x["q"], x["k"][:, perm], x["v"][:, perm], 0.3, False)
    assert_close(O1, O2, what="perm O")
    assert_close(L1, L2, what="perm LSE")


def pin_causal_prefix(orc):
    """Causal row i equals unmasked attention of query i over keys 0..i."""
    x = tiny_inputs(1, 1, 1, 9, 9, 32, seed=19)
    O, L = orc.forward(x["q"], x["k"], x["v"], 0.3, True)
    for i in (0, 3, 8):
        Oi, Li = orc.forward(x["q"][:, i:i + 1], x["k"][:, :i + 1], x["v"][:, :i + 1], 0.3, False)
        assert_close(O[0, i, 0], Oi[0, 0, 0], what="prefix O")
        assert_close(L[0, 0, i], Li[0, 0, 0], what="prefix LSE")


def pin_online_recurrence(orc):
    """The block-wise online-softmax recurrence reaches the oracle's result at every block size."""
    for (B, Hq, Hkv, Nq, Nk, d, causal) in [(1, 2, 1, 37, 37, 32, True), (2, 2, 2, 20, 45, 64, False),
                                             (1, 2, 2, 30, 17, 16, True)]:
        x = tiny_inputs(B, Hq, Hkv, Nq, Nk, d, seed=20 + Nq)
        O, L = orc.forward(x["q"], x["k"], x["v"], 0.2, causal)
        for block in (1, 5, 16, 64, 128):
            Ob, Lb = online_softmax_blocks(x, 0.2, causal, block)
            assert_close(O, Ob, what=f"online O block {block}")
            assert_close(L, Lb, what=f"online LSE block {block}")


def pin_rows_match_full(orc):
    """The selected-rows entry point gives the full forward's rows."""
    x = tiny_inputs(2, 4, 2, 13, 10, 32, seed=21)
    rows = [(0, 0, 0), (1, 3, 12), (0, 2, 5), (1, 1, 2)]
    for causal in (False, True):
        O, L = orc.forward(x["q"], x["k"], x["v"], 0.3, causal)
        Or, Lr = orc.rows(x["q"], x["k"], x["v"], rows, 0.3, causal)
        for r, (b, h, i) in enumerate(rows):
            assert np.array_equal(Or[r], O[b, i, h])
            assert Lr[r] == L[b, h, i] or (np.isinf(Lr[r]) and np.isinf(L[b, h, i]))


ALL_PINS = [
    pin_brute_force, pin_large_logits, pin_probs_rows_sum_to_one, pin_one_key, pin_constant_v,
    pin_zero_q, pin_causal_row0, pin_gqa_equals_repeated_mha, pin_key_permutation,
    pin_causal_prefix, pin_online_recurrence, pin_rows_match_full,
]


# ---------------------------------------------------------------- sliding window

WINDOW_CASES = [
    # B, Hq, Hkv, Nq, Nk, d, window, seed
    (1, 2, 1, 9, 9, 32, 3, 40),
    (1, 2, 2, 6, 11, 64, 4, 41),      # Nq < Nk
    (1, 1, 1, 10, 4, 16, 2, 42),      # Nq > Nk: early rows see nothing
    (2, 4, 2, 7, 7, 80, 1, 43),
]


def pin_window_brute_force(orc):
    for (B, Hq, Hkv, Nq, Nk, d, W, seed) in WINDOW_CASES:
        x = tiny_inputs(B, Hq, Hkv, Nq, Nk, d, seed)
        scale = 1.0 / math.sqrt(d)
        O, L = orc.forward(x["q"], x["k"], x["v"], scale, True, window=W)
        Ob, Lb = brute_force_decimal(x, scale, True, window=W)
        assert_close(O, Ob, what=f"window O {W}")
        assert_close(L, Lb, what=f"window LSE {W}")


def pin_window_one_key(orc):
    """W = 1: row i sees only key i + Nk - Nq: O = v, LSE = that single logit."""
    x = tiny_inputs(1, 2, 2, 6, 8, 32, seed=44)
    O, L = orc.forward(x["q"], x["k"], x["v"], 0.25, True, window=1)
    q, k, v = (bits_f64(x[n]) for n in ("q", "k", "v"))
    for i in range(6):
        j = i + 2
        for h in range(2):
            assert_close(O[0, i, h], v[0, j, h], what="W=1 O")
            assert_close(L[0, h, i], 0.25 * float(q[0, i, h] @ k[0, j, h]), what="W=1 LSE")


def pin_window_wide_is_causal(orc):
    x = tiny_inputs(1, 2, 1, 12, 12, 32, seed=45)
    Oc, Lc = orc.forward(x["q"], x["k"], x["v"], 0.2, True)
    Ow, Lw = orc.forward(x["q"], x["k"], x["v"], 0.2, True, window=12)
    assert np.array_equal(Oc, Ow) and np.array_equal(Lc, Lw)


def pin_window_row_is_segment(orc):
    """Row i with window W equals unmasked attention of query i over keys i-W+1 .. i."""
    x = tiny_inputs(1, 1, 1, 10, 10, 32, seed=46)
    W = 4
    O, L = orc.forward(x["q"], x["k"], x["v"], 0.3, True, window=W)
    for i in (0, 2, 7, 9):
        lo = max(0, i - W + 1)
        Oi, Li = orc.forward(x["q"][:, i:i + 1], x["k"][:, lo:i + 1], x["v"][:, lo:i + 1], 0.3, False)
        assert_close(O[0, i, 0], Oi[0, 0, 0], what="segment O")
        assert_close(L[0, 0, i], Li[0, 0, 0], what="segment LSE")


def pin_window_online_recurrence(orc):
    x = tiny_inputs(1, 2, 1, 40, 40, 32, seed=47)
    O, L = orc.forward(x["q"], x["k"], x["v"], 0.2, True, window=13)
    for block in (1, 7, 16, 64):
        Ob, Lb = online_softmax_blocks(x, 0.2, True, block, window=13)
        assert_close(O, Ob, what="window online O")
        assert_close(L, Lb, what="window online LSE")


WINDOW_PINS = [pin_window_brute_force, pin_window_one_key, pin_window_wide_is_causal,
               pin_window_row_is_segment, pin_window_online_recurrence]
ALL_PINS = ALL_PINS + WINDOW_PINS


# ---------------------------------------------------------------- fp16 inputs

def pin_f16_decode_every_pattern(orc):
    """One key: O = v exactly, so every finite IEEE half pattern placed in v must come back
    as numpy's float16 value (normals, subnormals, both zeros, both signs)."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    pats = pats[((pats >> 10) & 0x1F) != 0x1F]            # drop inf / NaN
    d = pats.size
    z = np.zeros((1, 1, 1, d), np.uint16)
    O, L = orc.forward(z, z, pats.reshape(1, 1, 1, d), 1.0, False, dtype="f16")
    assert np.array_equal(O[0, 0, 0], pats.view(np.float16).astype(np.float64)), "fp16 decode"
    assert L[0, 0, 0] == 0.0


def pin_f16_known_values(orc):
    """IEEE binary16 values fixed by the format: 1, -2, the largest finite 65504, the
    smallest normal 2^-14, the smallest subnormal 2^-24, and 1/3 rounded (1365/4096)."""
    table = {0x3C00: 1.0, 0xC000: -2.0, 0x7BFF: 65504.0, 0x0400: 2.0 ** -14, 0x0001: 2.0 ** -24,
             0x3555: 1365 / 4096, 0x8000: -0.0}
    v = np.array(list(table), dtype=np.uint16).reshape(1, 1, 1, -1)
    z = np.zeros_like(v)
    O, _ = orc.forward(z, z, v, 1.0, False, dtype="f16")
    assert list(O[0, 0, 0]) == list(table.values()), O[0, 0, 0]


def pin_f16_brute_force(orc):
    for (B, Hq, Hkv, Nq, Nk, d, causal, seed) in [(1, 2, 1, 5, 7, 32, False, 60), (1, 4, 2, 6, 4, 64, True, 61)]:
        x = tiny_inputs(B, Hq, Hkv, Nq, Nk, d, seed, q_mult=8.0, dtype="f16")
        scale = 1.0 / math.sqrt(d)
        O, L = orc.forward(x["q"], x["k"], x["v"], scale, causal, dtype="f16")
        Ob, Lb = brute_force_decimal(x, scale, causal, dtype="f16")
        assert_close(O, Ob, what="f16 O brute")
        assert_close(L, Lb, what="f16 LSE brute")


F16_PINS = [pin_f16_decode_every_pattern, pin_f16_known_values, pin_f16_brute_force]
ALL_PINS = ALL_PINS + F16_PINS


# ---------------------------------------------------------------- backward pass

def _dec(a):
    return np.array([Decimal(float(t)) for t in np.asarray(a, dtype=np.float64).ravel()], dtype=object).reshape(np.shape(a))


def decimal_loss(q, k, v, do, scale, causal, window=0):
    """L = sum O (.) dO by the definition, in Decimal arithmetic (object arrays)."""
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    rep = Hq // Hkv
    sc = Decimal(float(scale))
    total = Decimal(0)
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            for i in range(Nq):
                es = []
                for j in range(Nk):
                    if visible(i, j, Nq, Nk, causal, window):
                        es.append((j, (sc * sum(q[b, i, h, c] * k[b, j, g, c] for c in range(d))).exp()))
                Z = sum(e for _, e in es)
                if not es:
                    continue
                for c in range(d):
                    total += sum(e * v[b, j, g, c] for j, e in es) / Z * do[b, i, h, c]
    return total


def finite_difference_grads(x, do_bits, scale, causal, window=0, h="1e-15"):
    """Central differences of decimal_loss with respect to every element of q, k, v."""
    getcontext().prec = 60
    arrs = {n: _dec(bits_f64(x[n])) for n in ("q", "k", "v")}
    do = _dec(bits_f64(do_bits))
    hh = Decimal(h)
    grads = {}
    for name in ("q", "k", "v"):
        a = arrs[name]
        g = np.zeros(a.shape)
        for idx in np.ndindex(a.shape):
            x0 = a[idx]
            a[idx] = x0 + hh
            lp = decimal_loss(arrs["q"], arrs["k"], arrs["v"], do, scale, causal, window)
            a[idx] = x0 - hh
            lm = decimal_loss(arrs["q"], arrs["k"], arrs["v"], do, scale, causal, window)
            a[idx] = x0
            g[idx] = float((lp - lm) / (2 * hh))
        grads[name] = g
    return grads["q"], grads["k"], grads["v"]


def _bwd_inputs(B, Hq, Hkv, Nq, Nk, d, seed, dtype="bf16"):
    w = synth.Workload("tinybwd", 2000 + seed, B, Hq, Hkv, Nq, Nk, d, False, seed=seed, dtype=dtype)
    return synth.make_inputs(w), synth.make_grad_output(w)


BWD_FD_CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, seed
    (1, 2, 1, 3, 4, 3, False, 0, 70),
    (1, 2, 2, 4, 3, 2, True, 0, 71),     # Nq > Nk: row 0 sees no key
    (1, 1, 1, 5, 5, 2, True, 2, 72),     # sliding window
]


def pin_bwd_finite_difference(orc):
    """The oracle's dQ, dK, dV equal central differences of the loss sum O (.) dO taken in
    60-digit decimal arithmetic straight from the forward definition."""
    for (B, Hq, Hkv, Nq, Nk, d, causal, W, seed) in BWD_FD_CASES:
        x, do = _bwd_inputs(B, Hq, Hkv, Nq, Nk, d, seed)
        scale = 0.7
        dq, dk, dv = orc.backward(x["q"], x["k"], x["v"], do, scale, causal, window=W)
        fq, fk, fv = finite_difference_grads(x, do, scale, causal, window=W)
        assert_close(dq, fq, tol=1e-9, what=f"dQ fd {seed}")
        assert_close(dk, fk, tol=1e-9, what=f"dK fd {seed}")
        assert_close(dv, fv, tol=1e-9, what=f"dV fd {seed}")


def pin_bwd_one_key(orc):
    """Nk = 1: P = 1 for every row, so dS = 0 (dQ = dK = 0) and dV = sum of dO over the
    rows and query heads of the group."""
    x, do = _bwd_inputs(2, 4, 2, 5, 1, 16, seed=73)
    dq, dk, dv = orc.backward(x["q"], x["k"], x["v"], do, 0.25, False)
    assert np.abs(dq).max() < TOL and np.abs(dk).max() < TOL
    dof = bits_f64(do)
    for b in range(2):
        for g in range(2):
            assert_close(dv[b, 0, g], dof[b, :, 2 * g:2 * g + 2].sum(axis=(0, 1)), what="dV one key")


def pin_bwd_dk_sums_to_zero(orc):
    """Each softmax row is invariant to adding one vector to every key, so the key
    gradients of a head sum to zero (sum_j dS_ij = 0 per row)."""
    for causal in (False, True):
        x, do = _bwd_inputs(1, 4, 2, 7, 9, 16, seed=74)
        _, dk, _ = orc.backward(x["q"], x["k"], x["v"], do, 0.3, causal)
        assert np.abs(dk.sum(axis=1)).max() < 1e-12 * max(1.0, np.abs(dk).max() * 9)


def pin_bwd_gqa_is_summed_mha(orc):
    """GQA gradients: dQ equals MHA with K, V repeated per query head; dK, dV of a KV head
    are the sums over its query heads of the MHA ones."""
    x, do = _bwd_inputs(1, 6, 2, 5, 7, 8, seed=75)
    dq, dk, dv = orc.backward(x["q"], x["k"], x["v"], do, 0.4, True)
    kr = np.repeat(x["k"], 3, axis=2)
    vr = np.repeat(x["v"], 3, axis=2)
    dq2, dk2, dv2 = orc.backward(x["q"], kr, vr, do, 0.4, True)
    assert_close(dq, dq2, what="GQA dQ")
    assert_close(dk, dk2.reshape(1, 7, 2, 3, 8).sum(axis=3), what="GQA dK")
    assert_close(dv, dv2.reshape(1, 7, 2, 3, 8).sum(axis=3), what="GQA dV")


def pin_bwd_causal_first_row(orc):
    """Causal, Nq = Nk: row 0 sees only key 0, so its dQ is zero; the last key is seen
    only by the last row, so its dV is P_last,last * dO_last."""
    x, do = _bwd_inputs(1, 1, 1, 6, 6, 8, seed=76)
    dq, dk, dv = orc.backward(x["q"], x["k"], x["v"], do, 0.5, True)
    assert np.abs(dq[0, 0, 0]).max() < TOL
    _, _, P = orc.probs(x["q"], x["k"], x["v"], 0.5, True)
    assert_close(dv[0, 5, 0], P[0, 0, 5, 5] * bits_f64(do)[0, 5, 0], what="last key dV")


BWD_PINS = [pin_bwd_finite_difference, pin_bwd_one_key, pin_bwd_dk_sums_to_zero, pin_bwd_gqa_is_summed_mha,
            pin_bwd_causal_first_row]
ALL_PINS = ALL_PINS + BWD_PINS


# ---------------------------------------------------------------- FP8 (E4M3) inputs

def _fp8_inputs(B, Hq, Hkv, Nq, Nk, d, seed, q_mult=1.0):
    w = synth.Workload("tinyfp8", 4000 + seed, B, Hq, Hkv, Nq, Nk, d, False, q_mult=q_mult, seed=seed, dtype="e4m3")
    return synth.make_inputs(w)


def pin_e4m3_decode_every_pattern(orc):
    """One key: O = dv * v8 exactly, so every non-NaN E4M3 byte placed in v comes back as
    torch's float8_e4m3fn value (normals, subnormals, both zeros, both signs)."""
    pats = np.arange(256, dtype=np.uint8)
    pats = pats[(pats & 0x7F) != 0x7F]
    z = np.zeros((1, 1, 1, pats.size), np.uint8)
    O, L = orc.forward_fp8(z, z, pats.reshape(1, 1, 1, -1), 1.0, False)
    assert np.array_equal(O[0, 0, 0], e4m3_f64(pats)), "e4m3 decode"
    O2, _ = orc.forward_fp8(z, z, pats.reshape(1, 1, 1, -1), 1.0, False, descale=(1.0, 1.0, 0.375))
    assert np.array_equal(O2[0, 0, 0], 0.375 * e4m3_f64(pats)), "dv applied to V"
    assert L[0, 0, 0] == 0.0


def pin_e4m3_known_values(orc):
    """E4M3 values fixed by the format: 1, -1, the largest finite 448, the smallest normal
    2^-6, the smallest subnormal 2^-9, 1.125 (one fraction step above 1)."""
    table = {0x38: 1.0, 0xB8: -1.0, 0x7E: 448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0x39: 1.125}
    v = np.array(list(table), dtype=np.uint8).reshape(1, 1, 1, -1)
    z = np.zeros_like(v)
    O, _ = orc.forward_fp8(z, z, v, 1.0, False)
    assert list(O[0, 0, 0]) == list(table.values()), O[0, 0, 0]


def pin_fp8_brute_force_with_descales(orc):
    """Decimal brute force on Q = dq q8, K = dk k8, V = dv v8 (torch-decoded bytes)."""
    for (B, Hq, Hkv, Nq, Nk, d, causal, seed, ds) in [(1, 2, 1, 5, 6, 32, False, 80, (0.5, 2.0, 0.25)),
                                                       (1, 2, 2, 6, 4, 16, True, 81, (0.125, 1.0, 3.0))]:
        x = _fp8_inputs(B, Hq, Hkv, Nq, Nk, d, seed, q_mult=4.0)
        scale = 1.0 / math.sqrt(d)
        O, L = orc.forward_fp8(x["q"], x["k"], x["v"], scale, causal, descale=ds)
        qf, kf, vf = (c * e4m3_f64(x[n]) for c, n in zip(ds, ("q", "k", "v")))
        Ob, Lb = brute_force_values(qf, kf, vf, scale, causal)
        assert_close(O, Ob, what="fp8 O brute")
        assert_close(L, Lb, what="fp8 LSE brute")


def pin_fp8_rows_match_full(orc):
    x = _fp8_inputs(2, 4, 2, 9, 13, 32, seed=82)
    O, L = orc.forward_fp8(x["q"], x["k"], x["v"], 0.2, True, descale=(0.5, 0.5, 2.0))
    rows = np.array([(0, 0, 0), (1, 3, 8), (0, 2, 4), (1, 1, 2)], dtype=np.int32)
    Or, Lr = orc.rows_fp8(x["q"], x["k"], x["v"], rows, 0.2, True, descale=(0.5, 0.5, 2.0))
    for n, (b, h, i) in enumerate(rows):
        assert np.array_equal(Or[n], O[b, i, h]) and Lr[n] == L[b, h, i]


FP8_PINS = [pin_e4m3_decode_every_pattern, pin_e4m3_known_values, pin_fp8_brute_force_with_descales,
            pin_fp8_rows_match_full]
ALL_PINS = ALL_PINS + FP8_PINS

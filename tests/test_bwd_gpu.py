"""Backward pass (fa_bwd) against the CPU oracle's gradients of sum(O * dO).

Acceptance, per gradient tensor G against the fp64 oracle (derived from the arithmetic:
P, dS, the forward's O (through D) and the outputs are each rounded to bf16 once, unit
roundoff u = 2^-9 ~ 2e-3, so the relative L2 error stays within ~4u):
    ||dG||_2 / ||G||_2 <= 1e-2,    max |dG| <= 2e-2 * max |G|."""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import _parity

pytestmark = pytest.mark.gpu

TOL_BWD_REL_L2 = 1e-2
TOL_BWD_MAX_REL = 2e-2
# A gradient that is exactly zero by definition (one key: dQ = dK = 0) must stay below 1e-3
# of the largest gradient of the problem.


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


def inputs(B, Hq, Hkv, Nq, Nk, d, seed, **kw):
    w = synth.Workload("bwd", 3000 + seed, B, Hq, Hkv, Nq, Nk, d, False, seed=seed, **kw)
    return synth.make_inputs(w), synth.make_grad_output(w)


def run_bwd(x, do_bits, scale, causal, dtype="bf16"):
    """Forward (for O and LSE) then fa_bwd (fa_bwd_f16), both through the C ABI."""
    import torch
    import exact_attention_146_b200 as fa
    q, k, v = (_parity.to_device(x[n], torch, dtype) for n in ("q", "k", "v"))
    do = _parity.to_device(do_bits, torch, dtype)
    out, lse = fa.fa_fwd(q, k, v, causal=causal, scale=scale)
    dq = torch.full_like(q, float("nan"))
    dk = torch.full_like(k, float("nan"))
    dv = torch.full_like(v, float("nan"))
    fa.fa_bwd(q, k, v, out, do, lse, causal=causal, scale=scale, dq=dq, dk=dk, dv=dv)
    st, word = fa.device_status()
    assert st == fa.FA_OK, f"device status {st} (word {word:#x})"
    torch.cuda.synchronize()
    return tuple(_parity.bf16_to_f64(t) for t in (dq, dk, dv))


def compare_grads(got, ref, what):
    scale_all = max(float(np.abs(r).max()) if r.size else 0.0 for r in ref)
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        assert g.shape == r.shape, (name, g.shape, r.shape)
        assert np.isfinite(g).all(), f"{what} {name}: non-finite (unwritten rows?)"
        if r.size and not np.abs(r).max() > 0:
            # exactly zero in the definition (e.g. one key: dQ = dK = 0); only rounding
            # terms remain (D from the bf16 O), far below the problem's gradient scale
            assert float(np.abs(g).max()) <= 1e-3 * scale_all, f"{what} {name}: {np.abs(g).max():.3e} vs 0"
            continue
        nrm = float(np.linalg.norm(r))
        err = g - r
        rel = float(np.linalg.norm(err) / nrm) if nrm > 0 else float(np.linalg.norm(g))
        mx = float(np.abs(err).max()) if err.size else 0.0
        ref_max = float(np.abs(r).max()) if r.size else 0.0
        assert rel <= TOL_BWD_REL_L2 or nrm == 0, f"{what} {name}: rel L2 {rel:.3e}"
        assert mx <= TOL_BWD_MAX_REL * max(ref_max, 1e-6), f"{what} {name}: max|d| {mx:.3e} (ref max {ref_max:.3e})"


@pytest.mark.parametrize("d", [32, 64, 80, 96, 128])
@pytest.mark.parametrize("Nq,Nk", [(1, 1), (17, 17), (128, 128), (129, 300), (300, 129), (256, 256)])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_small(orc, d, Nq, Nk, causal):
    x, do = inputs(1, 2, 1, Nq, Nk, d, seed=Nq * 7 + Nk + d)
    scale = 1.0 / math.sqrt(d)
    got = run_bwd(x, do, scale, causal)
    ref = orc.backward(x["q"], x["k"], x["v"], do, scale, causal)
    compare_grads(got, ref, f"d={d} Nq={Nq} Nk={Nk} causal={causal}")


@pytest.mark.parametrize("case", [(2, 4, 2, 200, 333, 128, True), (2, 8, 2, 130, 130, 64, False),
                                  (1, 8, 1, 64, 500, 128, False), (1, 4, 4, 390, 390, 64, True)])
def test_bwd_gqa_batches(orc, case):
    B, Hq, Hkv, Nq, Nk, d, causal = case
    x, do = inputs(B, Hq, Hkv, Nq, Nk, d, seed=sum(case[:6]))
    scale = 1.0 / math.sqrt(d)
    got = run_bwd(x, do, scale, causal)
    ref = orc.backward(x["q"], x["k"], x["v"], do, scale, causal)
    compare_grads(got, ref, f"{case}")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_medium(orc, causal):
    """Several key tiles and query tiles per head, large logits (Q x 8)."""
    x, do = inputs(1, 2, 2, 1024, 1024, 128, seed=5, q_mult=8.0)
    scale = 1.0 / math.sqrt(128)
    got = run_bwd(x, do, scale, causal)
    ref = orc.backward(x["q"], x["k"], x["v"], do, scale, causal)
    compare_grads(got, ref, f"medium causal={causal}")


@pytest.mark.parametrize("d", [32, 80, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_f16(orc, d, causal):
    """fp16 inputs and gradients (fa_bwd_f16) against the oracle reading the same half bits."""
    x, do = inputs(2, 4, 2, 200, 333, d, seed=d + 17, dtype="f16")
    scale = 1.0 / math.sqrt(d)
    got = run_bwd(x, do, scale, causal, dtype="f16")
    ref = orc.backward(x["q"], x["k"], x["v"], do, scale, causal, dtype="f16")
    compare_grads(got, ref, f"f16 d={d} causal={causal}")


@pytest.mark.parametrize("W", [1, 100, 300, 5000])
@pytest.mark.parametrize("shape", [(1, 4, 2, 600, 600, 128), (1, 2, 1, 300, 700, 64), (1, 2, 2, 500, 260, 96)])
def test_bwd_window(orc, W, shape):
    """Sliding-window backward (fa_bwd_window) after fa_fwd_window, against the oracle's
    gradients with the same window (query tiles outside a key tile's band are skipped)."""
    import torch
    import exact_attention_146_b200 as fa
    B, Hq, Hkv, Nq, Nk, d = shape
    x, do_bits = inputs(B, Hq, Hkv, Nq, Nk, d, seed=W + Nq)
    scale = 1.0 / math.sqrt(d)
    q, k, v = (_parity.to_device(x[n], torch) for n in ("q", "k", "v"))
    do = _parity.to_device(do_bits, torch)
    out, lse = fa.fa_fwd(q, k, v, causal=True, scale=scale, window=W)
    dq, dk, dv = fa.fa_bwd(q, k, v, out, do, lse, causal=True, scale=scale, window=W,
                           dq=torch.full_like(q, float("nan")), dk=torch.full_like(k, float("nan")),
                           dv=torch.full_like(v, float("nan")))
    st, word = fa.device_status()
    assert st == fa.FA_OK, f"device status {st} ({word:#x})"
    torch.cuda.synchronize()
    got = tuple(_parity.bf16_to_f64(t) for t in (dq, dk, dv))
    ref = orc.backward(x["q"], x["k"], x["v"], do_bits, scale, True, window=W)
    compare_grads(got, ref, f"window W={W} {shape}")


def test_bwd_empty_sides():
    """Nq = 0: dK = dV = 0; Nk = 0: dQ = 0."""
    import torch
    import exact_attention_146_b200 as fa
    q = torch.randn(1, 0, 2, 64, device="cuda").bfloat16()
    k = torch.randn(1, 5, 2, 64, device="cuda").bfloat16()
    out = torch.empty_like(q)
    lse = torch.empty(1, 2, 0, device="cuda")
    dq, dk, dv = fa.fa_bwd(q, k, k.clone(), out, q.clone(), lse, dk=torch.full_like(k, 7.0),
                           dv=torch.full_like(k, 7.0))
    torch.cuda.synchronize()
    assert (dk == 0).all() and (dv == 0).all()
    q2 = torch.randn(1, 3, 2, 64, device="cuda").bfloat16()
    k2 = torch.randn(1, 0, 2, 64, device="cuda").bfloat16()
    lse2 = torch.full((1, 2, 3), float("-inf"), device="cuda")
    dq2, _, _ = fa.fa_bwd(q2, k2, k2.clone(), torch.zeros_like(q2), q2.clone(), lse2, dq=torch.full_like(q2, 7.0))
    torch.cuda.synchronize()
    assert (dq2 == 0).all()

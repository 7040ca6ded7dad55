"""The forward kernel's failure path on the GPU, made to run without faulting anything: the
failure-path test build (fa_test_withheld_load) leaves one K/V tile load out, so the wait
for it runs out after a short limit.  The kernel must then record FA_ERR_DEVICE_TIMEOUT with
the site of the wait that gave up, unwind every role (the producer waits for its copies in
flight, the MMA thread for its MMAs, TMEM is freed) and return; the context stays usable, so
the next ordinary call passes the oracle parity check."""
import time

import numpy as np
import pytest

import oracle
import synth
from tests import _parity

pytestmark = pytest.mark.gpu

SITE_KV_FULL = 3      # the MMA thread's wait for a K/V tile
SITE_S_FULL = 7       # a softmax warp's wait for its score tile
SITE_KV_EMPTY = 2     # the producer's wait for a slot to come back


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


def device_inputs(B, H, N, seed):
    import torch
    w = synth.Workload("failpath", 9100 + seed, B, H, H, N, N, 64, False, seed=seed)
    x = synth.make_inputs(w)
    return x, [_parity.to_device(x[n], torch) for n in ("q", "k", "v")]


def withheld_run(qkv, load, limit_us):
    import exact_attention_146_b200 as fa
    import torch
    q, k, v = qkv
    fa.device_status()                       # start from a clear status word
    t0 = time.perf_counter()
    fa.withheld_load_forward(q, k, v, load, limit_us)
    st, word = fa.device_status()            # synchronises the stream
    torch.cuda.synchronize()
    return st, word, time.perf_counter() - t0


@pytest.mark.parametrize("case", [(1, 1, 256, 1), (1, 2, 2048, 5)])
def test_withheld_load_times_out_then_recovers(orc, case):
    """(B, H, N, withheld load): one CTA whose MMA thread waits for V_0; sixteen CTAs, each
    missing V_2 while its producer also blocks on a slot that never comes back."""
    import exact_attention_146_b200 as fa
    B, H, N, load = case
    x, qkv = device_inputs(B, H, N, seed=N)
    st, word, secs = withheld_run(qkv, load, 20000)
    site, cta = (word >> 8) & 0xFF, word >> 16
    print(f"withheld load {load}: status {st}, word {word:#x} (site {site}, cta {cta}), {secs * 1e3:.1f} ms")
    assert st == fa.FA_ERR_DEVICE_TIMEOUT, (st, hex(word))
    assert site in (SITE_KV_FULL, SITE_S_FULL, SITE_KV_EMPTY), hex(word)
    assert cta < 148 and (B * H * N // 256 > 1 or cta == 0), hex(word)
    assert secs < 5.0, secs                  # bounded: the limit is 20 ms per wait
    assert fa.device_status() == (fa.FA_OK, 0)   # reading the status cleared it
    # the context is intact: an ordinary forward right after passes parity
    O, L = _parity.run_cuda(x, 0.125, False)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 0.125, False)
    _parity.compare(O, L, Oref, Lref, f"after timeout {case}")


def test_withheld_load_past_the_end_is_an_ordinary_forward(orc):
    """With the withheld index beyond every CTA's last load, the test build computes the
    forward like fa_fwd (parity) and reports no timeout."""
    import exact_attention_146_b200 as fa
    import torch
    x, (q, k, v) = device_inputs(2, 2, 300, seed=3)
    out = torch.full_like(q, float("nan"))
    lse = torch.full((2, 2, 300), float("nan"), dtype=torch.float32, device="cuda")
    fa.device_status()
    fa.withheld_load_forward(q, k, v, 1 << 30, 1000000, causal=True, out=out, lse=lse)
    assert fa.device_status() == (fa.FA_OK, 0)
    Oref, Lref = orc.forward(x["q"], x["k"], x["v"], 0.125, True)
    _parity.compare(_parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64), Oref, Lref, "test build")

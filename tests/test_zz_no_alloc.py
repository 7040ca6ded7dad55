"""fa_fwd_splitkv_static: the split-KV forward with its partials in the library's static
device scratch (no allocation around the call), called through the C ABI and compared with
the entry points that take caller memory.  Collected last, so it also runs after every
other test has used the library on the same device."""
import ctypes
import math

import numpy as np
import pytest

import exact_attention_146_b200 as fa
from tests import _parity
from tests._pins import tiny_inputs


@pytest.fixture(scope="module", autouse=True)
def built_library():
    from exact_attention_146_b200 import build
    build.build()
    yield


def _call_static(q, k, v, out, lse, causal, scale, splits):
    import torch
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    return fa.lib().fa_fwd_splitkv_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                          lse.data_ptr(),
                                          B, Hq, Hkv, Nq, Nk, d, ctypes.c_float(scale), int(causal), splits,
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_scratch_limit_rejected_before_any_device_work():
    """Partials beyond the 16 MiB static scratch: FA_ERR_SCRATCH_LIMIT (host-only check)."""
    L = fa.lib()
    B, Hq, Nq, d, S = 8, 32, 64, 128, 8
    assert fa.splitkv_workspace_bytes(B, Hq, Nq, d, S) > fa.SPLITKV_STATIC_SCRATCH_BYTES
    fake = 1 << 40
    rc = L.fa_fwd_splitkv_static(fake, fake + (1 << 34), fake + (2 << 34), fake + (3 << 34), None,
                                 B, Hq, Hq, Nq, 4096, d, ctypes.c_float(0.088), 0, S, None)
    assert rc == fa.FA_ERR_SCRATCH_LIMIT
    assert "static scratch" in fa.status_string(rc)
    assert L.fa_fwd_splitkv_static(fake, fake, fake, fake, None, 1, 1, 1, 1, 1, 128,
                                   ctypes.c_float(0.1), 0, 0, None) == fa.FA_ERR_INVALID_ARG


@pytest.mark.gpu
def test_static_scratch_matches_caller_memory_two_calls():
    """Two calls in a row (different shapes, split counts and masks), each equal to the
    caller-workspace split-KV forward bit for bit and to the plain forward within the
    parity tolerance."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cases = [(2, 8, 2, 16, 3000, 128, False, 4, 11), (1, 4, 4, 130, 2049, 64, True, 3, 12)]
    for (B, Hq, Hkv, Nq, Nk, d, causal, S, seed) in cases:
        assert fa.splitkv_workspace_bytes(B, Hq, Nq, d, S) <= fa.SPLITKV_STATIC_SCRATCH_BYTES
        x = tiny_inputs(B, Hq, Hkv, Nq, Nk, d, seed=seed)
        q, k, v = (_parity.to_device(x[n], torch) for n in ("q", "k", "v"))
        scale = 1.0 / math.sqrt(d)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, Hq, Nq), float("nan"), dtype=torch.float32, device="cuda")
        rc = _call_static(q, k, v, out, lse, causal, scale, S)
        assert rc == fa.FA_OK, fa.status_string(rc)
        st, word = fa.device_status()
        assert st == fa.FA_OK, f"device status {st} (word {word:#x})"

        o_ws, l_ws = fa.fa_fwd(q, k, v, causal=causal, scale=scale, num_splits=S)
        o_plain, l_plain = fa.fa_fwd(q, k, v, causal=causal, scale=scale)
        torch.cuda.synchronize()
        assert torch.equal(out, o_ws) and torch.equal(lse, l_ws)
        O, Lv = _parity.bf16_to_f64(out), lse.cpu().numpy().astype(np.float64)
        _parity.compare(O, Lv, _parity.bf16_to_f64(o_plain), l_plain.cpu().numpy().astype(np.float64),
                        f"static scratch B={B} Hq={Hq} Nq={Nq} Nk={Nk} d={d} S={S}")

"""B200-native exact attention: Python binding of libfa.so.

Forward (fa_fwd: bf16 / fp16, causal or sliding window, split-KV; fa_fwd_fp8: E4M3),
key-shard partials and their merge (fa_fwd_partial, fa_merge_partials; see kshard for the
multi-GPU exchange) and the backward pass (fa_bwd).

This module only marshals arguments (torch tensors -> device pointers, sizes and the
current CUDA stream) into the C ABI declared in ``include/fa.h``; every step of the
computation runs in the CUDA kernels of ``csrc/``.  There is no fallback: if the
library is missing or the device is not sm_100 the calls raise.
"""
from __future__ import annotations

import ctypes
import math
from pathlib import Path

__all__ = ["fa_fwd", "fa_fwd_fp8", "fa_fwd_partial", "fa_merge_partials", "fa_bwd", "fa_fwd_raw",
           "splitkv_workspace_bytes", "splitkv_default_splits", "bwd_workspace_bytes", "device_status",
           "tile_config", "status_string", "FaError", "lib", "SUPPORTED_HEAD_DIMS", "BWD_HEAD_DIMS", "LIB_PATH",
           "withheld_load_forward"]

LIB_PATH = Path(__file__).resolve().parent / "libfa.so"
SUPPORTED_HEAD_DIMS = (32, 64, 80, 96, 128, 192, 256)   # forward
BWD_HEAD_DIMS = (32, 64, 80, 96, 128)                    # backward

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED_HEAD_DIM = 2
FA_ERR_MISALIGNED = 3
FA_ERR_UNSUPPORTED_DEVICE = 4
FA_ERR_CUDA = 5
FA_ERR_DEVICE_TIMEOUT = 6
FA_ERR_NOT_DEVICE_MEMORY = 7
FA_ERR_OVERLAP = 8
FA_ERR_SCRATCH_LIMIT = 9
SPLITKV_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024

EXPORTED = ("fa_fwd", "fa_fwd_window", "fa_fwd_splitkv", "fa_splitkv_workspace_bytes", "fa_splitkv_default_splits",
            "fa_fwd_splitkv_static", "fa_fwd_f16", "fa_fwd_fp8", "fa_fwd_partial", "fa_merge_partials", "fa_bwd", "fa_bwd_f16", "fa_bwd_window", "fa_bwd_workspace_bytes", "fa_status_string", "fa_device_status", "fa_tile_config", "fa_version",
            "fa_test_withheld_load", "fa_fwd_window_f16", "fa_fwd_splitkv_f16")


class FaError(RuntimeError):
    def __init__(self, code: int, what: str = "fa_fwd"):
        self.code = code
        super().__init__(f"{what}: status {code}: {status_string(code)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libfa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_attention_146_b200.build`")
        L = ctypes.CDLL(str(LIB_PATH))
        vp, ci, cf = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, vp]
        L.fa_fwd.restype = ci
        L.fa_fwd_f16.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, vp]
        L.fa_fwd_f16.restype = ci
        L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, cf, cf, cf, ci, vp]
        L.fa_fwd_fp8.restype = ci
        L.fa_fwd_partial.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, ci, vp]
        L.fa_fwd_partial.restype = ci
        L.fa_merge_partials.argtypes = [vp, vp, ci, vp, vp, ci, ci, ci, ci, vp]
        L.fa_merge_partials.restype = ci
        L.fa_fwd_window.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, vp]
        L.fa_fwd_window_f16.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, vp]
        L.fa_fwd_window_f16.restype = ci
        L.fa_fwd_splitkv_f16.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, vp, ctypes.c_size_t, vp]
        L.fa_fwd_splitkv_f16.restype = ci
        L.fa_fwd_window.restype = ci
        L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, vp, ctypes.c_size_t, vp]
        L.fa_fwd_splitkv.restype = ci
        L.fa_fwd_splitkv_static.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, vp]
        L.fa_fwd_splitkv_static.restype = ci
        L.fa_splitkv_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
        L.fa_splitkv_workspace_bytes.restype = ctypes.c_size_t
        L.fa_splitkv_default_splits.argtypes = [ci, ci, ci, ci, ci, ci, ci]
        L.fa_splitkv_default_splits.restype = ci
        L.fa_bwd.argtypes = [vp] * 9 + [ci] * 6 + [cf, ci, vp, ctypes.c_size_t, vp]
        L.fa_bwd.restype = ci
        L.fa_bwd_f16.argtypes = [vp] * 9 + [ci] * 6 + [cf, ci, vp, ctypes.c_size_t, vp]
        L.fa_bwd_f16.restype = ci
        L.fa_bwd_window.argtypes = [vp] * 9 + [ci] * 6 + [cf, ci, vp, ctypes.c_size_t, vp]
        L.fa_bwd_window.restype = ci
        L.fa_bwd_workspace_bytes.argtypes = [ci, ci, ci, ci]
        L.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.fa_status_string.argtypes = [ci]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_test_withheld_load.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, ci, ctypes.c_uint, vp]
        L.fa_test_withheld_load.restype = ci
        L.fa_device_status.argtypes = [vp, ctypes.POINTER(ci)]
        L.fa_device_status.restype = ci
        L.fa_tile_config.argtypes = [ci] + [ctypes.POINTER(ci)] * 4
        L.fa_tile_config.restype = ci
        L.fa_version.argtypes = []
        L.fa_version.restype = ci
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().fa_status_string(int(code)).decode()


def tile_config(d: int) -> dict:
    """Tiling fa_fwd uses for head dim d: block_q, block_k, q_tiles_per_unit, kv_slots."""
    vals = [ctypes.c_int(0) for _ in range(4)]
    rc = lib().fa_tile_config(int(d), *[ctypes.byref(x) for x in vals])
    if rc != FA_OK:
        raise FaError(rc, "fa_tile_config")
    return dict(zip(("block_q", "block_k", "q_tiles_per_unit", "kv_slots"), (x.value for x in vals)))


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def fa_fwd_raw(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream_ptr) -> int:
    """Direct C-ABI call with integer pointers; returns the status code."""
    return lib().fa_fwd(q_ptr, k_ptr, v_ptr, out_ptr, lse_ptr, int(B), int(Hq), int(Hkv), int(Nq), int(Nk),
                        int(d), float(scale), int(causal), stream_ptr)


def splitkv_workspace_bytes(B: int, Hq: int, Nq: int, d: int, num_splits: int) -> int:
    return int(lib().fa_splitkv_workspace_bytes(int(B), int(Hq), int(Nq), int(d), int(num_splits)))


def splitkv_default_splits(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, sm_count: int) -> int:
    return int(lib().fa_splitkv_default_splits(int(B), int(Hq), int(Hkv), int(Nq), int(Nk), int(d), int(sm_count)))


def fa_fwd(q, k, v, *, causal: bool = False, scale: float | None = None, out=None, lse=None,
           return_lse: bool = True, stream=None, window: int | None = None,
           num_splits: int | None = None, workspace=None):
    """Exact attention forward on [B, N, H, d] bf16 (or fp16: fa_fwd_f16) CUDA tensors.

    q: [B, Nq, Hq, d]; k, v: [B, Nk, Hkv, d] with Hq % Hkv == 0 (GQA: query head h
    uses KV head h // (Hq // Hkv)).  Returns (out [B, Nq, Hq, d] bf16, lse [B, Hq, Nq]
    fp32 natural-log log-sum-exp, or None if return_lse is False).  scale defaults to
    1/sqrt(d).  window = W (>= 1) selects the sliding-window mask: row i sees the W keys
    ending at its causal diagonal (fa_fwd_window).  num_splits = S (> 1) runs the
    split-KV forward (fa_fwd_splitkv) with `workspace` (a device tensor of at least
    splitkv_workspace_bytes; allocated here if None).  Runs asynchronously on `stream`
    (default: torch's current stream)."""
    import torch
    dt = q.dtype
    if dt not in (torch.bfloat16, torch.float16):
        raise ValueError(f"q must be bf16 or fp16, got {dt}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D {dt} CUDA tensor, got {t.dtype} {tuple(t.shape)}")
    if out is not None and out.dtype != dt:
        raise ValueError(f"out must be {dt}, got {out.dtype}")
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    if v.shape != k.shape or Bk != B or dk != d:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    lse_ptr = lse.data_ptr() if lse is not None else None
    f16 = dt == torch.float16
    if num_splits is not None and num_splits > 1:
        if window is not None:
            raise ValueError("split-KV takes the causal or no mask")
        need = splitkv_workspace_bytes(B, Hq, Nq, d, num_splits)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
        entry = lib().fa_fwd_splitkv_f16 if f16 else lib().fa_fwd_splitkv
        rc = entry(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                   B, Hq, Hkv, Nq, Nk, d, float(scale), 1 if causal else 0, int(num_splits),
                   workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    elif window is not None:
        entry = lib().fa_fwd_window_f16 if f16 else lib().fa_fwd_window
        rc = entry(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                   B, Hq, Hkv, Nq, Nk, d, float(scale), int(window), _stream_handle(stream))
    elif f16:
        rc = lib().fa_fwd_f16(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                              B, Hq, Hkv, Nq, Nk, d, float(scale), 1 if causal else 0, _stream_handle(stream))
    else:
        rc = fa_fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_ptr,
                        B, Hq, Hkv, Nq, Nk, d, scale, 1 if causal else 0, _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc)
    return out, lse


def fa_fwd_fp8(q8, k8, v8, *, descale=(1.0, 1.0, 1.0), causal: bool = False, scale: float | None = None, out=None,
               lse=None, return_lse: bool = True, stream=None):
    """FP8 forward (fa_fwd_fp8): q8, k8, v8 are [B, N, H, d] uint8 CUDA tensors of OCP E4M3
    bytes (or torch.float8_e4m3fn), dequantised by descale = (dq, dk, dv); out is bf16."""
    import torch
    ts = []
    for name, t in (("q", q8), ("k", k8), ("v", v8)):
        if t.dtype == torch.float8_e4m3fn:
            t = t.view(torch.uint8)
        if t.dtype != torch.uint8 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D E4M3 (uint8) CUDA tensor, got {t.dtype} {tuple(t.shape)}")
        ts.append(t)
    q8, k8, v8 = ts
    B, Nq, Hq, d = q8.shape
    Nk, Hkv = k8.shape[1], k8.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=q8.device)
    if return_lse and lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device)
    if not return_lse:
        lse = None
    rc = lib().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(),
                          lse.data_ptr() if lse is not None else None, B, Hq, Hkv, Nq, Nk, d, float(scale),
                          float(descale[0]), float(descale[1]), float(descale[2]), 1 if causal else 0,
                          _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_fp8")
    return out, lse


def fa_fwd_partial(q, k, v, *, key_offset: int, nk_total: int, causal: bool = False, scale: float | None = None,
                   o_part=None, lse_part=None, stream=None):
    """Partial forward over a key shard (fa_fwd_partial): q [B, Nq, Hq, d] bf16, k/v the
    shard [B, Nk, Hkv, d] bf16 holding global keys key_offset .. key_offset + Nk - 1 of
    nk_total.  Returns (o_part [B, Nq, Hq, d] fp32 normalised over the shard, lse_part
    [B, Hq, Nq] fp32)."""
    import torch
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o_part is None:
        o_part = torch.empty((B, Nq, Hq, d), dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = lib().fa_fwd_partial(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_part.data_ptr(), lse_part.data_ptr(),
                              B, Hq, Hkv, Nq, Nk, d, float(scale), 1 if causal else 0, int(key_offset),
                              int(nk_total), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_partial")
    return o_part, lse_part


def fa_merge_partials(o_parts, lse_parts, *, out=None, lse=None, stream=None):
    """Merge R stacked partials (fa_merge_partials): o_parts [R, B, Nq, Hq, d] fp32,
    lse_parts [R, B, Hq, Nq] fp32 -> (out [B, Nq, Hq, d] bf16, lse [B, Hq, Nq] fp32)."""
    import torch
    R, B, Nq, Hq, d = o_parts.shape
    if out is None:
        out = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=o_parts.device)
    rc = lib().fa_merge_partials(o_parts.data_ptr(), lse_parts.data_ptr(), R, out.data_ptr(), lse.data_ptr(),
                                 B, Hq, Nq, d, _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_merge_partials")
    return out, lse


def bwd_workspace_bytes(B: int, Hq: int, Nq: int, d: int) -> int:
    return int(lib().fa_bwd_workspace_bytes(int(B), int(Hq), int(Nq), int(d)))


def fa_bwd(q, k, v, out, dout, lse, *, causal: bool = False, scale: float | None = None, dq=None, dk=None,
           dv=None, workspace=None, stream=None, window: int | None = None):
    """Exact attention backward (fa_bwd, fa_bwd_f16 for fp16) on [B, N, H, d] CUDA tensors:
    returns (dq, dk, dv) for the loss sum(out * dout), given the forward's out and lse
    [B, Hq, Nq] fp32.  `workspace` (uint8, >= bwd_workspace_bytes) is allocated here if None."""
    import torch
    dt = q.dtype
    if dt not in (torch.bfloat16, torch.float16):
        raise ValueError(f"q must be bf16 or fp16, got {dt}")
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous 4-D {dt} CUDA tensor, got {t.dtype} {tuple(t.shape)}")
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Nq) or not lse.is_contiguous():
        raise ValueError(f"lse must be contiguous fp32 [B, Hq, Nq], got {lse.dtype} {tuple(lse.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(max(1, bwd_workspace_bytes(B, Hq, Nq, d)), dtype=torch.uint8, device=q.device)
    mask = 1 if causal else 0
    if window is not None:      # fa_bwd_window: the sliding window (bf16)
        if dt != torch.bfloat16:
            raise ValueError("the sliding-window backward takes bf16")
        entry, mask = lib().fa_bwd_window, int(window)
    else:
        entry = lib().fa_bwd_f16 if dt == torch.float16 else lib().fa_bwd
    rc = entry(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                      dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale),
                      mask, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                      _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_bwd")
    return dq, dk, dv


def withheld_load_forward(q, k, v, withheld_load: int, wait_limit_us: int, *, causal: bool = False,
                          scale: float | None = None, out=None, lse=None, stream=None):
    """Failure-path test (fa_test_withheld_load): the d = 64 bf16 forward in a build whose
    waits give up after wait_limit_us and whose producer leaves out K/V load number
    `withheld_load`; the timeout is then reported by device_status().  Outputs undefined."""
    import torch
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    rc = lib().fa_test_withheld_load(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                     B, Hq, Hkv, Nq, Nk, float(scale), 1 if causal else 0, int(withheld_load),
                                     int(wait_limit_us), _stream_handle(stream))
    if rc != FA_OK:
        raise FaError(rc, "fa_test_withheld_load")
    return out, lse


def device_status(stream=None) -> tuple[int, int]:
    """Synchronise `stream`, return (status, raw word) of the device status word, and clear it."""
    detail = ctypes.c_int(0)
    rc = lib().fa_device_status(_stream_handle(stream), ctypes.byref(detail))
    return rc, detail.value

"""CPU fp64 oracle for the exact attention forward -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(plus ``bench.py --impl reference``) may import this package.  The product path
(``exact_attention_146_b200``) never does, and this package never imports it.

The arithmetic lives in ``attention_oracle.c`` (plain C, IEEE fp64, the definition of
softmax(scale * Q K^T [+ causal mask]) V written out with S and P materialised);
this module only compiles it with gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "attention_oracle.c"
LIB_PATH = _HERE / "liboracle.so"

_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")


def build(out: Path | None = None, defines: tuple[str, ...] = ()) -> Path:
    """Compile the oracle with gcc (-O2, IEEE semantics: no fast-math).

    ``defines`` (e.g. ``("ORACLE_PLANT_NO_SCALE",)``) builds one of the deliberately
    wrong variants used by the mutation tests; those go to ``out``, never to the
    default library path."""
    out = Path(out) if out is not None else LIB_PATH
    if not defines and out == LIB_PATH and LIB_PATH.exists() and LIB_PATH.stat().st_mtime >= _SRC.stat().st_mtime:
        return LIB_PATH
    tmp = out.with_name(out.name + f".tmp{os.getpid()}")
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           *[f"-D{d}" for d in defines], str(_SRC), "-o", str(tmp), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: Path | None = None):
        path = Path(path) if path is not None else build()
        lib = ctypes.CDLL(str(path))
        ci, cd, cl = ctypes.c_int, ctypes.c_double, ctypes.c_long
        lib.oracle_attention_fwd.argtypes = [_u16p, _u16p, _u16p, _f64p, _f64p,
                                             ci, ci, ci, ci, ci, ci, cd, ci, ci, ci, ci]
        lib.oracle_attention_fwd.restype = ci
        lib.oracle_attention_probs.argtypes = [_u16p, _u16p, _u16p, _f64p, _f64p, _f64p,
                                               ci, ci, ci, ci, ci, ci, cd, ci, ci, ci]
        lib.oracle_attention_probs.restype = ci
        lib.oracle_attention_rows.argtypes = [_u16p, _u16p, _u16p, _i32p, cl, _f64p, _f64p,
                                              ci, ci, ci, ci, ci, ci, cd, ci, ci, ci, ci]
        lib.oracle_attention_rows.restype = ci
        lib.oracle_attention_bwd.argtypes = [_u16p, _u16p, _u16p, _u16p, _f64p, _f64p, _f64p,
                                             ci, ci, ci, ci, ci, ci, cd, ci, ci, ci, ci]
        lib.oracle_attention_bwd.restype = ci
        lib.oracle_attention_fwd_fp8.argtypes = [_u8p, _u8p, _u8p, _f64p, _f64p, ci, ci, ci, ci, ci, ci,
                                                 cd, cd, cd, cd, ci, ci, ci]
        lib.oracle_attention_fwd_fp8.restype = ci
        lib.oracle_attention_rows_fp8.argtypes = [_u8p, _u8p, _u8p, _i32p, cl, _f64p, _f64p, ci, ci, ci, ci, ci, ci,
                                                  cd, cd, cd, cd, ci, ci, ci]
        lib.oracle_attention_rows_fp8.restype = ci
        self.lib = lib

    @staticmethod
    def _dims(q, k, v):
        q, k, v = (np.ascontiguousarray(x, dtype=np.uint16) for x in (q, k, v))
        B, Nq, Hq, d = q.shape
        Bk, Nk, Hkv, dk = k.shape
        if v.shape != k.shape or Bk != B or dk != d:
            raise ValueError(f"shape mismatch q{q.shape} k{k.shape} v{v.shape}")
        return q, k, v, B, Hq, Hkv, Nq, Nk, d

    @staticmethod
    def _elem(dtype: str) -> int:
        if dtype not in ("bf16", "f16"):
            raise ValueError(f"dtype must be 'bf16' or 'f16', got {dtype!r}")
        return 1 if dtype == "f16" else 0

    def forward(self, q, k, v, scale: float, causal: bool, threads: int | None = None, window: int = 0,
                dtype: str = "bf16"):
        """O [B,Nq,Hq,d] and LSE [B,Hq,Nq] in fp64 from bf16 (dtype="f16": IEEE fp16)
        bit-pattern inputs (window = W >= 1: sliding window of the W keys ending at the
        causal diagonal)."""
        q, k, v, B, Hq, Hkv, Nq, Nk, d = self._dims(q, k, v)
        out = np.zeros((B, Nq, Hq, d), dtype=np.float64)
        lse = np.zeros((B, Hq, Nq), dtype=np.float64)
        rc = self.lib.oracle_attention_fwd(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d,
                                           float(scale), int(bool(causal)), int(window), self._elem(dtype),
                                           threads or os.cpu_count() or 1)
        if rc != 0:
            raise RuntimeError(f"oracle_attention_fwd failed: {rc}")
        return out, lse

    def probs(self, q, k, v, scale: float, causal: bool, window: int = 0, dtype: str = "bf16"):
        """(O, LSE, P) with P [B,Hq,Nq,Nk]; for tiny problems."""
        q, k, v, B, Hq, Hkv, Nq, Nk, d = self._dims(q, k, v)
        out = np.zeros((B, Nq, Hq, d), dtype=np.float64)
        lse = np.zeros((B, Hq, Nq), dtype=np.float64)
        P = np.zeros((B, Hq, Nq, Nk), dtype=np.float64)
        rc = self.lib.oracle_attention_probs(q, k, v, out, lse, P, B, Hq, Hkv, Nq, Nk, d,
                                             float(scale), int(bool(causal)), int(window), self._elem(dtype))
        if rc != 0:
            raise RuntimeError(f"oracle_attention_probs failed: {rc}")
        return out, lse, P

    def rows(self, q, k, v, rows, scale: float, causal: bool, threads: int | None = None, window: int = 0,
             dtype: str = "bf16"):
        """O [n,d] and LSE [n] of the listed (b, hq, i) rows."""
        q, k, v, B, Hq, Hkv, Nq, Nk, d = self._dims(q, k, v)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
        n = rows.shape[0]
        out = np.zeros((n, d), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        rc = self.lib.oracle_attention_rows(q, k, v, rows, n, out, lse, B, Hq, Hkv, Nq, Nk, d,
                                            float(scale), int(bool(causal)), int(window), self._elem(dtype),
                                            threads or os.cpu_count() or 1)
        if rc != 0:
            raise RuntimeError(f"oracle_attention_rows failed: {rc}")
        return out, lse


    def forward_fp8(self, q8, k8, v8, scale: float, causal: bool, descale=(1.0, 1.0, 1.0), threads: int | None = None,
                    window: int = 0):
        """O, LSE in fp64 for OCP E4M3 byte inputs with dequantisation factors
        descale = (dq, dk, dv): Q = dq * q8, K = dk * k8, V = dv * v8."""
        q8, k8, v8 = (np.ascontiguousarray(x, dtype=np.uint8) for x in (q8, k8, v8))
        B, Nq, Hq, d = q8.shape
        Bk, Nk, Hkv, dk_ = k8.shape
        if v8.shape != k8.shape or Bk != B or dk_ != d:
            raise ValueError(f"shape mismatch q{q8.shape} k{k8.shape} v{v8.shape}")
        out = np.zeros((B, Nq, Hq, d), dtype=np.float64)
        lse = np.zeros((B, Hq, Nq), dtype=np.float64)
        rc = self.lib.oracle_attention_fwd_fp8(q8, k8, v8, out, lse, B, Hq, Hkv, Nq, Nk, d, float(scale),
                                               float(descale[0]), float(descale[1]), float(descale[2]),
                                               int(bool(causal)), int(window), threads or os.cpu_count() or 1)
        if rc != 0:
            raise RuntimeError(f"oracle_attention_fwd_fp8 failed: {rc}")
        return out, lse

    def rows_fp8(self, q8, k8, v8, rows, scale: float, causal: bool, descale=(1.0, 1.0, 1.0),
                 threads: int | None = None, window: int = 0):
        """O [n,d] and LSE [n] of the listed (b, hq, i) rows for E4M3 inputs."""
        q8, k8, v8 = (np.ascontiguousarray(x, dtype=np.uint8) for x in (q8, k8, v8))
        B, Nq, Hq, d = q8.shape
        Nk, Hkv = k8.shape[1], k8.shape[2]
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
        n = rows.shape[0]
        out = np.zeros((n, d), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        rc = self.lib.oracle_attention_rows_fp8(q8, k8, v8, rows, n, out, lse, B, Hq, Hkv, Nq, Nk, d, float(scale),
                                                float(descale[0]), float(descale[1]), float(descale[2]),
                                                int(bool(causal)), int(window), threads or os.cpu_count() or 1)
        if rc != 0:
            raise RuntimeError(f"oracle_attention_rows_fp8 failed: {rc}")
        return out, lse

    def backward(self, q, k, v, dout, scale: float, causal: bool, threads: int | None = None, window: int = 0,
                 dtype: str = "bf16"):
        """(dQ [B,Nq,Hq,d], dK [B,Nk,Hkv,d], dV [B,Nk,Hkv,d]) in fp64: the gradient of
        sum(O * dO) for bit-pattern inputs q, k, v, dout of element type `dtype`."""
        q, k, v, B, Hq, Hkv, Nq, Nk, d = self._dims(q, k, v)
        dout = np.ascontiguousarray(dout, dtype=np.uint16)
        if dout.shape != q.shape:
            raise ValueError(f"dout shape {dout.shape} != q shape {q.shape}")
        dq = np.zeros((B, Nq, Hq, d), dtype=np.float64)
        dk = np.zeros((B, Nk, Hkv, d), dtype=np.float64)
        dv = np.zeros((B, Nk, Hkv, d), dtype=np.float64)
        rc = self.lib.oracle_attention_bwd(q, k, v, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, float(scale),
                                           int(bool(causal)), int(window), self._elem(dtype),
                                           threads or os.cpu_count() or 1)
        if rc != 0:
            raise RuntimeError(f"oracle_attention_bwd failed: {rc}")
        return dq, dk, dv


_default: Oracle | None = None


def default() -> Oracle:
    """The normally built oracle (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default

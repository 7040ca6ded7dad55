"""Seeded synthetic inputs for the attention forward: the only module that both the
CUDA path's tests/bench and the CPU oracle's tests draw inputs from.

It holds none of the attention arithmetic.  It turns (seed, workload id, tensor id)
into bf16 bit patterns:

  * splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014) used in counter mode: the i-th 64-bit word of a stream
    is mix(key + (i + 1) * golden_gamma);
  * 53-bit uniforms u = (w >> 11 + 1) / 2**53 in (0, 1];
  * Box & Muller (1958) pairs: z0 = sqrt(-2 ln u1) cos(2 pi u2),
    z1 = sqrt(-2 ln u1) sin(2 pi u2), computed in fp64;
  * fp64 -> fp32 (round to nearest even) -> bf16 (round to nearest even).

Layouts follow the [batch, seq, heads, head_dim] convention of the `flash_attn_func`
call shown on "Transformer efficient attention: Flash Attention vs GQA"
(yunthe.com, section "Flash Attention IO optimisation ... code practice").

The workload table mirrors the shapes the pages talk about: the YOLO11 C2PSA feature
maps (lpnh.cn/news/2773597, sections 1.2-1.3: a 20x20 map gives N=400, an 80x80 map
N=6400), the sequence-length sweep of the Atlas 800T A2 table (coreui.cn/article/2637497,
section 3), a Llama-2-70B-like GQA prefill (yunthe.com, GQA section: 32 query heads,
8 KV heads), a 16K context (yunthe.com, Flash Attention section) and the head-dim list
32/64/80/96/128/192/256 (datacanvas.csdn.net head-dim article, "head-dim limits").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "do": 4}


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function on a uint64 array (wrapping arithmetic)."""
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, workload_id: int, tensor_id: int) -> np.uint64:
    """64-bit key of one tensor's stream: mix of (seed, workload, tensor)."""
    packed = ((seed & 0xFFFFFFFF) << 32) ^ ((workload_id & 0xFFFFFF) << 8) ^ (tensor_id & 0xFF)
    with np.errstate(over="ignore"):
        return _mix(np.array([packed], dtype=np.uint64))[0]


def splitmix64_words(key: np.uint64, start: int, count: int) -> np.ndarray:
    """Words start .. start+count-1 of the counter-mode splitmix64 stream `key`."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + idx * GOLDEN_GAMMA)


def normal_f64(key: np.uint64, count: int, chunk: int = 1 << 24) -> np.ndarray:
    """`count` N(0,1) fp64 samples by Box-Muller over the stream `key`."""
    out = np.empty(count, dtype=np.float64)
    npairs = (count + 1) // 2
    scale = 1.0 / 9007199254740992.0  # 2**-53
    for p0 in range(0, npairs, chunk):
        p1 = min(npairs, p0 + chunk)
        w = splitmix64_words(key, 2 * p0, 2 * (p1 - p0))
        u = ((w >> np.uint64(11)).astype(np.float64) + 1.0) * scale  # (0, 1]
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log(u1))
        th = (2.0 * math.pi) * u2
        z = np.empty(2 * (p1 - p0), dtype=np.float64)
        z[0::2] = r * np.cos(th)
        z[1::2] = r * np.sin(th)
        lo, hi = 2 * p0, min(count, 2 * p1)
        out[lo:hi] = z[: hi - lo]
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bit patterns.
    Inputs are finite (the generator never makes NaN/Inf)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def scale_bf16_bits_pow2(bits: np.ndarray, factor: float) -> np.ndarray:
    """Multiply bf16 values by a power of two (exact: no over/underflow at these magnitudes)."""
    assert factor > 0 and math.log2(factor) == int(math.log2(factor))
    return f32_to_bf16_bits(bf16_bits_to_f32(bits) * np.float32(factor))


@dataclass(frozen=True)
class Workload:
    """One attention-forward problem: shapes, mask, scale and input recipe."""
    name: str
    wid: int                 # workload id mixed into the stream keys
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    q_mult: float = 1.0      # exact power-of-two multiplier applied to the bf16 Q values
    k_mult: float = 1.0      # same for K
    seed: int = 0
    window: int = 0          # sliding window of W keys (0: none; implies causal)
    splitkv: bool = False    # run with the library's default split-KV count (decode shapes)
    dtype: str = "bf16"      # element type of q, k, v: "bf16", "f16" (IEEE half) or "e4m3" (OCP FP8; out bf16)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """4*B*Hq*Nq*Nk*d, halved when causal (the throughput convention used here); with a
        sliding window of W keys, 4*B*Hq*d times the number of visible (query, key) pairs."""
        if self.window:
            off = self.Nk - self.Nq
            pairs = sum(max(0, min(i + off + 1, self.Nk) - max(0, i + off - self.window + 1))
                        for i in range(self.Nq))
            return 4.0 * self.B * self.Hq * self.d * pairs
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d
        return f / 2 if self.causal else f

    @property
    def io_bytes(self) -> int:
        """Algorithmic HBM bytes: Q, K, V read once, O written once (2-byte), LSE fp32."""
        q = self.B * self.Nq * self.Hq * self.d
        kv = self.B * self.Nk * self.Hkv * self.d
        es = 1 if self.dtype == "e4m3" else 2     # input element bytes; O is 2-byte either way
        return es * (q + 2 * kv) + 2 * q + 4 * self.B * self.Hq * self.Nq

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> IEEE half, round to nearest even (numpy's cast), as uint16 bit patterns."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> OCP FP8 E4M3 (round to nearest even, torch's cast), as uint8 bytes."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def make_inputs(w: Workload) -> dict[str, np.ndarray]:
    """Seeded bf16 (w.dtype "f16": IEEE half) bit patterns for q [B,Nq,Hq,d], k and v
    [B,Nk,Hkv,d].  The fp16 inputs are the same normal draws rounded to half, with the
    power-of-two multipliers applied before rounding (exact either way)."""
    if w.dtype == "e4m3":   # FP8 bytes of the same draws (times the multipliers); |x| << 448
        shapes = {"q": (w.B, w.Nq, w.Hq, w.d), "k": (w.B, w.Nk, w.Hkv, w.d), "v": (w.B, w.Nk, w.Hkv, w.d)}
        out = {}
        for name, shp in shapes.items():
            z = normal_f64(stream_key(w.seed, w.wid, TENSOR_IDS[name]), int(np.prod(shp)))
            mult = {"q": w.q_mult, "k": w.k_mult}.get(name, 1.0)
            out[name] = f32_to_e4m3_bits(z.astype(np.float32) * np.float32(mult)).reshape(shp)
        return out
    if w.dtype == "f16":
        shapes = {"q": (w.B, w.Nq, w.Hq, w.d), "k": (w.B, w.Nk, w.Hkv, w.d), "v": (w.B, w.Nk, w.Hkv, w.d)}
        out = {}
        for name, shp in shapes.items():
            z = normal_f64(stream_key(w.seed, w.wid, TENSOR_IDS[name]), int(np.prod(shp)))
            mult = {"q": w.q_mult, "k": w.k_mult}.get(name, 1.0)
            out[name] = f32_to_f16_bits(z.astype(np.float32) * np.float32(mult)).reshape(shp)
        return out
    shapes = {"q": (w.B, w.Nq, w.Hq, w.d), "k": (w.B, w.Nk, w.Hkv, w.d), "v": (w.B, w.Nk, w.Hkv, w.d)}
    out = {}
    for name, shp in shapes.items():
        n = int(np.prod(shp))
        z = normal_f64(stream_key(w.seed, w.wid, TENSOR_IDS[name]), n)
        bits = f32_to_bf16_bits(z.astype(np.float32))
        mult = {"q": w.q_mult, "k": w.k_mult}.get(name, 1.0)
        if mult != 1.0:
            bits = scale_bf16_bits_pow2(bits, mult)
        out[name] = bits.reshape(shp)
    return out


def make_grad_output(w: Workload) -> np.ndarray:
    """Seeded upstream gradient dO [B,Nq,Hq,d] for the backward pass: N(0,1) draws from
    their own stream, rounded to the workload's element type like the inputs."""
    shp = (w.B, w.Nq, w.Hq, w.d)
    z = normal_f64(stream_key(w.seed, w.wid, TENSOR_IDS["do"]), int(np.prod(shp))).astype(np.float32)
    bits = f32_to_f16_bits(z) if w.dtype == "f16" else f32_to_bf16_bits(z)
    return bits.reshape(shp)


def _wl(name, wid, B, H, N, d, causal=False, Hkv=None, Nk=None, **kw):
    return Workload(name, wid, B, H, Hkv or H, N, Nk or N, d, causal, **kw)


# The workload table.  Ids are stable: changing one changes every seeded input of it.
WORKLOADS: dict[str, Workload] = {}
for _w in [
    _wl("yolo20x20_b1_h4_d64", 1, 1, 4, 400, 64),
    _wl("yolo20x20_b1_h4_d64_qx8", 2, 1, 4, 400, 64, q_mult=8.0),
    _wl("yolo20x20_b32_h16_d64", 3, 32, 16, 400, 64),
    _wl("yolo80x80_b4_h16_d64", 4, 4, 16, 6400, 64),
    _wl("seq512_b8_h32_d128", 5, 8, 32, 512, 128),
    _wl("seq1024_b8_h32_d128", 6, 8, 32, 1024, 128),
    _wl("seq2048_b8_h32_d128", 7, 8, 32, 2048, 128),
    _wl("seq4096_b8_h32_d128", 8, 8, 32, 4096, 128),
    _wl("gqa_prefill_b4_n4096_hq32_hkv8_d128_causal", 9, 4, 32, 4096, 128, causal=True, Hkv=8, k_mult=0.5),
    _wl("long16k_b1_h32_d128_causal", 10, 1, 32, 16384, 128, causal=True),
    _wl("hdim32_b2_n4096_h16", 11, 2, 16, 4096, 32),
    _wl("hdim64_b2_n4096_h16", 12, 2, 16, 4096, 64),
    _wl("hdim80_b2_n4096_h16", 13, 2, 16, 4096, 80),
    _wl("hdim96_b2_n4096_h16", 14, 2, 16, 4096, 96),
    _wl("hdim192_b2_n4096_h16", 15, 2, 16, 4096, 192),
    _wl("hdim256_b2_n4096_h16", 16, 2, 16, 4096, 256),
    _wl("window4k_long16k_b1_h32_d128", 17, 1, 32, 16384, 128, causal=True, window=4096),
    _wl("decode_b4_hq32_hkv8_nq16_nk32k_d128", 18, 4, 32, 16, 128, Hkv=8, Nk=32768, splitkv=True),
    _wl("seq4096_b8_h32_d128_f16", 19, 8, 32, 4096, 128, dtype="f16"),
    _wl("gqa_prefill_b4_n4096_hq32_hkv8_d128_causal_f16", 20, 4, 32, 4096, 128, causal=True, Hkv=8, k_mult=0.5,
        dtype="f16"),
    _wl("seq4096_b8_h32_d128_fp8", 21, 8, 32, 4096, 128, dtype="e4m3"),
]:
    WORKLOADS[_w.name] = _w

# The workload the headline throughput number is quoted on: the longest point of the
# sequence-length sweep (d=128, N=4096), where the >=60%-of-peak target applies.
HEADLINE = "seq4096_b8_h32_d128"

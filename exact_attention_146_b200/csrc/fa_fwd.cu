// fa_fwd.cu -- the C ABI of libfa.so (declared in include/fa.h): argument validation,
// device and pointer checks, TMA tensor-map encoding, per-head-dim dispatch, launch,
// and the device status word.  One tuned kernel instantiation per head dimension, the
// per-hdim specialisation the datacanvas.csdn.net head-dim article describes (section
// "technical roots of the head-dim limit"), as C++ template instances.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_host.h"
#include "fa_kernel.cuh"

// ------------------------------------------------------------------ host helpers (fa_host.h)

namespace fa_host {

using fa::fa_no_keys_kernel;

__device__ int g_fa_status;   // per-device kernel status word (0 = OK)

DeviceState g_devices[kMaxDevices];
std::mutex g_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
using AddressRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

static void *driver_fn(const char *name) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return fn;
}

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(driver_fn("cuTensorMapEncodeTiled"));
    return fn;
}

static AddressRangeFn address_range_fn() {
    static AddressRangeFn fn = reinterpret_cast<AddressRangeFn>(driver_fn("cuMemGetAddressRange"));
    return fn;
}

// Current device, probed once: sm_100 (compute capability 10.0) or not.
int current_device(DeviceState **out, int *dev_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FA_ERR_UNSUPPORTED_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState &st = g_devices[dev];
    if (!st.probed) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return FA_ERR_UNSUPPORTED_DEVICE;
        }
        st.supported = (major == 10 && minor == 0);
        st.num_sms = sms;
        if (st.supported) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_fa_status) != cudaSuccess) {
                cudaGetLastError();
                return FA_ERR_CUDA;
            }
            st.status_ptr = static_cast<int *>(p);
        }
        st.probed = true;
    }
    if (!st.supported) return FA_ERR_UNSUPPORTED_DEVICE;
    *out = &st;
    *dev_out = dev;
    return FA_OK;
}

// `bytes` starting at `p` must be device (or managed) memory of device `dev`, inside one
// allocation.
int check_device_range(const void *p, size_t bytes, int dev) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_NOT_DEVICE_MEMORY;
    }
    if (!(a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) || a.device != dev)
        return FA_ERR_NOT_DEVICE_MEMORY;
    if (AddressRangeFn fn = address_range_fn()) {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS)
            return FA_ERR_NOT_DEVICE_MEMORY;
        const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
        if (lo + bytes > uintptr_t(base) + size) return FA_ERR_NOT_DEVICE_MEMORY;
    }
    return FA_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// 4-D view (d, H, N, B) of a [B, N, H, d] bf16 tensor, box (CW, heads, rows, 1): the box
// lands in shared memory as heads*rows swizzled rows, row-major over (row, head).
// elem: 0 bf16, 1 fp16, 2 E4M3 bytes.
int encode_bnhd(CUtensorMap *m, const void *base, int d, int H, int N, int B, int cw, int rows, int heads,
                int elem) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return FA_ERR_CUDA;
    const cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(H), cuuint64_t(N), cuuint64_t(B)};
    const cuuint64_t es = elem == 2 ? 1 : 2;
    const cuuint64_t strides[3] = {cuuint64_t(d) * es, cuuint64_t(H) * d * es, cuuint64_t(N) * H * d * es};
    const cuuint32_t box[4] = {cuuint32_t(cw), cuuint32_t(heads), cuuint32_t(rows), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw = (cw * es == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapDataType dt = elem == 2   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : elem == 1 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUresult r = fn(m, dt, 4, const_cast<void *>(base), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

int zero_fill(void *dst, size_t bytes, float *lse, size_t n_lse, int num_sms, cudaStream_t st) {
    const size_t n16 = bytes / 16;
    const int grid = int(std::min<size_t>((std::max(n16, n_lse) + 255) / 256, size_t(num_sms) * 8));
    fa_no_keys_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(static_cast<uint4 *>(dst), n16, lse, n_lse);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa_host

namespace {

using namespace fa;
using namespace fa_host;

// Tiling per head dim: TileCfg<d, key rows per tile, query tiles per unit, K/V slots,
// buffers per Q tile, S buffers per Q tile, P in TMEM columns of its own, exponential
// pairs per 8 on the FMA pipe, fp16 elements (H) instead of bf16, E4M3, failure-path
// build, one S buffer shared by the two query tiles>.  d = 80 ... 192: the two query tiles
// take turns in one S buffer and P has columns of its own (S + O_0 + O_1 + P_0 + P_1 fit
// the 512 TMEM columns), so no tile's next S waits for its own P V.  d = 256 runs one
// 128-row query tile, so it has TMEM room for a second S buffer (S_{j+1} computed while the
// softmax works on S_j); d <= 64 keeps an S buffer per tile with P apart from S (handed
// over in two halves), and is where the exponentials dominate.
template <bool H> using Cfg32 = TileCfg<32, 128, 2, 8, 2, 1, true, 2, H>;
template <bool H> using Cfg64 = TileCfg<64, 128, 2, 8, 2, 1, true, 2, H>;
template <bool H> using Cfg80 = TileCfg<80, 128, 2, 4, 1, 1, true, 0, H, false, false, true>;
template <bool H> using Cfg96 = TileCfg<96, 128, 2, 4, 1, 1, true, 0, H, false, false, true>;
template <bool H> using Cfg128 = TileCfg<128, 128, 2, 4, 1, 1, true, 0, H, false, false, true>;
template <bool H> using Cfg192 = TileCfg<192, 64, 2, 4, 1, 1, true, 0, H, false, false, true>;
template <bool H> using Cfg256 = TileCfg<256, 64, 1, 4, 1, 2, false, 0, H>;
// FP8 (E4M3) inputs.  d = 128: 16 KB tiles, so eight K/V slots; d = 64: 64-byte rows
// (64-byte swizzle, 8 KB tiles); both with the shared S buffer and P (E4M3, four per
// column) in columns of its own.  d = 256: one 128-row query tile with two S buffers
// (S 2 x 128 + O 256 TMEM columns), 32 KB tiles, P rounded to E4M3 over S.
using Cfg128F8 = TileCfg<128, 128, 2, 8, 1, 1, true, 0, false, true, false, true>;
using Cfg64F8 = TileCfg<64, 128, 2, 8, 1, 1, true, 0, false, true, false, true>;
using Cfg256F8 = TileCfg<256, 128, 1, 4, 1, 2, false, 0, false, true>;
// The d = 64 bf16 tiling built for the failure-path test (fa_test_withheld_load): wait limit
// taken from the parameters, one K/V load left out by the producer.
using Cfg64Fault = TileCfg<64, 128, 2, 8, 2, 1, true, 2, false, false, true>;
struct Problem {
    const void *q, *k, *v;
    void *out;
    float *lse;
    int B, Hq, Hkv, Nq, Nk, d;
    float scale;
    int causal;
    int window;
    int num_splits;     // 1: plain forward; > 1: split-KV into the workspace, then merge
    float *o_part;      // workspace: fp32 partial O [split][B][Nq][Hq][d]
    float *lse_part;    // workspace: partial LSE [split][B][Hq][Nq]
    float o_scale;      // FP8: V dequantisation factor (1 otherwise)
    int diag;           // causal diagonal offset (Nk - Nq unless a key shard)
    int partial;        // write the shard partial (fp32 O, LSE) to o_part / lse_part
    unsigned long long wait_limit_ns = kWaitLimitNs;   // failure-path test build only
    int withheld_load = -1;                              // failure-path test build only
};

// Workspace layout of the split-KV forward: partial O, then (256-byte aligned) partial LSE.
size_t splitkv_o_bytes(int B, int Hq, int Nq, int d, int splits) {
    return size_t(splits) * size_t(B) * size_t(Nq) * size_t(Hq) * size_t(d) * 4;
}
size_t splitkv_bytes(int B, int Hq, int Nq, int d, int splits) {
    if (splits <= 1) return 0;
    const size_t o = (splitkv_o_bytes(B, Hq, Nq, d, splits) + 255) & ~size_t(255);
    return o + size_t(splits) * size_t(B) * size_t(Hq) * size_t(Nq) * 4;
}

// GQA packing: with fewer than 128 queries, the n_rep query heads that share a KV head
// share one unit, their rows stacked in the tile (flat row i * n_rep + r), so a decode-sized
// Nq does not leave most of each 128-row tile empty.  Needs n_rep to divide 128 (the Q
// load box is n_rep heads x 128 / n_rep rows).  Each row's arithmetic is unchanged.
int pack_factor(int Hq, int Hkv, int Nq) {
    const int n_rep = Hq / Hkv;
    return (n_rep > 1 && kBlockQ % n_rep == 0 && Nq < kBlockQ) ? n_rep : 1;
}

template <class C>
int launch(const Problem &pr, DeviceState &dev, int cfg_slot, cudaStream_t stream) {
    auto kern = fa_fwd_kernel<C>;
    if (!dev.smem_attr_set[cfg_slot]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
            cudaSuccess) {
            cudaGetLastError();
            return FA_ERR_CUDA;
        }
        dev.smem_attr_set[cfg_slot] = true;
    }
    if (dev.regs_ok[cfg_slot] == 0) {
        // The in-kernel register reallocation assumes the kernel is launched with exactly
        // C::LAUNCH_REGS registers per thread; refuse to launch a build that differs.
        cudaFuncAttributes fattr{};
        if (cudaFuncGetAttributes(&fattr, kern) != cudaSuccess) {
            cudaGetLastError();
            return FA_ERR_CUDA;
        }
        dev.regs_ok[cfg_slot] = (!C::REALLOC_REGS || fattr.numRegs == C::LAUNCH_REGS) ? 1 : -1;
    }
    if (dev.regs_ok[cfg_slot] != 1) return FA_ERR_CUDA;
    CUtensorMap mq, mk, mv;
    int rc;
    const int pack = pack_factor(pr.Hq, pr.Hkv, pr.Nq);
    constexpr int elem = C::FP8 ? 2 : (C::F16 ? 1 : 0);
    if ((rc = encode_bnhd(&mq, pr.q, C::D, pr.Hq, pr.Nq, pr.B, C::CW, kBlockQ / pack, pack, elem)) != FA_OK)
        return rc;
    if ((rc = encode_bnhd(&mk, pr.k, C::D, pr.Hkv, pr.Nk, pr.B, C::CW, C::BC, 1, elem)) != FA_OK) return rc;
    if ((rc = encode_bnhd(&mv, pr.v, C::D, pr.Hkv, pr.Nk, pr.B, C::CW, C::BC, 1, elem)) != FA_OK) return rc;
    // O through shared memory and TMA stores: boxes of 64 columns x one warp's 32 flat rows
    // (pack heads x 32 / pack queries); only for the bf16 / fp16 output of a plain forward
    CUtensorMap mo = mq;
    const bool o_tma = C::OSTAGE && pr.partial == 0 && pr.num_splits <= 1 && pack <= 32;
    if (o_tma && (rc = encode_bnhd(&mo, pr.out, C::D, pr.Hq, pr.Nq, pr.B, 64, 32 / pack, pack, C::F16 ? 1 : 0)) != FA_OK)
        return rc;

    FwdParams p{};
    p.out = pr.out;
    p.lse = pr.lse;
    p.status = dev.status_ptr;
    p.B = pr.B;
    p.Hq = pr.Hq;
    p.Hkv = pr.Hkv;
    p.Nq = pr.Nq;
    p.Nk = pr.Nk;
    p.n_rep = pr.Hq / pr.Hkv;
    p.causal = pr.causal;
    p.window = pr.window;
    p.pack = pack;
    // Causal / window masks with GQA: pair two query heads of a KV group in a unit (both tiles
    // over the same rows, so they see the same key tiles and share every K/V load); otherwise
    // a unit is NQT consecutive 128-row tiles of one head.
    p.hpair = (C::NQT == 2 && pack == 1 && pr.causal && (pr.Hq / pr.Hkv) % 2 == 0) ? 1 : 0;
    p.nqb = p.hpair ? (pr.Nq + kBlockQ - 1) / kBlockQ
                    : (pr.Nq * pack + C::NQT * kBlockQ - 1) / (C::NQT * kBlockQ);
    const int nkv = (pr.Nk + C::BC - 1) / C::BC;
    p.num_splits = pr.num_splits > 1 ? pr.num_splits : 1;
    p.split_tiles = (nkv + p.num_splits - 1) / p.num_splits;
    p.o_part = pr.o_part;
    p.lse_part = pr.lse_part;
    const long long units = (long long)pr.B * (pr.Hq / (p.hpair ? C::NQT : pack)) * p.nqb * p.num_splits;
    if (units > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
    p.num_units = int(units);
    p.scale_log2 = pr.scale * 1.4426950408889634f;
    p.o_scale = pr.o_scale;
    p.diag = pr.diag;
    p.partial = pr.partial;
    p.wait_limit_ns = pr.wait_limit_ns;
    p.withheld_load = pr.withheld_load;
    p.o_tma = o_tma ? 1 : 0;

    const int grid = int(units < dev.num_sms ? units : dev.num_sms);
    fa_fwd_kernel<C><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(mq, mk, mv, mo, p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    if (p.num_splits > 1 && !p.partial) {
        const long long rows = (long long)pr.B * pr.Nq * pr.Hq;
        const long long want = (rows + 7) / 8;   // 8 rows (warps) per 256-thread block
        const int mgrid = int(want < 8LL * dev.num_sms ? want : 8LL * dev.num_sms);
        fa_splitkv_merge_kernel<C::D, C::F16><<<mgrid > 0 ? mgrid : 1, 256, 0, stream>>>(
            pr.o_part, pr.lse_part, static_cast<uint16_t *>(pr.out), pr.lse, pr.B, pr.Hq, pr.Nq, p.num_splits);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    return FA_OK;
}

// Per-head-dim launch for element type H (config slots 0-6 bf16, 8-14 fp16).
template <bool H>
int dispatch(const Problem &pr, DeviceState &dev, cudaStream_t st) {
    constexpr int base = H ? 8 : 0;
    switch (pr.d) {
        case 32: return launch<Cfg32<H>>(pr, dev, base + 0, st);
        case 64: return launch<Cfg64<H>>(pr, dev, base + 1, st);
        case 80: return launch<Cfg80<H>>(pr, dev, base + 2, st);
        case 96: return launch<Cfg96<H>>(pr, dev, base + 3, st);
        case 128: return launch<Cfg128<H>>(pr, dev, base + 4, st);
        case 192: return launch<Cfg192<H>>(pr, dev, base + 5, st);
        case 256: return launch<Cfg256<H>>(pr, dev, base + 6, st);
        default: return FA_ERR_UNSUPPORTED_HEAD_DIM;
    }
}

int tile_config(int d, int *bq, int *bk, int *nqt, int *ns) {
    int BC, NQT, NS;
    switch (d) {
        case 32: BC = Cfg32<false>::BC; NQT = Cfg32<false>::NQT; NS = Cfg32<false>::NS; break;
        case 64: BC = Cfg64<false>::BC; NQT = Cfg64<false>::NQT; NS = Cfg64<false>::NS; break;
        case 80: BC = Cfg80<false>::BC; NQT = Cfg80<false>::NQT; NS = Cfg80<false>::NS; break;
        case 96: BC = Cfg96<false>::BC; NQT = Cfg96<false>::NQT; NS = Cfg96<false>::NS; break;
        case 128: BC = Cfg128<false>::BC; NQT = Cfg128<false>::NQT; NS = Cfg128<false>::NS; break;
        case 192: BC = Cfg192<false>::BC; NQT = Cfg192<false>::NQT; NS = Cfg192<false>::NS; break;
        case 256: BC = Cfg256<false>::BC; NQT = Cfg256<false>::NQT; NS = Cfg256<false>::NS; break;
        default: return FA_ERR_UNSUPPORTED_HEAD_DIM;
    }
    if (bq) *bq = kBlockQ;
    if (bk) *bk = BC;
    if (nqt) *nqt = NQT;
    if (ns) *ns = NS;
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_version(void) { return 100; }

const char *fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "ok";
        case FA_ERR_INVALID_ARG:
            return "invalid argument (null pointer, negative size, Hq not a multiple of Hkv, scale not "
                   "finite and positive, causal not 0/1, or sizes beyond 32-bit indexing)";
        case FA_ERR_UNSUPPORTED_HEAD_DIM:
            return "unsupported head dimension: fa_fwd supports head dimensions 32, 64, 80, 96, 128, 192, 256";
        case FA_ERR_MISALIGNED: return "misaligned pointer: q/k/v/out need 16-byte, lse 4-byte alignment";
        case FA_ERR_UNSUPPORTED_DEVICE: return "no CUDA device, or the current device is not sm_100 (B200)";
        case FA_ERR_CUDA: return "a CUDA runtime or driver call failed";
        case FA_ERR_DEVICE_TIMEOUT: return "a kernel pipeline wait timed out; outputs are undefined";
        case FA_ERR_NOT_DEVICE_MEMORY:
            return "a tensor is not device memory of the current device, or runs past its allocation";
        case FA_ERR_OVERLAP: return "out or lse overlaps an input or each other";
        case FA_ERR_SCRATCH_LIMIT:
            return "the split-KV partials need more than the library's 16 MiB static scratch: use "
                   "fa_fwd_splitkv with a caller workspace, or fewer splits";
        default: return "unknown status";
    }
}

int fa_tile_config(int d, int *block_q, int *block_k, int *q_tiles_per_unit, int *kv_slots) {
    return tile_config(d, block_q, block_k, q_tiles_per_unit, kv_slots);
}

}  // extern "C"

namespace {

// The shared forward: mask = none (causal 0, window 0), causal (1, 0) or sliding window
// (1, W >= 1).
// `library_scratch`: the workspace is the library's own static scratch (already known to be
// device memory of the current device), so its device-range check is skipped.
// `fault`: run the failure-path test build instead (d = 64, bf16): {wait limit in ns, index of
// the withheld K/V load}.
struct FaultHook {
    unsigned long long wait_limit_ns;
    int withheld_load;
};

int forward(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq, int Hkv,
            int Nq, int Nk, int d, float scale, int causal, int window, int num_splits, void *workspace,
            size_t workspace_bytes, void *stream, bool library_scratch = false, int elem = 0, float o_scale = 1.f,
            const FaultHook *fault = nullptr) {
    // ---- host-only validation (no CUDA call before this block passes)
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (window < 0 || (window > 0 && !causal)) return FA_ERR_INVALID_ARG;
    if (num_splits < 1 || num_splits > kMaxSplits) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (tile_config(d, nullptr, nullptr, nullptr, nullptr) != FA_OK) return FA_ERR_UNSUPPORTED_HEAD_DIM;
    if (elem == 2 && d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED_HEAD_DIM;
    if (!std::isfinite(o_scale) || !(o_scale > 0.f)) return FA_ERR_INVALID_ARG;
    const size_t es = elem == 2 ? 1 : 2;   // input element bytes; out is 2-byte
    const size_t q_bytes = size_t(B) * size_t(Nq) * size_t(Hq) * size_t(d) * es;
    const size_t out_bytes = size_t(B) * size_t(Nq) * size_t(Hq) * size_t(d) * 2;
    const size_t kv_bytes = size_t(B) * size_t(Nk) * size_t(Hkv) * size_t(d) * es;
    const size_t lse_bytes = size_t(B) * size_t(Hq) * size_t(Nq) * 4;
    if (q_bytes == 0) return FA_OK;   // B == 0 or Nq == 0: no output rows
    if (q == nullptr || out == nullptr) return FA_ERR_INVALID_ARG;
    if (kv_bytes > 0 && (k == nullptr || v == nullptr)) return FA_ERR_INVALID_ARG;
    auto mis = [](const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (mis(q, 16) || mis(out, 16) || (kv_bytes > 0 && (mis(k, 16) || mis(v, 16))) || (lse && mis(lse, 4)))
        return FA_ERR_MISALIGNED;
    if (overlaps(out, out_bytes, q, q_bytes) || overlaps(out, out_bytes, k, kv_bytes) ||
        overlaps(out, out_bytes, v, kv_bytes) || overlaps(lse, lse_bytes, q, q_bytes) ||
        overlaps(lse, lse_bytes, k, kv_bytes) || overlaps(lse, lse_bytes, v, kv_bytes) ||
        overlaps(lse, lse_bytes, out, out_bytes))
        return FA_ERR_OVERLAP;
    const size_t ws_bytes = (Nk > 0) ? splitkv_bytes(B, Hq, Nq, d, num_splits) : 0;
    if (ws_bytes > 0) {
        if (workspace == nullptr || workspace_bytes < ws_bytes) return FA_ERR_INVALID_ARG;
        if (mis(workspace, 256)) return FA_ERR_MISALIGNED;
        if (overlaps(workspace, ws_bytes, q, q_bytes) || overlaps(workspace, ws_bytes, k, kv_bytes) ||
            overlaps(workspace, ws_bytes, v, kv_bytes) || overlaps(workspace, ws_bytes, out, out_bytes) ||
            overlaps(workspace, ws_bytes, lse, lse_bytes))
            return FA_ERR_OVERLAP;
    }

    // ---- device checks
    DeviceState *dev = nullptr;
    int dev_id = -1;
    int rc = current_device(&dev, &dev_id);
    if (rc != FA_OK) return rc;
    if ((rc = check_device_range(q, q_bytes, dev_id)) != FA_OK) return rc;
    if ((rc = check_device_range(out, out_bytes, dev_id)) != FA_OK) return rc;
    if (kv_bytes > 0) {
        if ((rc = check_device_range(k, kv_bytes, dev_id)) != FA_OK) return rc;
        if ((rc = check_device_range(v, kv_bytes, dev_id)) != FA_OK) return rc;
    }
    if (lse && (rc = check_device_range(lse, lse_bytes, dev_id)) != FA_OK) return rc;
    if (ws_bytes > 0 && !library_scratch && (rc = check_device_range(workspace, ws_bytes, dev_id)) != FA_OK)
        return rc;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (Nk == 0) {
        const size_t n16 = out_bytes / 16;
        const int grid = int(std::min<size_t>((n16 + 255) / 256, size_t(dev->num_sms) * 8));
        fa_no_keys_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(static_cast<uint4 *>(out), n16, lse,
                                                             lse ? size_t(B) * Hq * Nq : 0);
        return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }

    float *o_part = nullptr, *lse_part = nullptr;
    if (ws_bytes > 0) {
        o_part = static_cast<float *>(workspace);
        lse_part = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                             ((splitkv_o_bytes(B, Hq, Nq, d, num_splits) + 255) & ~size_t(255)));
    }
    const Problem pr{q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, window,
                     ws_bytes > 0 ? num_splits : 1, o_part, lse_part, o_scale, Nk - Nq, 0};
    if (fault != nullptr) {
        if (d != 64 || elem != 0 || ws_bytes > 0) return FA_ERR_UNSUPPORTED_HEAD_DIM;
        Problem pf = pr;
        pf.wait_limit_ns = fault->wait_limit_ns;
        pf.withheld_load = fault->withheld_load;
        return launch<Cfg64Fault>(pf, *dev, kFaultSlot, st);
    }
    if (elem == 2) {
        if (d == 64) return launch<Cfg64F8>(pr, *dev, kFp8Slot64, st);
        if (d == 256) return launch<Cfg256F8>(pr, *dev, kFp8Slot256, st);
        return launch<Cfg128F8>(pr, *dev, kFp8Slot, st);
    }
    return elem == 1 ? dispatch<true>(pr, *dev, st) : dispatch<false>(pr, *dev, st);
}

}  // namespace

extern "C" {

int fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq, int Hkv,
           int Nq, int Nk, int d, float scale, int causal, void *stream) {
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, 1, nullptr, 0, stream);
}

size_t fa_splitkv_workspace_bytes(int B, int Hq, int Nq, int d, int num_splits) {
    if (B < 0 || Hq < 0 || Nq < 0 || d <= 0 || num_splits < 1 || num_splits > kMaxSplits) return 0;
    return splitkv_bytes(B, Hq, Nq, d, num_splits);
}

int fa_splitkv_default_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d, int sm_count) {
    int bq, bk, nqt, ns;
    if (tile_config(d, &bq, &bk, &nqt, &ns) != FA_OK || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 ||
        Nq <= 0 || Nk <= 0 || sm_count <= 0)
        return 1;
    const int pack = pack_factor(Hq, Hkv, Nq);
    const long long units = (long long)B * (Hq / pack) * ((Nq * pack + bq * nqt - 1) / (bq * nqt));
    if (units >= sm_count) return 1;
    // Cost of S splits in key-tile steps of the busiest SM: waves x (tiles per split + one
    // step of per-unit overhead: Q load, pipeline fill, epilogue).  Keep >= 4 key tiles per
    // split; the smallest S of equal cost wins.
    const long long nkv = (Nk + bk - 1) / bk;
    long long best = 1, best_cost = -1;
    for (long long sp = 1; sp <= kMaxSplits && (sp == 1 || nkv / sp >= 4); ++sp) {
        const long long waves = (units * sp + sm_count - 1) / sm_count;
        const long long cost = waves * ((nkv + sp - 1) / sp + 1);
        if (best_cost < 0 || cost < best_cost) {
            best = sp;
            best_cost = cost;
        }
    }
    return int(best);
}

int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, int d, float scale, int causal, int num_splits, void *workspace,
                   size_t workspace_bytes, void *stream) {
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, num_splits, workspace,
                   workspace_bytes, stream);
}

}  // extern "C"

namespace {

// Scratch of fa_fwd_splitkv_static, for callers that cannot allocate device memory around
// the call (see include/fa.h).  One array per device (a __device__ variable exists once in
// every device context); its address is looked up once per device, with that device current.
static __device__ __align__(256) unsigned char g_splitkv_scratch[FA_SPLITKV_STATIC_SCRATCH_BYTES];
void *g_scratch_addr[kMaxDevices] = {};

int static_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FA_ERR_UNSUPPORTED_DEVICE;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_splitkv_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return FA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_fwd_splitkv_static(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq,
                          int Hkv, int Nq, int Nk, int d, float scale, int causal, int num_splits,
                          void *stream) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || num_splits < 1 || num_splits > kMaxSplits)
        return FA_ERR_INVALID_ARG;
    if (tile_config(d, nullptr, nullptr, nullptr, nullptr) != FA_OK) return FA_ERR_UNSUPPORTED_HEAD_DIM;
    const size_t need = (Nk > 0) ? splitkv_bytes(B, Hq, Nq, d, num_splits) : 0;
    if (need > sizeof(g_splitkv_scratch)) return FA_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if (need > 0) {
        const int rc = static_scratch(&scratch);
        if (rc != FA_OK) return rc;
    }
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, num_splits, scratch,
                   sizeof(g_splitkv_scratch), stream, true);
}

int fa_fwd_f16(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq, int Hkv,
               int Nq, int Nk, int d, float scale, int causal, void *stream) {
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, 1, nullptr, 0, stream, false, 1);
}

int fa_fwd_fp8(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq, int Hkv,
               int Nq, int Nk, int d, float scale, float descale_q, float descale_k, float descale_v, int causal,
               void *stream) {
    if (!std::isfinite(descale_q) || !(descale_q > 0.f) || !std::isfinite(descale_k) || !(descale_k > 0.f))
        return FA_ERR_INVALID_ARG;
    const float s = scale * descale_q * descale_k;   // logits of the dequantised Q, K
    if (!std::isfinite(scale) || !(scale > 0.f) || !std::isfinite(s) || !(s > 0.f)) return FA_ERR_INVALID_ARG;
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, s, causal, 0, 1, nullptr, 0, stream, false, 2,
                   descale_v);
}

int fa_fwd_window(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq,
                  int Hkv, int Nq, int Nk, int d, float scale, int window, void *stream) {
    if (window < 1) return FA_ERR_INVALID_ARG;
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, 1, window, 1, nullptr, 0, stream);
}

int fa_fwd_window_f16(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq,
                      int Hkv, int Nq, int Nk, int d, float scale, int window, void *stream) {
    if (window < 1) return FA_ERR_INVALID_ARG;
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, 1, window, 1, nullptr, 0, stream, false, 1);
}

int fa_fwd_splitkv_f16(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq,
                       int Hkv, int Nq, int Nk, int d, float scale, int causal, int num_splits, void *workspace,
                       size_t workspace_bytes, void *stream) {
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, num_splits, workspace,
                   workspace_bytes, stream, false, 1);
}

int fa_test_withheld_load(const void *q, const void *k, const void *v, void *out, float *lse, int B, int Hq,
                          int Hkv, int Nq, int Nk, float scale, int causal, int withheld_load,
                          unsigned int wait_limit_us, void *stream) {
    if (withheld_load < 0 || wait_limit_us < 1u || wait_limit_us > 1000000u) return FA_ERR_INVALID_ARG;
    const FaultHook hook{1000ull * wait_limit_us, withheld_load};
    return forward(q, k, v, out, lse, B, Hq, Hkv, Nq, Nk, 64, scale, causal, 0, 1, nullptr, 0, stream, false, 0, 1.f,
                   &hook);
}

int fa_device_status(void *stream, int *detail) {
    DeviceState *dev = nullptr;
    int dev_id = -1;
    int rc = current_device(&dev, &dev_id);
    if (rc != FA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int word = 0;
    const int zero = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&word, g_fa_status, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(g_fa_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_CUDA;
    }
    if (detail) *detail = word;
    return (word & 0xFF) == 0 ? FA_OK : (word & 0xFF);
}

}  // extern "C"

// ------------------------------------------------------------------ key-sharded partials

namespace {

template <int D>
void merge_launch(const float *o_parts, const float *lse_parts, int R, void *out, float *lse, int B, int Hq, int Nq,
                  int num_sms, cudaStream_t st) {
    const long long rows = (long long)B * Nq * Hq;
    const long long want = (rows + 7) / 8;
    const int grid = int(want < 8LL * num_sms ? want : 8LL * num_sms);
    fa_splitkv_merge_kernel<D, false><<<grid > 0 ? grid : 1, 256, 0, st>>>(o_parts, lse_parts,
                                                                          static_cast<uint16_t *>(out), lse, B, Hq, Nq, R);
}

}  // namespace

extern "C" {

int fa_fwd_partial(const void *q, const void *k, const void *v, float *o_part, float *lse_part, int B, int Hq,
                   int Hkv, int Nq, int Nk, int d, float scale, int causal, int key_offset, int Nk_total,
                   void *stream) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (key_offset < 0 || Nk_total < 0 || (long long)key_offset + Nk > Nk_total) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (tile_config(d, nullptr, nullptr, nullptr, nullptr) != FA_OK) return FA_ERR_UNSUPPORTED_HEAD_DIM;
    const size_t q_bytes = size_t(B) * size_t(Nq) * size_t(Hq) * size_t(d) * 2;
    const size_t kv_bytes = size_t(B) * size_t(Nk) * size_t(Hkv) * size_t(d) * 2;
    const size_t op_bytes = size_t(B) * size_t(Nq) * size_t(Hq) * size_t(d) * 4;
    const size_t lse_bytes = size_t(B) * size_t(Hq) * size_t(Nq) * 4;
    if (q_bytes == 0) return FA_OK;
    if (q == nullptr || o_part == nullptr || lse_part == nullptr) return FA_ERR_INVALID_ARG;
    if (kv_bytes > 0 && (k == nullptr || v == nullptr)) return FA_ERR_INVALID_ARG;
    auto mis = [](const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (mis(q, 16) || mis(o_part, 16) || mis(lse_part, 4) || (kv_bytes > 0 && (mis(k, 16) || mis(v, 16))))
        return FA_ERR_MISALIGNED;
    if (overlaps(o_part, op_bytes, q, q_bytes) || overlaps(o_part, op_bytes, k, kv_bytes) ||
        overlaps(o_part, op_bytes, v, kv_bytes) || overlaps(lse_part, lse_bytes, q, q_bytes) ||
        overlaps(lse_part, lse_bytes, k, kv_bytes) || overlaps(lse_part, lse_bytes, v, kv_bytes) ||
        overlaps(lse_part, lse_bytes, o_part, op_bytes))
        return FA_ERR_OVERLAP;
    DeviceState *dev = nullptr;
    int dev_id = -1;
    int rc = current_device(&dev, &dev_id);
    if (rc != FA_OK) return rc;
    if ((rc = check_device_range(q, q_bytes, dev_id)) != FA_OK) return rc;
    if ((rc = check_device_range(o_part, op_bytes, dev_id)) != FA_OK) return rc;
    if ((rc = check_device_range(lse_part, lse_bytes, dev_id)) != FA_OK) return rc;
    if (kv_bytes > 0) {
        if ((rc = check_device_range(k, kv_bytes, dev_id)) != FA_OK) return rc;
        if ((rc = check_device_range(v, kv_bytes, dev_id)) != FA_OK) return rc;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (Nk == 0) {   // an empty shard: O = 0, LSE = -inf (weight 0 in the merge)
        const size_t n16 = op_bytes / 16;
        const int grid = int(std::min<size_t>((n16 + 255) / 256, size_t(dev->num_sms) * 8));
        fa_no_keys_kernel<<<grid > 0 ? grid : 1, 256, 0, st>>>(reinterpret_cast<uint4 *>(o_part), n16, lse_part,
                                                             size_t(B) * Hq * Nq);
        return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    const Problem pr{q, k, v, nullptr, nullptr, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0,
                     1, o_part, lse_part, 1.f, Nk_total - Nq - key_offset, 1};
    return dispatch<false>(pr, *dev, st);
}

int fa_merge_partials(const float *o_parts, const float *lse_parts, int R, void *out, float *lse, int B, int Hq,
                      int Nq, int d, void *stream) {
    if (R < 1 || B < 0 || Hq <= 0 || Nq < 0) return FA_ERR_INVALID_ARG;
    if (tile_config(d, nullptr, nullptr, nullptr, nullptr) != FA_OK) return FA_ERR_UNSUPPORTED_HEAD_DIM;
    const size_t rows = size_t(B) * size_t(Nq) * size_t(Hq);
    if (rows == 0) return FA_OK;
    if (o_parts == nullptr || lse_parts == nullptr || out == nullptr) return FA_ERR_INVALID_ARG;
    const size_t op_bytes = size_t(R) * rows * size_t(d) * 4, lp_bytes = size_t(R) * rows * 4;
    const size_t out_bytes = rows * size_t(d) * 2, lse_bytes = rows * 4;
    auto mis = [](const void *p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (mis(o_parts, 4) || mis(lse_parts, 4) || mis(out, 2) || mis(lse, 4)) return FA_ERR_MISALIGNED;
    if (overlaps(out, out_bytes, o_parts, op_bytes) || overlaps(out, out_bytes, lse_parts, lp_bytes) ||
        overlaps(lse, lse_bytes, o_parts, op_bytes) || overlaps(lse, lse_bytes, lse_parts, lp_bytes) ||
        overlaps(lse, lse_bytes, out, out_bytes))
        return FA_ERR_OVERLAP;
    DeviceState *dev = nullptr;
    int dev_id = -1;
    int rc = current_device(&dev, &dev_id);
    if (rc != FA_OK) return rc;
    if ((rc = check_device_range(o_parts, op_bytes, dev_id)) != FA_OK) return rc;
    if ((rc = check_device_range(lse_parts, lp_bytes, dev_id)) != FA_OK) return rc;
    if ((rc = check_device_range(out, out_bytes, dev_id)) != FA_OK) return rc;
    if (lse && (rc = check_device_range(lse, lse_bytes, dev_id)) != FA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (d) {
        case 32: merge_launch<32>(o_parts, lse_parts, R, out, lse, B, Hq, Nq, dev->num_sms, st); break;
        case 64: merge_launch<64>(o_parts, lse_parts, R, out, lse, B, Hq, Nq, dev->num_sms, st); break;
        case 80: merge_launch<80>(o_parts, lse_parts, R, out, lse, B, Hq, Nq, dev->num_sms, st); break;
        case 96: merge_launch<96>(o_parts, lse_parts, R, out, lse, B, Hq, Nq, dev->num_sms, st); break;
        case 128: merge_launch<128>(o_parts, lse_parts, R, out, lse, B, Hq, Nq, dev->num_sms, st); break;
        case 192: merge_launch<192>(o_parts, lse_parts, R, out, lse, B, Hq, Nq, dev->num_sms, st); break;
        default: merge_launch<256>(o_parts, lse_parts, R, out, lse, B, Hq, Nq, dev->num_sms, st); break;
    }
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"

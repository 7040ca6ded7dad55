// fa_bwd.cu -- the C ABI of the backward pass (declared in include/fa.h): argument
// validation, workspace layout, tensor maps and the three launches (D and the zeroed dQ
// accumulator, the main kernel of fa_bwd_kernel.cuh, dQ = bf16(scale * acc)).
#include <algorithm>
#include <cmath>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_bwd_kernel.cuh"
#include "fa_host.h"

// ------------------------------------------------------------------ backward

namespace {

using namespace fa_host;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The fp32 dQ accumulator [B, Nq, Hq, d] as a 4-D (d, Hq, Nq, B) tensor with [64 x 32] boxes
// (128-byte rows, 128-byte swizzle): the destination of the TMA reductions.
int encode_dq_acc(CUtensorMap *m, float *base, int d, int Hq, int Nq, int B) {
    static EncodeTiledFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    if (fn == nullptr) return FA_ERR_CUDA;
    const cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(Hq), cuuint64_t(Nq), cuuint64_t(B)};
    const cuuint64_t strides[3] = {cuuint64_t(d) * 4, cuuint64_t(Hq) * d * 4, cuuint64_t(Nq) * Hq * d * 4};
    const cuuint32_t box[4] = {32, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// The backward covers every forward head dim whose S^T, dP^T, dV and dK fit the 512 TMEM
// columns (256 + 2 d <= 512): d in {32, 64, 80, 96, 128}.  Per device, whether the dynamic
// shared-memory size of each bf16 / fp16 instantiation has been set.
bool g_bwd_smem_set[kMaxDevices][10] = {};

// Workspace of the backward: the fp32 dQ accumulator [B, Nq, Hq, d], then (256-byte
// aligned) D = rowsum(dO * O) [B, Hq, Nq].
size_t bwd_acc_bytes(int B, int Hq, int Nq, int d) {
    return (size_t(B) * size_t(Nq) * size_t(Hq) * size_t(d) * 4 + 255) & ~size_t(255);
}
size_t bwd_bytes(int B, int Hq, int Nq, int d) {
    return bwd_acc_bytes(B, Hq, Nq, d) + size_t(B) * size_t(Hq) * size_t(Nq) * 4;
}

template <class C>
int launch_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
               void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, float scale, int causal,
               int window, float *dq_acc, float *delta, DeviceState &dev, int dev_id, int slot, cudaStream_t st) {
    auto kern = fa::bwd::fa_bwd_kernel<C>;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!g_bwd_smem_set[dev_id][slot]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess) {
                cudaGetLastError();
                return FA_ERR_CUDA;
            }
            g_bwd_smem_set[dev_id][slot] = true;
        }
    }
    constexpr int elem = C::F16 ? 1 : 0;
    CUtensorMap mq, mk, mv, mdo, mdq;
    int rc;
    if ((rc = encode_bnhd(&mq, q, C::D, Hq, Nq, B, C::CW, fa::bwd::kRows, 1, elem)) != FA_OK) return rc;
    if ((rc = encode_bnhd(&mdo, dout, C::D, Hq, Nq, B, C::CW, fa::bwd::kRows, 1, elem)) != FA_OK) return rc;
    if ((rc = encode_bnhd(&mk, k, C::D, Hkv, Nk, B, C::CW, fa::bwd::kRows, 1, elem)) != FA_OK) return rc;
    if ((rc = encode_bnhd(&mv, v, C::D, Hkv, Nk, B, C::CW, fa::bwd::kRows, 1, elem)) != FA_OK) return rc;
    if ((rc = encode_dq_acc(&mdq, dq_acc, C::D, Hq, Nq, B)) != FA_OK) return rc;

    // D and the zeroed accumulator
    const long long rows = (long long)B * Nq * Hq;
    const long long want = (rows + 7) / 8;
    const int pgrid = int(want < 8LL * dev.num_sms ? want : 8LL * dev.num_sms);
    fa::bwd::fa_bwd_pre_kernel<C::D, C::F16><<<pgrid > 0 ? pgrid : 1, 256, 0, st>>>(
        static_cast<const uint16_t *>(out), static_cast<const uint16_t *>(dout), delta, dq_acc, B, Hq, Nq);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;

    fa::bwd::BwdParams p{};
    p.lse = lse;
    p.delta = delta;
    p.dq_acc = dq_acc;
    p.dk = static_cast<uint16_t *>(dk);
    p.dv = static_cast<uint16_t *>(dv);
    p.status = dev.status_ptr;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.Nq = Nq;
    p.Nk = Nk;
    p.n_rep = Hq / Hkv;
    p.causal = causal;
    p.window = window;
    p.nkt = (Nk + fa::bwd::kRows - 1) / fa::bwd::kRows;
    p.nqt = (Nq + fa::bwd::kRows - 1) / fa::bwd::kRows;
    const long long units = (long long)B * Hkv * p.nkt;
    if (units > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
    p.num_units = int(units);
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    const int grid = int(units < dev.num_sms ? units : dev.num_sms);
    kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(mq, mk, mv, mdo, mdq, p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;

    const size_t n4 = size_t(rows) * C::D / 4;
    const int qgrid = int(std::min<size_t>((n4 + 255) / 256, size_t(dev.num_sms) * 8));
    fa::bwd::fa_bwd_post_kernel<C::F16><<<qgrid > 0 ? qgrid : 1, 256, 0, st>>>(reinterpret_cast<const float4 *>(dq_acc),
                                                                      static_cast<uint2 *>(dq), n4, scale);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool H>
int dispatch_bwd(int d, const void *q, const void *k, const void *v, const void *out, const void *dout,
                 const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, float scale,
                 int causal, int window, float *dq_acc, float *delta, DeviceState &dev, int dev_id, cudaStream_t st) {
    constexpr int base = H ? 5 : 0;
#define FA_BWD_CASE(DIM, IDX)                                                                                      \
    case DIM:                                                                                                      \
        return launch_bwd<fa::bwd::BwdCfg<DIM, H>>(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, \
                                                   causal, window, dq_acc, delta, dev, dev_id, base + IDX, st);
    switch (d) {
        FA_BWD_CASE(32, 0)
        FA_BWD_CASE(64, 1)
        FA_BWD_CASE(80, 2)
        FA_BWD_CASE(96, 3)
        FA_BWD_CASE(128, 4)
        default: return FA_ERR_UNSUPPORTED_HEAD_DIM;
    }
#undef FA_BWD_CASE
}

int backward(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
             void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
             int window, void *workspace, size_t workspace_bytes, void *stream, bool f16) {
    // ---- host-only validation
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (window < 0 || (window > 0 && !causal)) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 32 && d != 64 && d != 80 && d != 96 && d != 128) return FA_ERR_UNSUPPORTED_HEAD_DIM;
    const size_t q_bytes = size_t(B) * size_t(Nq) * size_t(Hq) * size_t(d) * 2;
    const size_t kv_bytes = size_t(B) * size_t(Nk) * size_t(Hkv) * size_t(d) * 2;
    const size_t lse_bytes = size_t(B) * size_t(Hq) * size_t(Nq) * 4;
    if (q_bytes == 0 && kv_bytes == 0) return FA_OK;
    if (q_bytes > 0 && (q == nullptr || out == nullptr || dout == nullptr || lse == nullptr || dq == nullptr))
        return FA_ERR_INVALID_ARG;
    if (kv_bytes > 0 && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr)) return FA_ERR_INVALID_ARG;
    auto mis = [](const void *p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) != 0; };
    if (mis(q, 16) || mis(k, 16) || mis(v, 16) || mis(out, 16) || mis(dout, 16) || mis(dq, 16) || mis(dk, 16) ||
        mis(dv, 16) || mis(lse, 4))
        return FA_ERR_MISALIGNED;
    // outputs must not overlap any input or each other
    const void *ins[6] = {q, k, v, out, dout, lse};
    const size_t in_bytes[6] = {q_bytes, kv_bytes, kv_bytes, q_bytes, q_bytes, lse_bytes};
    void *outs[3] = {dq, dk, dv};
    const size_t out_bytes[3] = {q_bytes, kv_bytes, kv_bytes};
    for (int o = 0; o < 3; ++o) {
        for (int i = 0; i < 6; ++i)
            if (overlaps(outs[o], out_bytes[o], ins[i], in_bytes[i])) return FA_ERR_OVERLAP;
        for (int o2 = o + 1; o2 < 3; ++o2)
            if (overlaps(outs[o], out_bytes[o], outs[o2], out_bytes[o2])) return FA_ERR_OVERLAP;
    }
    const bool work = q_bytes > 0 && kv_bytes > 0;
    const size_t ws_bytes = work ? bwd_bytes(B, Hq, Nq, d) : 0;
    if (work) {
        if (workspace == nullptr || workspace_bytes < ws_bytes) return FA_ERR_INVALID_ARG;
        if (mis(workspace, 256)) return FA_ERR_MISALIGNED;
        for (int i = 0; i < 6; ++i)
            if (overlaps(workspace, ws_bytes, ins[i], in_bytes[i])) return FA_ERR_OVERLAP;
        for (int o = 0; o < 3; ++o)
            if (overlaps(workspace, ws_bytes, outs[o], out_bytes[o])) return FA_ERR_OVERLAP;
    }

    // ---- device checks
    DeviceState *dev = nullptr;
    int dev_id = -1;
    int rc = current_device(&dev, &dev_id);
    if (rc != FA_OK) return rc;
    for (int i = 0; i < 6; ++i)
        if (in_bytes[i] > 0 && (rc = check_device_range(ins[i], in_bytes[i], dev_id)) != FA_OK) return rc;
    for (int o = 0; o < 3; ++o)
        if (out_bytes[o] > 0 && (rc = check_device_range(outs[o], out_bytes[o], dev_id)) != FA_OK) return rc;
    if (work && (rc = check_device_range(workspace, ws_bytes, dev_id)) != FA_OK) return rc;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!work) {   // no query rows or no keys: every gradient that exists is zero
        for (int o = 0; o < 3; ++o) {
            if (out_bytes[o] == 0) continue;
            if (zero_fill(outs[o], out_bytes[o], nullptr, 0, dev->num_sms, st) != FA_OK) return FA_ERR_CUDA;
        }
        return FA_OK;
    }
    float *dq_acc = static_cast<float *>(workspace);
    float *delta = reinterpret_cast<float *>(static_cast<char *>(workspace) + bwd_acc_bytes(B, Hq, Nq, d));
    return f16 ? dispatch_bwd<true>(d, q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, causal, window,
                                    dq_acc, delta, *dev, dev_id, st)
               : dispatch_bwd<false>(d, q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, scale, causal, window,
                                     dq_acc, delta, *dev, dev_id, st);
}

}  // namespace

extern "C" {

size_t fa_bwd_workspace_bytes(int B, int Hq, int Nq, int d) {
    if (B < 0 || Hq < 0 || Nq < 0 || d <= 0) return 0;
    return bwd_bytes(B, Hq, Nq, d);
}

int fa_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
           void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
           void *workspace, size_t workspace_bytes, void *stream) {
    return backward(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, workspace,
                    workspace_bytes, stream, false);
}

int fa_bwd_f16(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
               void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
               void *workspace, size_t workspace_bytes, void *stream) {
    return backward(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, 0, workspace,
                    workspace_bytes, stream, true);
}

int fa_bwd_window(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
                  void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                  void *workspace, size_t workspace_bytes, void *stream) {
    if (window < 1) return FA_ERR_INVALID_ARG;
    return backward(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, 1, window, workspace,
                    workspace_bytes, stream, false);
}

}  // extern "C"


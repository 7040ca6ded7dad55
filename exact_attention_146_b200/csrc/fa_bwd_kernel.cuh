// fa_bwd_kernel.cuh -- exact attention backward for sm_100a (tcgen05 + TMEM + TMA).
//
// The backward pass recomputes S and P from Q, K, V instead of storing them: the
// lpnh.cn YOLO11 / FlashAttention-2 article (section 2.3, "reverse recomputation") and the
// hwcomputing.csdn.net article "FlashAttention in CANN ops-transformer" ("performance
// tuning") describe it; with the forward's log-sum-exp L_i, P_ij = exp(scale S_ij - L_i)
// exactly, so nothing but L (and D_i = dO_i . O_i) has to be kept from the forward.  The
// gradients of sum O (.) dO are
//
//     dV = P^T dO,   dP = dO V^T,   dS = P (.) (dP - D),   dQ = scale dS K,   dK = scale dS^T Q.
//
// Work unit: (batch b, KV head g, 128-key tile j).  The unit keeps K_j and V_j in shared
// memory and dK_j, dV_j in TMEM, and walks every (query head of g, 128-row query tile i)
// that can see the tile (causal: from the diagonal on), one "step" per pair:
//
//   MMA  S^T  = K_j Q_i^T     (128 keys x 128 queries, TMEM region A)
//   MMA  dP^T = V_j dO_i^T    (region B)
//   warpgroup SG (thread = key row): P^T = exp2(S^T scale log2e - L log2e), masked;
//        dS^T = P^T (.) (dP^T - D); P^T and dS^T back to TMEM as bf16 (over A and B),
//        dS^T also to shared memory (128-byte swizzled, M-major: the A operand of dQ)
//   MMA  dV_j += P^T dO_i     (A = P^T from TMEM)
//   MMA  dK_j += dS^T Q_i     (A = dS^T from TMEM)
//   MMA  dQ_i  = dS K_j       (A = dS^T in shared memory, M-major; into region A once
//                              P^T has been consumed)
//   warpgroup DW (thread = query row): dQ_i rows -> shared memory (the step's Q and dO
//        slots, free once its MMAs are done) -> TMA bulk tensor reductions (add) into an
//        fp32 dQ accumulator in global memory (every key tile of the head contributes);
//        the slots go back to the TMA producer when the reductions have read them
//
// and at the end of the unit DW writes dV_j and scale * dK_j as bf16.  Each shared-memory
// tile serves two MMAs in both roles (K-major where it is reduced over d, M/N-major where
// it is reduced over its rows), so nothing is loaded twice.  A preprocessing kernel
// computes D and zeroes the accumulator; a postprocessing kernel writes dQ = scale * acc.
#pragma once

#include <cstdint>
#include <type_traits>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int kRows = 128;   // key rows per unit = query rows per step = TMEM lanes

enum BwdSite : int {
    kSiteKvFull = 21, kSiteKvEmpty = 22, kSiteQFull = 23, kSiteQEmpty = 24, kSiteSFull = 25, kSitePFull = 26,
    kSiteMma34 = 27, kSiteDqFull = 28, kSiteDqEmpty = 29, kSiteAccFull = 30, kSiteAccEmpty = 31, kSiteVec = 32,
    kSiteDrain = 33, kSiteStaged = 34
};

struct BwdParams {
    const float *lse;     // [B, Hq, Nq] natural-log LSE of the forward
    const float *delta;   // [B, Hq, Nq] D_i = dO_i . O_i
    float *dq_acc;        // [B, Nq, Hq, d] fp32, zeroed before the kernel
    uint16_t *dk, *dv;    // [B, Nk, Hkv, d] bf16 bits
    int *status;
    int B, Hq, Hkv, Nq, Nk, n_rep, causal;
    int window;           // 0, or W >= 1: sliding window of the W keys ending at the causal diagonal
    int nkt, nqt;         // key tiles, query tiles (of 128 rows)
    int num_units;        // B * Hkv * nkt
    float scale, scale_log2;
};

template <int D_, bool F16_ = false>
struct BwdCfg {
    static constexpr int D = D_;
    static constexpr bool F16 = F16_;                 // fp16 Q, K, V, O, dO and gradients, else bf16
    static constexpr int CW = (D == 32) ? 32 : 64;    // elements per swizzled row of a Q/K/V/dO tile
    static constexpr int RB = CW * 2;                 // bytes per swizzled row (64 or 128)
    static constexpr uint32_t LAYOUT = (RB == 128) ? 2u : 4u;   // UMMA 128-byte / 64-byte swizzle
    static constexpr int SBO = 8 * RB;                // 8-row swizzle atom
    static constexpr int NCH = (D + CW - 1) / CW;     // column chunks of a [128 x D] tile (the last
                                                      // one zero-filled past d for d = 80, 96)
    static constexpr int CHUNK = kRows * RB;          // one chunk of a 128-row tile
    static constexpr int TILE = NCH * CHUNK;          // [128 x D] tile
    static constexpr int DS_RB = 128, DS_CHUNK = kRows * DS_RB;  // dS^T: 128 queries, 128-byte swizzle
    static constexpr int DCH = (D + 31) / 32;         // 32-column TMEM chunks of a D-wide row
    static constexpr int NQS = 2;                     // Q / dO slots
    static constexpr int SMEM_K = 0;
    static constexpr int SMEM_V = TILE;
    static constexpr int SMEM_Q = 2 * TILE;
    static constexpr int SMEM_DO = SMEM_Q + NQS * TILE;
    static constexpr int SMEM_DS = SMEM_DO + NQS * TILE;     // dS^T: two 64-query chunks
    static constexpr int SMEM_VEC = SMEM_DS + 2 * DS_CHUNK;  // (L log2e, D) x 128 floats
    static constexpr int SMEM_BAR = SMEM_VEC + 2 * kRows * 4;
    // barriers
    static constexpr int B_KV_FULL = 0, B_KV_EMPTY = 1, B_Q_FULL = 2, B_Q_EMPTY = B_Q_FULL + NQS,
                         B_S_FULL = B_Q_EMPTY + NQS, B_P_FULL = B_S_FULL + 1, B_MMA34 = B_P_FULL + 1,
                         B_DQ_FULL = B_MMA34 + 1, B_DQ_EMPTY = B_DQ_FULL + 1, B_ACC_FULL = B_DQ_EMPTY + 1,
                         B_ACC_EMPTY = B_ACC_FULL + 1, B_VEC = B_ACC_EMPTY + 1, B_DRAIN = B_VEC + 1,
                         B_P_HALF = B_DRAIN + 1,   // P^T, dS^T of the first 64 queries in TMEM
                         B_STAGED = B_P_HALF + 1,  // all 128 dQ rows of a step staged
                         NUM_BARS = B_STAGED + 1;
    // dQ leaves through [64 rows x 32 fp32] boxes (8 KB, 128-byte swizzle) staged in the
    // step's Q slot, then its dO slot (B_Q_EMPTY is arrived once their reductions have
    // read them)
    static constexpr int DQ_BOX = 64 * 128;
    static constexpr int DQ_NBOX = DCH * 2;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    // Each CTA holds all 512 TMEM columns: ask for enough shared memory that a second CTA
    // can never be resident on the same SM (it would only wait in the allocation).
    static constexpr int SMEM_NEEDED = SMEM_MISC + 16 + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEEDED > 120 * 1024 ? SMEM_NEEDED : 120 * 1024;
    // TMEM columns
    static constexpr int COL_A = 0, COL_B = 128, COL_DV = 256, COL_DK = 256 + DCH * 32;
    // dQ of a step: d <= 64 fits the upper half of region A (S^T columns the SG warpgroup has
    // read; P^T uses the lower half), so its MMA need not wait for the dV MMAs to read P^T;
    // larger d take all of region A once they have
    static constexpr bool DQ_UPPER = D <= 64;
    static constexpr int COL_DQ = DQ_UPPER ? COL_A + 64 : COL_A;
    static constexpr int TMEM_COLS = 512;
    // warps: 0 TMA, 1 MMA, 2-3 idle, 4-7 SG, 8-11 DW
    static constexpr int THREADS = 384;
    static constexpr int SG_WARP0 = 4, DW_WARP0 = 8;
    static constexpr uint32_t IDESC_SS = sm100::idesc_f16kind_f32(kRows, kRows, 0, 0, F16);
    static constexpr uint32_t IDESC_TS = sm100::idesc_f16kind_f32(kRows, D, 0, 1, F16);
    static constexpr uint32_t IDESC_DQ = sm100::idesc_f16kind_f32(kRows, D, 1, 1, F16);

    static_assert(D % 16 == 0 && D >= 32 && D <= 128, "backward head dims: MMA N granularity, TMEM budget");
    static_assert(COL_DK + DCH * 32 <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_DS % 1024 == 0, "dS^T needs 1024-byte alignment (128-byte swizzle atoms)");
    static_assert(DQ_NBOX * DQ_BOX <= 2 * TILE && TILE % DQ_BOX == 0, "dQ staging fits the Q and dO slots");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Unit {
    int b, kvh, kt, i_lo, i_hi, nsteps;   // query tiles [i_lo, i_hi) see the key tile
};

__device__ __forceinline__ Unit decode_unit(int u, const BwdParams &p) {
    Unit w;
    const int bh = p.B * p.Hkv;
    int r;
    if (p.causal) {   // key tile 0 first: it has the most query tiles
        w.kt = u / bh;
        r = u - w.kt * bh;
    } else {          // the key tiles of one head adjacent: they share Q and dO through L2
        r = u / p.nkt;
        w.kt = u - r * p.nkt;
    }
    w.b = r / p.Hkv;
    w.kvh = r - w.b * p.Hkv;
    w.i_lo = 0;
    w.i_hi = p.nqt;
    const int diag = p.Nk - p.Nq;
    if (p.causal) {   // first query tile whose last row sees key k0 = kt * 128
        const int x = w.kt * kRows - diag;
        w.i_lo = x > 0 ? x / kRows : 0;
        if (w.i_lo > p.nqt) w.i_lo = p.nqt;
    }
    if (p.window > 0) {   // query q sees key k only if q < k - diag + W: the tile's last key bounds it
        const long long q_end = (long long)w.kt * kRows + (kRows - 1) - diag + p.window;   // exclusive
        const long long t_end = q_end <= 0 ? 0 : (q_end + kRows - 1) / kRows;
        if (t_end < w.i_hi) w.i_hi = int(t_end);
        if (w.i_hi < w.i_lo) w.i_hi = w.i_lo;
    }
    w.nsteps = p.n_rep * (w.i_hi - w.i_lo);
    return w;
}

// The static schedule: in pass r the CTAs take units r * G .. r * G + G - 1 (G = gridDim.x),
// CTA i unit r * G + i in even passes and r * G + G - 1 - i in odd ones.  The causal order
// puts the key tiles with the most query tiles first, so alternating the direction pairs the
// CTAs that drew the longest units of one pass with the shortest of the next (the busiest
// CTA 1.6 % above the mean on the causal GQA 4K workload, where a plain stride left it 13.7 %
// above).  Every role walks the same sequence; an index past the end is skipped by all.
__device__ __forceinline__ int sched_unit(int r) {
    const int g = int(gridDim.x), i = int(blockIdx.x);
    return r * g + ((r & 1) ? g - 1 - i : i);
}

// step s of a unit -> (query head, query tile)
__device__ __forceinline__ void step_of(const Unit &w, int s, const BwdParams &p, int &hq, int &it) {
    const int per_head = w.i_hi - w.i_lo;
    const int r = s / per_head;
    hq = w.kvh * p.n_rep + r;
    it = w.i_lo + (s - r * per_head);
}

struct Ctl {
    volatile int *abort_flag;
    int *status;
};

__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, const Ctl &ctl, int site, bool drain = false,
                                          uint64_t limit_ns = 1000000000ull) {
    const uint64_t t0 = sm100::global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (sm100::mbar_try_wait(bar, parity)) return true;
        if (!drain && *ctl.abort_flag) return false;
        if (sm100::global_timer_ns() - t0 > limit_ns) {
            *ctl.abort_flag = 1;
            atomicCAS(ctl.status, 0, 6 | (site << 8) | (min(int(blockIdx.x), 0xFFFF) << 16));
            return false;
        }
    }
}

// Warp-uniform bounded wait.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Ctl &ctl, int site) {
    bool ok = sm100::mbar_try_wait(bar, parity) || wait_slow(bar, parity, ctl, site);
    const bool all = __all_sync(0xffffffffu, ok);
    if (!all) *ctl.abort_flag = 1;
    return all;
}

// Two 32-column TMEM loads of this thread's lane (a from ta, b from tb) behind one wait.
#define FA_BWD_R8(a, i) "=r"(a[i]), "=r"(a[i + 1]), "=r"(a[i + 2]), "=r"(a[i + 3]), "=r"(a[i + 4]), "=r"(a[i + 5]), \
                        "=r"(a[i + 6]), "=r"(a[i + 7])
__device__ __forceinline__ void tmem_ld32x2_sync(uint32_t ta, uint32_t (&a)[32], uint32_t tb, uint32_t (&b)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : FA_BWD_R8(a, 0), FA_BWD_R8(a, 8), FA_BWD_R8(a, 16), FA_BWD_R8(a, 24), FA_BWD_R8(b, 0), FA_BWD_R8(b, 8),
          FA_BWD_R8(b, 16), FA_BWD_R8(b, 24)
        : "r"(ta), "r"(tb)
        : "memory");
}
#undef FA_BWD_R8

// 16 consecutive TMEM columns of this thread's lane from registers (not yet waited on).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Element-wise add of a [64 rows x 32 fp32] shared-memory box (128-byte swizzle) into the
// tensor at (x, y, z, w) of `map`, tracked by this thread's bulk-async group.
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap *map, uint32_t src, int x, int y, int z, int w) {
    asm volatile("cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the tensor core.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMA producer (warp 0)

template <class C>
__device__ void producer(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                         const CUtensorMap *tm_do, const BwdParams &p, uint32_t sbase, const Ctl &ctl) {
    auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
    uint32_t n_kv = 0, n_q = 0;   // loads issued
    bool ok = true;
    for (int r_ = 0; ok && r_ * int(gridDim.x) < p.num_units; ++r_) {
        const int u = sched_unit(r_);
        if (u >= p.num_units) continue;
        const Unit w = decode_unit(u, p);
        if (w.nsteps == 0) continue;
        if (n_kv > 0 && !warp_wait(bar(C::B_KV_EMPTY), (n_kv - 1) & 1u, ctl, kSiteKvEmpty)) { ok = false; break; }
        sm100::mbar_arrive_expect_tx_elected(bar(C::B_KV_FULL), 2 * C::TILE);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
            sm100::tma_load_4d_elected(sbase + C::SMEM_K + c * C::CHUNK, tm_k, bar(C::B_KV_FULL), c * C::CW, w.kvh,
                                       w.kt * kRows, w.b);
            sm100::tma_load_4d_elected(sbase + C::SMEM_V + c * C::CHUNK, tm_v, bar(C::B_KV_FULL), c * C::CW, w.kvh,
                                       w.kt * kRows, w.b);
        }
        ++n_kv;
        for (int s = 0; s < w.nsteps; ++s) {
            int hq, it;
            step_of(w, s, p, hq, it);
            const int slot = int(n_q % C::NQS);
            if (n_q >= uint32_t(C::NQS) &&
                !warp_wait(bar(C::B_Q_EMPTY + slot), ((n_q / C::NQS) - 1u) & 1u, ctl, kSiteQEmpty)) {
                ok = false;
                break;
            }
            const uint32_t fb = bar(C::B_Q_FULL + slot);
            sm100::mbar_arrive_expect_tx_elected(fb, 2 * C::TILE);
#pragma unroll
            for (int c = 0; c < C::NCH; ++c) {
                sm100::tma_load_4d_elected(sbase + C::SMEM_Q + slot * C::TILE + c * C::CHUNK, tm_q, fb, c * C::CW, hq,
                                           it * kRows, w.b);
                sm100::tma_load_4d_elected(sbase + C::SMEM_DO + slot * C::TILE + c * C::CHUNK, tm_do, fb, c * C::CW,
                                           hq, it * kRows, w.b);
            }
            ++n_q;
        }
    }
    // Before the CTA can exit, every load issued must have landed.
    if (n_kv > 0) wait_slow(bar(C::B_KV_FULL), (n_kv - 1) & 1u, ctl, kSiteDrain, true, 100000000ull);
    for (uint32_t n = n_q > uint32_t(C::NQS) ? n_q - C::NQS : 0u; n < n_q; ++n)
        wait_slow(bar(C::B_Q_FULL + int(n % C::NQS)), (n / C::NQS) & 1u, ctl, kSiteDrain, true, 100000000ull);
}

// ------------------------------------------------------------------ MMA issuer (warp 1)

template <class C>
__device__ void mma_issuer(const BwdParams &p, uint32_t sbase, uint32_t tmem, const Ctl &ctl) {
    auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
    // K-major descriptors (reduction over d): 16 elements = 32 bytes per k-slice inside a
    // C::CW-column chunk, chunks C::CHUNK bytes apart.
    auto kmaj = [&](uint32_t addr) { return sm100::opaque(sm100::smem_desc(addr, 16, C::SBO, C::LAYOUT)); };
    // M/N-major descriptors (reduction over the 128 rows): 16 rows = 16 * C::RB bytes per
    // k-slice, the column chunks C::CHUNK bytes apart (leading byte offset).
    auto mnmaj = [&](uint32_t addr) { return sm100::opaque(sm100::smem_desc(addr, C::CHUNK, C::SBO, C::LAYOUT)); };
    uint32_t n_step = 0, n_unit = 0;
    bool ok = true;
    for (int r_ = 0; ok && r_ * int(gridDim.x) < p.num_units; ++r_) {
        const int u = sched_unit(r_);
        if (u >= p.num_units) continue;
        const Unit w = decode_unit(u, p);
        if (w.nsteps == 0) continue;
        if (!warp_wait(bar(C::B_KV_FULL), n_unit & 1u, ctl, kSiteKvFull)) { ok = false; break; }
        const uint64_t k_km = kmaj(sbase + C::SMEM_K), v_km = kmaj(sbase + C::SMEM_V);
        const uint64_t k_mn = mnmaj(sbase + C::SMEM_K);
        const uint64_t ds_mn = sm100::opaque(sm100::smem_desc(sbase + C::SMEM_DS, C::DS_CHUNK, 1024, 2));
        for (int s = 0; s < w.nsteps; ++s, ++n_step) {
            const int slot = int(n_step % C::NQS);
            if (!warp_wait(bar(C::B_Q_FULL + slot), (n_step / C::NQS) & 1u, ctl, kSiteQFull)) { ok = false; break; }
            // region A is free once DW has read the previous step's dQ out of it
            if (n_step > 0 && !warp_wait(bar(C::B_DQ_EMPTY), (n_step - 1u) & 1u, ctl, kSiteDqEmpty)) { ok = false; break; }
            sm100::tc_fence_after_sync();
            const uint32_t q_addr = sbase + C::SMEM_Q + slot * C::TILE, do_addr = sbase + C::SMEM_DO + slot * C::TILE;
            const uint64_t q_km = kmaj(q_addr), do_km = kmaj(do_addr), q_mn = mnmaj(q_addr), do_mn = mnmaj(do_addr);
#pragma unroll
            for (int kk = 0; kk < C::D / 16; ++kk) {   // S^T = K Q^T, dP^T = V dO^T
                const uint32_t off = uint32_t(((kk * 16) / C::CW) * C::CHUNK + ((kk * 16) % C::CW) * 2) >> 4;
                sm100::mma_bf16_ss_elected(tmem + C::COL_A, k_km + off, q_km + off, C::IDESC_SS, kk > 0 ? 1u : 0u);
                sm100::mma_bf16_ss_elected(tmem + C::COL_B, v_km + off, do_km + off, C::IDESC_SS, kk > 0 ? 1u : 0u);
            }
            sm100::tc_commit_elected(bar(C::B_S_FULL));
            // dV += P^T dO, dK += dS^T Q over the step's queries: the first 64 as soon as the
            // SG warpgroup has written them, the rest once it has finished
            if (!warp_wait(bar(C::B_P_HALF), n_step & 1u, ctl, kSitePFull)) { ok = false; break; }
            if (s == 0 && n_unit > 0 && !warp_wait(bar(C::B_ACC_EMPTY), (n_unit - 1u) & 1u, ctl, kSiteAccEmpty)) {
                ok = false;
                break;
            }
            for (int half = 0; half < 2; ++half) {
                if (half == 1 && !warp_wait(bar(C::B_P_FULL), n_step & 1u, ctl, kSitePFull)) { ok = false; break; }
                sm100::tc_fence_after_sync();
#pragma unroll
                for (int k4 = 0; k4 < kRows / 32; ++k4) {
                    const int kk = half * (kRows / 32) + k4;
                    const uint32_t boff = uint32_t(kk * 16 * C::RB) >> 4;
                    const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
                    sm100::mma_bf16_ts_elected(tmem + C::COL_DV, tmem + C::COL_A + uint32_t(kk * 8), do_mn + boff,
                                               C::IDESC_TS, acc);
                    sm100::mma_bf16_ts_elected(tmem + C::COL_DK, tmem + C::COL_B + uint32_t(kk * 8), q_mn + boff,
                                               C::IDESC_TS, acc);
                }
            }
            if (!ok) break;
            if constexpr (!C::DQ_UPPER) sm100::tc_commit_elected(bar(C::B_MMA34));
            if (s == w.nsteps - 1) sm100::tc_commit_elected(bar(C::B_ACC_FULL));
            // dQ over all of region A: wait until the dV MMAs have read P^T from it
            if constexpr (!C::DQ_UPPER) {
                if (!warp_wait(bar(C::B_MMA34), n_step & 1u, ctl, kSiteMma34)) { ok = false; break; }
                sm100::tc_fence_after_sync();
            }
#pragma unroll
            for (int kk = 0; kk < kRows / 16; ++kk) {   // dQ = dS K
                const uint32_t a_off = uint32_t(kk * 16 * C::DS_RB) >> 4, b_off = uint32_t(kk * 16 * C::RB) >> 4;
                sm100::mma_bf16_ss_elected(tmem + C::COL_DQ, ds_mn + a_off, k_mn + b_off, C::IDESC_DQ, kk > 0 ? 1u : 0u);
            }
            sm100::tc_commit_elected(bar(C::B_DQ_FULL));
        }
        if (!ok) break;
        sm100::tc_commit_elected(bar(C::B_KV_EMPTY));
        ++n_unit;
    }
    // Every MMA this warp issued is complete before the CTA may free TMEM.
    sm100::tc_commit_elected(bar(C::B_DRAIN));
    wait_slow(bar(C::B_DRAIN), 0u, ctl, kSiteDrain, true);
}

// ------------------------------------------------------------------ SG: P, dS (warps 4-7)

template <class C>
__device__ void sg_role(const BwdParams &p, uint32_t sbase, uint8_t *smem, uint32_t tmem, const Ctl &ctl, int warp,
                        int lane) {
    auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
    const int r = (warp % 4) * 32 + lane;                  // key row of the tile = TMEM lane
    const uint32_t lane_off = uint32_t((warp % 4) * 32) << 16;
    float *vec = reinterpret_cast<float *>(smem + C::SMEM_VEC);
    const int diag = p.Nk - p.Nq;
    uint32_t n_step = 0;
    for (int r_ = 0; r_ * int(gridDim.x) < p.num_units; ++r_) {
        const int u = sched_unit(r_);
        if (u >= p.num_units) continue;
        const Unit w = decode_unit(u, p);
        const int key = w.kt * kRows + r;
        for (int s = 0; s < w.nsteps; ++s, ++n_step) {
            int hq, it;
            step_of(w, s, p, hq, it);
            const int i0 = it * kRows;
            // this step's L log2e and D, one column per thread, through shared memory; the
            // buffer is refilled once every SG thread is done with the previous step
            if (n_step > 0 && !warp_wait(bar(C::B_P_FULL), (n_step - 1u) & 1u, ctl, kSitePFull)) goto unwind;
            {
                const int q = i0 + r;
                float l2 = INFINITY, dv = 0.f;
                if (q < p.Nq) {
                    const size_t off = (size_t(w.b) * p.Hq + hq) * p.Nq + q;
                    const float l = p.lse[off];
                    l2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
                    dv = p.delta[off];
                }
                vec[r] = l2;
                vec[kRows + r] = dv;
                sm100::mbar_arrive(bar(C::B_VEC));
            }
            if (!warp_wait(bar(C::B_VEC), n_step & 1u, ctl, kSiteVec)) goto unwind;
            if (!warp_wait(bar(C::B_S_FULL), n_step & 1u, ctl, kSiteSFull)) goto unwind;
            sm100::tc_fence_after_sync();
            {
                const float *l2v = vec;
                const float *dvv = l2v + kRows;
                // key visible to query q iff key < Nk, q < Nq and (causal) key <= q + diag
                const int q_lim = p.Nq - i0;                         // local query bound
                const int key_lo_q = p.causal ? key - diag - i0 : -0x7fffffff;   // first local q seeing key
                // sliding window: local queries q < key - diag + W - i0 still see the key
                const int key_hi_q = p.window > 0 ? key - diag + p.window - i0 : 0x7fffffff;
                const bool key_ok = key < p.Nk;
                uint8_t *ds_row = smem + C::SMEM_DS + r * C::DS_RB;
#pragma unroll 1
                for (int c = 0; c < kRows / 32; ++c) {
                    uint32_t sv[32], dp[32];
                    if constexpr (C::D < 128) {   // both loads behind one wait (d = 128: the
                                                  // extra live registers cost more than it saves)
                        tmem_ld32x2_sync(tmem + lane_off + uint32_t(C::COL_A + 32 * c), sv,
                                         tmem + lane_off + uint32_t(C::COL_B + 32 * c), dp);
                    } else {
                        sm100::tmem_ld32_sync(tmem + lane_off + uint32_t(C::COL_A + 32 * c), sv);
                        sm100::tmem_ld32_sync(tmem + lane_off + uint32_t(C::COL_B + 32 * c), dp);
                    }
                    uint32_t pk[16], dk[16];
                    // the chunk's 32 queries all see this thread's key (most chunks): no
                    // per-element test when that holds for the whole warp
                    const int q0 = 32 * c;
                    const bool full = key_ok && q0 + 32 <= q_lim && q0 >= key_lo_q && q0 + 32 <= key_hi_q;
                    const bool warp_full = __all_sync(0xffffffffu, full);
                    // L log2e and D of the chunk's queries: broadcast 16-byte shared loads
                    const float4 *l2v4 = reinterpret_cast<const float4 *>(l2v + q0);
                    const float4 *dvv4 = reinterpret_cast<const float4 *>(dvv + q0);
                    // two straight-line copies of the loop (no branch per element, so the
                    // 32 exponentials of a chunk can overlap)
                    auto chunk = [&](auto masked) {
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const float4 l4 = l2v4[e4], d4 = dvv4[e4];
                            float pr[4], dsr[4];
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const int e = 4 * e4 + h;
                                const float lq = h == 0 ? l4.x : h == 1 ? l4.y : h == 2 ? l4.z : l4.w;
                                const float dq = h == 0 ? d4.x : h == 1 ? d4.y : h == 2 ? d4.z : d4.w;
                                const float x = fmaf(__uint_as_float(sv[e]), p.scale_log2, -lq);
                                float pv;
                                if constexpr (decltype(masked)::value) {
                                    const int ql = q0 + e;
                                    const bool vis = key_ok && ql < q_lim && ql >= key_lo_q && ql < key_hi_q;
                                    pv = vis ? sm100::ex2_approx(x) : 0.f;
                                } else {
                                    pv = sm100::ex2_approx(x);
                                }
                                pr[h] = pv;
                                dsr[h] = pv * (__uint_as_float(dp[e]) - dq);
                            }
                            pk[2 * e4] = sm100::pack_x2<C::F16>(pr[0], pr[1]);
                            pk[2 * e4 + 1] = sm100::pack_x2<C::F16>(pr[2], pr[3]);
                            dk[2 * e4] = sm100::pack_x2<C::F16>(dsr[0], dsr[1]);
                            dk[2 * e4 + 1] = sm100::pack_x2<C::F16>(dsr[2], dsr[3]);
                        }
                    };
                    if (warp_full) chunk(std::false_type{});
                    else chunk(std::true_type{});
                    tmem_st16(tmem + lane_off + uint32_t(C::COL_A + 16 * c), pk);
                    tmem_st16(tmem + lane_off + uint32_t(C::COL_B + 16 * c), dk);
                    // dS^T row r, queries 32c .. 32c+31: chunk c/2, 16-byte units (c%2)*4 .. +3,
                    // 128-byte swizzle (unit index XOR row % 8)
                    uint8_t *chunk_row = ds_row + (c / 2) * C::DS_CHUNK;
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const int unit = ((c % 2) * 4 + v4) ^ (r & 7);
                        *reinterpret_cast<uint4 *>(chunk_row + unit * 16) =
                            make_uint4(dk[4 * v4], dk[4 * v4 + 1], dk[4 * v4 + 2], dk[4 * v4 + 3]);
                    }
                    if (c == 1) {   // the first 64 queries' P^T and dS^T are in TMEM
                        sm100::tmem_st_wait();
                        sm100::tc_fence_before_sync();
                        sm100::mbar_arrive(bar(C::B_P_HALF));
                    }
                }
            }
            sm100::tmem_st_wait();
            fence_proxy_async_smem();
            sm100::tc_fence_before_sync();
            sm100::mbar_arrive(bar(C::B_P_FULL));
        }
    }
unwind:
    sm100::tmem_st_wait();
}

// ------------------------------------------------------------------ DW: dQ, dK, dV out (warps 8-11)

template <class C>
__device__ void dw_role(const BwdParams &p, const CUtensorMap *tm_dq, uint32_t sbase, uint8_t *smem, uint32_t tmem,
                        const Ctl &ctl, int warp, int lane) {
    auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
    const int r = (warp % 4) * 32 + lane;
    const uint32_t lane_off = uint32_t((warp % 4) * 32) << 16;
    const bool issuer = warp == C::DW_WARP0;   // this warp's lane 0 issues the reductions
    // staging box bi of a slot: the Q slot's bytes first, then the dO slot's
    auto box_off = [&](int slot, int bi) -> int {
        const int off = bi * C::DQ_BOX;
        return off < C::TILE ? C::SMEM_Q + slot * C::TILE + off : C::SMEM_DO + slot * C::TILE + (off - C::TILE);
    };
    uint32_t n_step = 0, n_unit = 0;
    for (int r_ = 0; r_ * int(gridDim.x) < p.num_units; ++r_) {
        const int u = sched_unit(r_);
        if (u >= p.num_units) continue;
        const Unit w = decode_unit(u, p);
        const int key = w.kt * kRows + r;
        const size_t kv_row = (size_t(w.b) * p.Nk + size_t(key)) * p.Hkv + w.kvh;
        if (w.nsteps == 0) {   // no query sees this key tile: dK = dV = 0
            if (key < p.Nk)
                for (int c = 0; c < C::D; c += 8) {
                    *reinterpret_cast<uint4 *>(p.dk + kv_row * C::D + c) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(p.dv + kv_row * C::D + c) = make_uint4(0u, 0u, 0u, 0u);
                }
            continue;
        }
        for (int s = 0; s < w.nsteps; ++s, ++n_step) {
            int hq, it;
            step_of(w, s, p, hq, it);
            const int q = it * kRows + r;
            if (!warp_wait(bar(C::B_DQ_FULL), n_step & 1u, ctl, kSiteDqFull)) goto done;
            sm100::tc_fence_after_sync();
            (void)q;
            // the whole dQ row into registers first, so region A is free for the next
            // step's S^T while the reductions run
            uint32_t v[C::DCH * 32];
#pragma unroll
            for (int c = 0; c < C::DCH; ++c)
                sm100::tmem_ld32_sync(tmem + lane_off + uint32_t(C::COL_DQ + 32 * c),
                                      *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
            sm100::tc_fence_before_sync();
            sm100::mbar_arrive(bar(C::B_DQ_EMPTY));
            // stage the row (its MMAs are complete, so the step's Q and dO slots are free):
            // row r of box (c, r / 64), 128-byte swizzle (16-byte unit index XOR row % 8)
            const int slot = int(n_step % C::NQS);
#pragma unroll
            for (int c = 0; c < C::DCH; ++c) {
                uint8_t *row = smem + box_off(slot, 2 * c + r / 64) + (r % 64) * 128;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<uint4 *>(row + ((u ^ (r & 7)) * 16)) =
                        make_uint4(v[32 * c + 4 * u], v[32 * c + 4 * u + 1], v[32 * c + 4 * u + 2], v[32 * c + 4 * u + 3]);
            }
            fence_proxy_async_smem();
            sm100::mbar_arrive(bar(C::B_STAGED));
            if (issuer) {
                if (!warp_wait(bar(C::B_STAGED), n_step & 1u, ctl, kSiteStaged)) goto done;
                if (lane == 0) {
                    // rows past Nq and columns past d fall outside the tensor and are skipped;
                    // a box that starts past Nq is not issued
#pragma unroll
                    for (int bi = 0; bi < C::DQ_NBOX; ++bi) {
                        const int row0 = it * kRows + (bi % 2) * 64;
                        if (row0 < p.Nq)
                            tma_reduce_add_4d(tm_dq, sbase + box_off(slot, bi), (bi / 2) * 32, hq, row0, w.b);
                    }
                    bulk_commit();
                    bulk_wait_read_all();
                    sm100::mbar_arrive(bar(C::B_Q_EMPTY + slot));   // the slot back to the producer
                }
                __syncwarp();
            }
        }
        if (!warp_wait(bar(C::B_ACC_FULL), n_unit & 1u, ctl, kSiteAccFull)) goto done;
        sm100::tc_fence_after_sync();
#pragma unroll 1
        for (int c = 0; c < C::DCH; ++c) {
            uint32_t dv[32], dk[32];
            sm100::tmem_ld32_sync(tmem + lane_off + uint32_t(C::COL_DV + 32 * c), dv);
            sm100::tmem_ld32_sync(tmem + lane_off + uint32_t(C::COL_DK + 32 * c), dk);
            if (key < p.Nk) {
                uint32_t pv[16], pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    pv[i] = sm100::pack_x2<C::F16>(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1]));
                    pk[i] = sm100::pack_x2<C::F16>(__uint_as_float(dk[2 * i]) * p.scale,
                                                   __uint_as_float(dk[2 * i + 1]) * p.scale);
                }
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4) {
                    if (32 * c + 8 * v4 >= C::D) break;   // d = 80, 96: the last chunk is partial
                    *reinterpret_cast<uint4 *>(p.dv + kv_row * C::D + 32 * c + 8 * v4) =
                        make_uint4(pv[4 * v4], pv[4 * v4 + 1], pv[4 * v4 + 2], pv[4 * v4 + 3]);
                    *reinterpret_cast<uint4 *>(p.dk + kv_row * C::D + 32 * c + 8 * v4) =
                        make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                }
            }
        }
        sm100::tc_fence_before_sync();
        sm100::mbar_arrive(bar(C::B_ACC_EMPTY));
        ++n_unit;
    }
done:
    if (issuer && lane == 0) bulk_wait_all();   // every reduction has landed before the CTA exits
}

// ------------------------------------------------------------------ kernels

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sm100::smem_u32(smem);
    const int warp = int(threadIdx.x) / 32;
    const int lane = int(threadIdx.x) % 32;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::SMEM_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::SMEM_MISC + 4);
    const Ctl ctl{abort_flag, p.status};

    if (threadIdx.x == 0) {
        auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
        sm100::mbar_init(bar(C::B_KV_FULL), 1);
        sm100::mbar_init(bar(C::B_KV_EMPTY), 1);
        for (int s = 0; s < C::NQS; ++s) {
            sm100::mbar_init(bar(C::B_Q_FULL + s), 1);
            sm100::mbar_init(bar(C::B_Q_EMPTY + s), 1);
        }
        sm100::mbar_init(bar(C::B_S_FULL), 1);
        sm100::mbar_init(bar(C::B_P_FULL), kRows);
        sm100::mbar_init(bar(C::B_P_HALF), kRows);
        sm100::mbar_init(bar(C::B_STAGED), kRows);
        sm100::mbar_init(bar(C::B_MMA34), 1);
        sm100::mbar_init(bar(C::B_DQ_FULL), 1);
        sm100::mbar_init(bar(C::B_DQ_EMPTY), kRows);
        sm100::mbar_init(bar(C::B_ACC_FULL), 1);
        sm100::mbar_init(bar(C::B_ACC_EMPTY), kRows);
        sm100::mbar_init(bar(C::B_VEC), kRows);
        sm100::mbar_init(bar(C::B_DRAIN), 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
    }
    if (warp == 0) {
        sm100::tmem_alloc(sm100::smem_u32(tmem_holder), C::TMEM_COLS);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before_sync();
    __syncthreads();
    sm100::tc_fence_after_sync();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        producer<C>(&tm_q, &tm_k, &tm_v, &tm_do, p, sbase, ctl);
    } else if (warp == 1) {
        mma_issuer<C>(p, sbase, tmem, ctl);
    } else if (warp >= C::SG_WARP0 && warp < C::SG_WARP0 + 4) {
        sg_role<C>(p, sbase, smem, tmem, ctl, warp, lane);
    } else if (warp >= C::DW_WARP0 && warp < C::DW_WARP0 + 4) {
        dw_role<C>(p, &tm_dq, sbase, smem, tmem, ctl, warp, lane);
    }
    __syncwarp();

    sm100::tc_fence_before_sync();
    __syncthreads();
    sm100::tc_fence_after_sync();
    if (warp == 0) sm100::tmem_dealloc(tmem, C::TMEM_COLS);
}

// D_i = dO_i . O_i in fp32 (one warp per row) and a zeroed dQ accumulator.
template <bool F16>
__device__ __forceinline__ float elem_to_f32(uint16_t bits) {
    if constexpr (F16) return __half2float(__ushort_as_half(bits));
    else return __uint_as_float(uint32_t(bits) << 16);
}

template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const uint16_t *out, const uint16_t *dout, float *delta,
                                                         float *dq_acc, int B, int Hq, int Nq) {
    const long rows = long(B) * Nq * Hq;
    const int lane = int(threadIdx.x) % 32;
    for (long r = (long(blockIdx.x) * blockDim.x + threadIdx.x) / 32; r < rows;
         r += long(gridDim.x) * blockDim.x / 32) {
        float acc = 0.f;
        for (int c = lane; c < D; c += 32) {
            const float o = elem_to_f32<F16>(out[r * D + c]);
            const float g = elem_to_f32<F16>(dout[r * D + c]);
            acc = fmaf(o, g, acc);
            dq_acc[r * D + c] = 0.f;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) {
            const int hq = int(r % Hq);
            const long bi = r / Hq;   // b * Nq + i
            const int i = int(bi % Nq);
            const int b = int(bi / Nq);
            delta[(long(b) * Hq + hq) * Nq + i] = acc;
        }
    }
}

// dQ = bf16 (fp16) of scale * acc
template <bool F16>
__global__ void fa_bwd_post_kernel(const float4 *acc, uint2 *dq, size_t n4, float scale) {
    const size_t stride = size_t(gridDim.x) * blockDim.x;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 a = acc[i];
        dq[i] = make_uint2(sm100::pack_x2<F16>(a.x * scale, a.y * scale), sm100::pack_x2<F16>(a.z * scale, a.w * scale));
    }
}

}  // namespace bwd
}  // namespace fa

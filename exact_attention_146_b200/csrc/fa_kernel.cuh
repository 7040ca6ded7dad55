// fa_kernel.cuh -- persistent sm_100a kernel for the exact attention forward.
//
// The method is the tiled FlashAttention forward described on the hwcomputing.csdn.net
// article "FlashAttention in CANN ops-transformer": Q is cut into row blocks, K/V into
// column blocks; for each Q block the K/V blocks stream through on-chip memory while a
// running row max m and running sum l keep the softmax exact (section "online
// softmax"), scale and mask are fused into the same pass (section "fusion"), the next
// block is fetched while the current one is computed (section "double buffering"), and
// the output is divided by l once at the end.
//
// How it maps onto a B200 SM (one CTA per SM, persistent over work units):
//   * work unit = (batch b, query head hq, block of NQT x 128 query rows; with GQA
//     packing the n_rep heads of one KV head share a unit, their rows stacked; with a
//     causal or window mask and GQA, the NQT tiles are NQT query heads of one KV head over
//     the same 128 rows; with split-KV or a key-shard partial, also a slice of the key
//     tiles); units are taken in a static snake order (sched_unit);
//   * TMA warp (one thread): Q tiles once per unit, then K_j, V_j into an NS-slot
//     shared-memory ring guarded by full/empty mbarriers;
//   * MMA warp (one thread): S_t = Q_t K_j^T with tcgen05.mma into TMEM (fp32), and
//     O_t += P_t V_j with P read straight from TMEM (it overwrites S_t as bf16 / fp16 /
//     E4M3, or has columns of its own);
//     the two query tiles are interleaved so that one tile's softmax runs while the
//     tensor core works on the other tile.  At d = 80 ... 192 (and E4M3 at d = 64, 128) the
//     two tiles share ONE S buffer and P has columns of its own (d = 128: S 128 + O 2 x 128
//     + P 2 x 64 of the 512 TMEM columns): the next S, of either tile, is issued as soon as the
//     softmax that owns the current one has loaded it into registers, so no tile's S
//     waits for its own P V to finish reading P (the softmax instead waits for that P V
//     before it stores the next P);
//   * softmax warpgroup t (128 threads, thread r owns row r of tile t, which is TMEM
//     lane r): loads its row of S_t, masks, takes the row max, p = 2^(s*scale*log2e - m)
//     with one FFMA + ex2 per element, writes P back (in two halves for d <= 80, so the
//     first half of P V overlaps the second half of the exponentials), keeps m and l in
//     registers, rescales its O row in TMEM only when the max grew by more than
//     2^8 (the final O / l is unchanged by the reference max used), and at the end
//     writes O / l (d >= 64: through a per-warp shared-memory box and a TMA store) and
//     LSE = (m + log2 l) ln 2 (split-KV / key shards: fp32 O / l and the slice's LSE to a
//     workspace, combined by fa_splitkv_merge_kernel).
// Every pipeline wait is bounded: after a time limit the kernel records
// FA_ERR_DEVICE_TIMEOUT in a device status word, unwinds every role, waits for its own
// in-flight copies and MMAs, frees TMEM and returns.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace fa {

constexpr int kBlockQ = 128;                          // query rows per tile = TMEM lanes = MMA M
constexpr uint64_t kWaitLimitNs = 1000000000ull;      // 1 s per wait
constexpr float kRescaleLog2 = 8.0f;                  // lazy-rescale threshold (log2 units)
constexpr int kStatusTimeout = 6;                     // = FA_ERR_DEVICE_TIMEOUT

// Which wait gave up (bits 8..15 of the status word).
enum WaitSite : int {
    kSiteQEmpty = 1, kSiteKvEmpty = 2, kSiteKvFull = 3, kSiteQFull = 4, kSitePFull = 5,
    kSiteOEmpty = 6, kSiteSFull = 7, kSiteODone = 8, kSiteDrain = 9, kSiteProducerDrain = 10,
    kSitePvDone = 11, kSiteOFinal = 12, kSiteSEmpty = 13
};

struct FwdParams {
    void *out;            // [B, Nq, Hq, d], bf16 or fp16 (the config's element type)
    float *lse;           // [B, Hq, Nq] or nullptr
    int *status;          // device status word
    int B, Hq, Hkv, Nq, Nk;
    int n_rep;            // Hq / Hkv
    int causal;           // 1 for the causal and the sliding-window masks
    int window;           // 0, or the sliding-window width W (keys i+Nk-Nq-W < j <= i+Nk-Nq)
    int nqb;              // blocks of NQT*128 (flat) rows per (b, head group)
    int pack;             // query heads per unit (GQA packing): 1, or n_rep when the n_rep heads
                          // of one KV head stack their rows into the tile (flat row = i*pack + r)
    int num_splits;       // key-range splits per query block (1: no split)
    int split_tiles;      // key tiles per split
    int num_units;        // B * Hq * nqb * num_splits
    float *o_part;        // num_splits > 1: fp32 partial O [split][B][Nq][Hq][d], normalised
    float *lse_part;      // num_splits > 1: partial LSE [split][B][Hq][Nq]
    float scale_log2;     // scale * log2(e) (FP8: times the Q and K dequantisation factors)
    float o_scale;        // FP8: the V dequantisation factor, applied to O with 1 / l
    int diag;             // causal / window: row i sees keys j <= i + diag (Nk - Nq; for a key
                          // shard at offset o of Nk_total keys, Nk_total - Nq - o)
    int partial;          // 1: write the fp32 normalised O and the LSE of these keys to
                          // o_part / lse_part (a key shard's partial) instead of out / lse
    // Failure-path test instantiation only (TileCfg FAULT): the per-wait limit, and the index
    // (in issue order K_0, V_0, K_1, ...) of one K/V load the producer leaves out, so the wait
    // for it runs out and the kernel takes its timeout path.  Ignored by every other build.
    unsigned long long wait_limit_ns;
    int withheld_load;
    int o_tma;            // 1: the epilogue writes O through shared memory and TMA stores (tm_o)
    int hpair;            // 1: the two query tiles of a unit are two query heads of one KV group
                          // over the same 128 query rows (same keys, so causal tiles end together)
};

// Compile-time tiling for one head dimension.
template <int D_, int BC_, int NQT_, int NS_, int NQB_ = 1, int SB_ = 1, bool PSEP_ = false, int SOFT_EXP_ = 0,
          bool F16_ = false, bool FP8_ = false, bool FAULT_ = false, bool SSHARE_ = false>
struct TileCfg {
    static constexpr int D = D_;        // head dim
    static constexpr int BC = BC_;      // key/value rows per tile
    static constexpr int NQT = NQT_;    // query tiles per unit (1 or 2)
    static constexpr int NS = NS_;      // K/V slots in the ring
    static constexpr int NQB = NQB_;    // buffers per query tile (2: next unit's Q loads early)
    static constexpr int SB = SB_;      // S buffers per query tile (2: S_{j+1} computed during softmax j)
    static constexpr bool PSEP = PSEP_; // P in TMEM columns of its own instead of over S
    static constexpr int SOFT_EXP = SOFT_EXP_;   // exponentials on the FMA pipe: pairs per 8
    static constexpr bool F16 = F16_;   // element type of Q, K, V, P and O: fp16, else bf16
    static constexpr bool FP8 = FP8_;   // Q, K, V and P in OCP E4M3 (kind::f8f6f4); O stays bf16
    static constexpr bool FAULT = FAULT_;   // failure-path test build: wait limit from the
                                            // parameters, one K/V load withheld
    // One S buffer for both query tiles (P in columns of its own): the next S, of either
    // tile, is computed as soon as the softmax that owns the current one has read it into
    // registers, so no tile's S waits for its own P V.  The two tiles' S tiles take turns
    // in the buffer (S_0(j), S_1(j), S_0(j+1), ...).
    static constexpr bool SSHARE = SSHARE_;
    static constexpr int ES = FP8 ? 1 : 2;                // bytes per Q/K/V/P element
    static constexpr int RB = (D * ES >= 128) ? 128 : 64; // bytes per swizzled smem row
    static constexpr int CW = RB / ES;                    // elements per swizzled smem row
    static constexpr int KSTEP = 32 / ES;                 // K elements per MMA (32 bytes)
    static constexpr int PCOLS = BC * ES / 4;             // TMEM columns of one row of P
    // P is handed to the P V MMAs in two 64-key halves: the first half of P V runs while
    // the softmax computes the second half of P.  Worth it where the exponentials dominate
    // (d <= 80: 6-10 % faster); at d >= 96 the extra register pressure costs more than the
    // overlap gains, so the hand-off stays whole there.
    static constexpr bool PSPLIT = (BC == 128) && !FP8 && D <= 80 && !SSHARE;
    static constexpr int NCH = (D + CW - 1) / CW;         // column chunks of a tile
    static constexpr int Q_CHUNK = kBlockQ * RB;
    static constexpr int KV_CHUNK = BC * RB;
    static constexpr int Q_TILE = NCH * Q_CHUNK;
    static constexpr int KV_TILE = NCH * KV_CHUNK;
    static constexpr uint32_t LAYOUT = (RB == 128) ? 2u : 4u;   // UMMA 128B / 64B swizzle
    static constexpr int SBO = 8 * RB;                          // 8-row swizzle atom
    // TMEM columns: S buffer b of tile t at (t*SB + b)*BC (SSHARE: the one S buffer at 0),
    // O_t after the S buffers, and P_t either over the first BC/2 columns of its S buffer
    // or (PSEP) after all O.
    static constexpr int OST = (D == 256) ? 256 : ((D + 63) / 64) * 64;
    static constexpr int O_COL0 = SSHARE ? BC : NQT * SB * BC;
    static constexpr int P_COL0 = O_COL0 + NQT * OST;
    static constexpr int TMEM_COLS = 512;
    static constexpr int O_CHUNKS = (D + 31) / 32;
    // shared memory (offsets from a 1024-byte aligned base)
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_KV = NQT * NQB * Q_TILE;
    static constexpr int SMEM_BAR = SMEM_KV + NS * KV_TILE;
    static constexpr int NUM_BARS = 2 * NS + 2 * NQT * NQB + 4 * NQT * SB + 3 * NQT + 2;
    static constexpr int SMEM_MISC = SMEM_BAR + NUM_BARS * 8;
    // Output staging (d >= 64): each softmax warp writes its 32 rows of O, 64 columns at a
    // time, into 4 KB of its own (128-byte rows, 128-byte swizzle) and stores them with one
    // TMA box, so the epilogue writes whole lines instead of one 16-byte piece per row.
    static constexpr bool OSTAGE = (D >= 64);
    static constexpr int SMEM_OST = ((SMEM_MISC + 16 + 1023) / 1024) * 1024;
    static constexpr int OST_BYTES = OSTAGE ? 32 * 128 : 0;   // per warp
    // Each CTA holds all 512 TMEM columns, so ask for enough shared memory that a
    // second CTA can never be resident on the same SM (it would only wait in alloc).
    static constexpr int SMEM_NEEDED = SMEM_OST + 4 * NQT * OST_BYTES + 1024;
    static constexpr int SMEM_BYTES = SMEM_NEEDED > 120 * 1024 ? SMEM_NEEDED : 120 * 1024;
    // warps: one warpgroup per query tile (softmax), then a control warpgroup holding the
    // TMA warp and the MMA warp (two warps of it idle: register reallocation works on
    // whole warpgroups).
    static constexpr int SOFTMAX_WARPS = 4 * NQT;
    static constexpr int TMA_WARP = SOFTMAX_WARPS;
    static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
    static constexpr int THREADS = 32 * (SOFTMAX_WARPS + 4);
    // Registers per thread: the launch budget (65536 / THREADS rounded down to 8) and,
    // for two query tiles, the split moved from the control warpgroup to the softmax
    // warpgroups.  The control share (88) keeps the MMA issuer's loop free of register
    // spills; the softmax needs no more than 208.  LAUNCH_REGS is checked against the
    // compiled kernel on the host before the first launch.
    static constexpr int LAUNCH_REGS = ((65536 / THREADS) / 8) * 8 > 255 ? 255 : ((65536 / THREADS) / 8) * 8;
    static constexpr bool REALLOC_REGS = (NQT == 2);
    static constexpr int SOFTMAX_REGS = 208;
    static constexpr int CONTROL_REGS = 88;
    static_assert(!REALLOC_REGS || (SOFTMAX_REGS * 32 * SOFTMAX_WARPS + CONTROL_REGS * 128 <= LAUNCH_REGS * THREADS),
                  "register split exceeds the launch budget");
    // format code 0 is F16 under kind::f16 and E4M3 under kind::f8f6f4
    static constexpr uint32_t IDESC_S = sm100::idesc_f16kind_f32(kBlockQ, BC, 0, 0, F16 || FP8);
    static constexpr uint32_t IDESC_O = sm100::idesc_f16kind_f32(kBlockQ, D, 0, 1, F16 || FP8);

    static_assert(NQT == 1 || NQT == 2, "one or two query tiles per unit");
    static_assert(NQB == 1 || NQB == 2, "one or two buffers per query tile");
    static_assert(SB == 1 || SB == 2, "one or two S buffers per query tile");
    static_assert(D % 16 == 0 && D >= 32 && D <= 256, "MMA N and K granularity");
    static_assert(BC % 64 == 0 && BC <= 256, "key tile: whole 32-column TMEM chunks of P");
    static_assert(P_COL0 + (PSEP ? NQT * PCOLS : 0) <= TMEM_COLS, "TMEM budget");
    static_assert(!FP8 || (!F16 && (!PSEP || SSHARE) && SOFT_EXP == 0 && BC % 128 == 0), "FP8 tiling");
    static_assert(!SSHARE || (PSEP && SB == 1 && NQT == 2), "shared S tiling");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    // Barrier indices (Q barriers indexed t * NQB + buffer, S/P barriers t * SB + buffer).
    // Every barrier is waited on densely (each completion in order) by its waiter, except
    // O_DONE, whose rare waits provably trail it by at most one phase; parity waits
    // cannot tell phases two apart.
    static constexpr int B_FULL = 0, B_EMPTY = NS, B_QFULL = 2 * NS, B_QEMPTY = 2 * NS + NQT * NQB,
                         B_SFULL = 2 * NS + 2 * NQT * NQB,   // S_t in buffer b computed
                         B_PFULL = B_SFULL + NQT * SB,       // P_t written over buffer b
                         B_PHALF = B_PFULL + NQT * SB,       // its first 64 keys written (PSPLIT)
                         B_PVDONE = B_PHALF + NQT * SB,      // the P V MMA reading buffer b done
                         B_ODONE = B_PVDONE + NQT * SB,      // a P V MMA of tile t done (rescale; with one S
                                                             // buffer and P over S, PVDONE serves)
                         B_OFINAL = B_ODONE + NQT,           // the last P V of tile t in a unit done
                         B_OEMPTY = B_OFINAL + NQT,          // epilogue finished reading O_t
                         B_DRAIN = B_OEMPTY + NQT,
                         B_SEMPTY = B_DRAIN + 1;             // SSHARE: the S buffer read into registers
};

struct UnitInfo {
    int b, hq, kvh, q0;   // hq: first query head of the unit; q0: first flat row (i*pack + r)
    int js[2], je[2];   // key tiles [js, je) each query tile visits (empty: js == je)
    int j_lo, j_hi;     // union of the ranges: the K/V tiles the unit loads
    int split;          // which key-range split (0 when not split)
};

// Static schedule shared by all roles.  Causal: longest query blocks first, heads of
// one KV group adjacent.  Non-causal: the query blocks of one head adjacent, so the
// CTAs running at the same time share K/V through L2.
template <class C>
__device__ __forceinline__ UnitInfo decode_unit(int u, const FwdParams &p) {
    UnitInfo w;
    w.split = u % p.num_splits;
    u /= p.num_splits;
    const int hstep = p.hpair ? C::NQT : p.pack;   // query heads per unit
    const int groups = p.Hq / hstep;               // head groups (= Hq without packing or pairing)
    const int bh = p.B * groups;
    int qb, r;
    if (p.causal) {
        const int outer = u / bh;
        qb = p.nqb - 1 - outer;
        r = u - outer * bh;
    } else {
        r = u / p.nqb;
        qb = u - r * p.nqb;
    }
    w.b = r / groups;
    w.hq = (r - w.b * groups) * hstep;
    w.kvh = w.hq / p.n_rep;
    w.q0 = qb * (p.hpair ? kBlockQ : C::NQT * kBlockQ);
    const int flat_rows = p.Nq * p.pack;
    const int nkv = (p.Nk + C::BC - 1) / C::BC;
    const int diag = p.diag;         // row i sees keys up to i + diag (causal / window)
    w.j_lo = 0x7fffffff;
    w.j_hi = 0;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        int js = 0, je = 0;
        const int f_lo = w.q0 + (p.hpair ? 0 : t * kBlockQ);
        if (t < C::NQT && f_lo < flat_rows) {
            const int q_lo = f_lo / p.pack;   // the tile's first and last query
            je = nkv;
            if (p.causal) {
                const int q_hi = min(f_lo + kBlockQ - 1, flat_rows - 1) / p.pack;
                const int lim = q_hi + diag;   // last visible key of the tile's last row
                je = lim < 0 ? 0 : min(nkv, lim / C::BC + 1);
            }
            if (p.window > 0) {
                const int first = q_lo + diag - p.window + 1;   // first visible key of the first row
                js = first <= 0 ? 0 : min(first / C::BC, nkv);
            }
            if (p.num_splits > 1) {   // this split's share of the key tiles
                js = max(js, w.split * p.split_tiles);
                je = min(je, (w.split + 1) * p.split_tiles);
            }
            if (je <= js) js = je = 0;
        }
        w.js[t] = js;
        w.je[t] = je;
        if (je > js) {
            w.j_lo = min(w.j_lo, js);
            w.j_hi = max(w.j_hi, je);
        }
    }
    if (w.j_hi == 0) w.j_lo = 0;
    return w;
}

// The static schedule: in pass r the CTAs take units r * G .. r * G + G - 1 (G = gridDim.x),
// CTA i unit r * G + i in even passes and r * G + G - 1 - i in odd ones (a snake order).
// The causal order sorts units longest first, so alternating the direction pairs the CTAs
// that drew the longest units of one pass with the shortest of the next: the busiest CTA
// ends within about 1 % of the mean on the causal 4K and 16K workloads, where a plain
// stride left it 6-7 % above.  Every role walks the same sequence; a unit index past the
// end (only in the schedule's last pass) is skipped by all of them.
__device__ __forceinline__ int sched_unit(int r) {
    const int g = int(gridDim.x), i = int(blockIdx.x);
    return r * g + ((r & 1) ? g - 1 - i : i);
}

struct Ctl {
    volatile int *abort_flag;
    int *status;
    uint64_t limit_ns;   // per-wait limit (kWaitLimitNs outside the failure-path test build)
};

// Poll `bar` until the phase of parity `parity` completes.  Gives up when another role
// has raised the abort flag (unless `drain`: unwinding waits for the hardware's own
// copies/MMAs regardless) or after `limit_ns`, recording the timeout in the status word.
// Out of line and instantiated per role (ROLE), so each copy is compiled under the
// register budget of the warpgroup that calls it.
template <int ROLE>
__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, Ctl ctl, int site,
                                       uint64_t limit_ns, bool drain = false) {
    const uint64_t t0 = sm100::global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (sm100::mbar_try_wait(bar, parity)) return true;
        if (!drain && *ctl.abort_flag) return false;
        if (sm100::global_timer_ns() - t0 > limit_ns) {
            *ctl.abort_flag = 1;
            atomicCAS(ctl.status, 0, kStatusTimeout | (site << 8) | (min(int(blockIdx.x), 0xFFFF) << 16));
            return false;
        }
    }
}

constexpr int kRoleSoftmax = 0, kRoleControl = 1;

template <int ROLE = kRoleControl>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl &ctl, int site) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    return wait_slow<ROLE>(bar, parity, ctl, site, ctl.limit_ns);
}

// Warp-uniform wait: every lane polls, the warp proceeds only if all lanes saw it.
template <int ROLE = kRoleSoftmax>
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, const Ctl &ctl, int site) {
    const bool ok = wait_bar<ROLE>(bar, parity, ctl, site);
    const bool all = __all_sync(0xffffffffu, ok);
    if (!all) *ctl.abort_flag = 1;
    return all;
}

// ------------------------------------------------------------------ TMA producer

template <class C>
__device__ void producer_role(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                              const FwdParams &p, uint32_t sbase, const Ctl &ctl) {
    auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
    sm100::prefetch_tensormap(tm_q);
    sm100::prefetch_tensormap(tm_k);
    sm100::prefetch_tensormap(tm_v);
    uint32_t kv_cnt = 0;
    uint32_t qcnt[2] = {0, 0};
    bool ok = true;
    for (int r = 0; ok && r * int(gridDim.x) < p.num_units; ++r) {
        const int u = sched_unit(r);
        if (u >= p.num_units) continue;
        const UnitInfo w = decode_unit<C>(u, p);
        if (w.j_hi == w.j_lo) continue;
#pragma unroll
        for (int t = 0; t < C::NQT; ++t) {
            if (!ok || w.je[t] == w.js[t]) continue;
            const int qb = int(qcnt[t] % C::NQB);
            if (!warp_wait_bar<kRoleControl>(bar(C::B_QEMPTY + t * C::NQB + qb), ((qcnt[t] / C::NQB) & 1u) ^ 1u, ctl, kSiteQEmpty)) {
                ok = false;
                break;
            }
            ++qcnt[t];
            const uint32_t fb = bar(C::B_QFULL + t * C::NQB + qb);
            sm100::mbar_arrive_expect_tx_elected(fb, C::Q_TILE);
            const uint32_t dst = sbase + C::SMEM_Q + (t * C::NQB + qb) * C::Q_TILE;
#pragma unroll
            for (int c = 0; c < C::NCH; ++c)
                sm100::tma_load_4d_elected(dst + c * C::Q_CHUNK, tm_q, fb, c * C::CW, w.hq + (p.hpair ? t : 0),
                                           (w.q0 + (p.hpair ? 0 : t * kBlockQ)) / p.pack, w.b);
        }
        for (int j = w.j_lo; ok && j < w.j_hi; ++j) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const int s = int(kv_cnt % C::NS);
                if constexpr (C::FAULT) {
                    if (kv_cnt == uint32_t(p.withheld_load)) {   // left out: nothing will fill this slot
                        ++kv_cnt;
                        continue;
                    }
                }
                if (!warp_wait_bar<kRoleControl>(bar(C::B_EMPTY + s), ((kv_cnt / C::NS) & 1u) ^ 1u, ctl, kSiteKvEmpty)) { ok = false; break; }
                const uint32_t fb = bar(C::B_FULL + s);
                sm100::mbar_arrive_expect_tx_elected(fb, C::KV_TILE);
                const uint32_t dst = sbase + C::SMEM_KV + s * C::KV_TILE;
                const CUtensorMap *m = which ? tm_v : tm_k;
#pragma unroll
                for (int c = 0; c < C::NCH; ++c)
                    sm100::tma_load_4d_elected(dst + c * C::KV_CHUNK, m, fb, c * C::CW, w.kvh, j * C::BC, w.b);
                ++kv_cnt;
            }
        }
    }
    if (!ok || *ctl.abort_flag) {
        // Unwinding after a timeout (here or in another role): let this thread's copies
        // still in flight land before the CTA exits (the last load issued into each slot,
        // and each Q tile).
        const uint32_t first = kv_cnt > uint32_t(C::NS) ? kv_cnt - C::NS : 0u;
        for (uint32_t n = first; n < kv_cnt; ++n)
            wait_slow<kRoleControl>(bar(C::B_FULL + int(n % C::NS)), (n / C::NS) & 1u, ctl, kSiteProducerDrain,
                      ctl.limit_ns / 10, true);
#pragma unroll
        for (int t = 0; t < C::NQT; ++t) {
            const uint32_t first_q = qcnt[t] > uint32_t(C::NQB) ? qcnt[t] - C::NQB : 0u;
            for (uint32_t n = first_q; n < qcnt[t]; ++n)
                wait_slow<kRoleControl>(bar(C::B_QFULL + t * C::NQB + int(n % C::NQB)), (n / C::NQB) & 1u, ctl,
                          kSiteProducerDrain, ctl.limit_ns / 10, true);
        }
    }
}

// ------------------------------------------------------------------ MMA issuer

template <class C>
__device__ __forceinline__ void issue_qk(uint32_t sbase, uint32_t tmem, int t, int qbuf, int slot, int sbuf) {
    // Descriptors are built once; k-slice kk of the 128-byte (64-byte) swizzled rows
    // starts at a compile-time byte offset, added to the start-address field (the
    // address stays below 256 KB, so the 14-bit field never carries).
    const uint64_t a0 = sm100::opaque(sm100::smem_desc(sbase + C::SMEM_Q + (t * C::NQB + qbuf) * C::Q_TILE, 16, C::SBO, C::LAYOUT));
    const uint64_t b0 = sm100::opaque(sm100::smem_desc(sbase + C::SMEM_KV + slot * C::KV_TILE, 16, C::SBO, C::LAYOUT));
    const uint32_t d_tmem = tmem + uint32_t(C::SSHARE ? 0 : (t * C::SB + sbuf) * C::BC);
#pragma unroll
    for (int kk = 0; kk < C::D / C::KSTEP; ++kk) {
        constexpr int kCW = C::CW;
        const uint32_t a_off = uint32_t(((kk * C::KSTEP) / kCW) * C::Q_CHUNK + ((kk * C::KSTEP) % kCW) * C::ES);
        const uint32_t b_off = uint32_t(((kk * C::KSTEP) / kCW) * C::KV_CHUNK + ((kk * C::KSTEP) % kCW) * C::ES);
        if constexpr (C::FP8)
            sm100::mma_f8_ss_elected(d_tmem, a0 + (a_off >> 4), b0 + (b_off >> 4), C::IDESC_S, kk > 0 ? 1u : 0u);
        else
            sm100::mma_bf16_ss_elected(d_tmem, a0 + (a_off >> 4), b0 + (b_off >> 4), C::IDESC_S, kk > 0 ? 1u : 0u);
    }
}

template <class C, int KK_BEGIN = 0, int KK_END = C::BC / C::KSTEP>
__device__ __forceinline__ void issue_pv(uint32_t sbase, uint32_t tmem, int t, int slot, int sbuf, bool accumulate) {
    // V tile is [BC rows x d] row-major: MN-major B operand; 16 key rows per MMA,
    // 64-element column chunks C::KV_CHUNK bytes apart (leading byte offset).  P is the
    // A operand, read from TMEM (16 bf16 = 8 columns per MMA).
    const uint64_t b0 = sm100::opaque(sm100::smem_desc(sbase + C::SMEM_KV + slot * C::KV_TILE, C::KV_CHUNK, C::SBO, C::LAYOUT));
    const uint32_t a_tmem = tmem + uint32_t(C::PSEP ? C::P_COL0 + t * C::PCOLS : (t * C::SB + sbuf) * C::BC);
    const uint32_t d_tmem = tmem + uint32_t(C::O_COL0 + t * C::OST);
    // one MMA takes KSTEP keys: 32 bytes of each P row = 8 TMEM columns, KSTEP rows of V
#pragma unroll
    for (int kk = KK_BEGIN; kk < KK_END; ++kk) {
        if constexpr (C::FP8)
            sm100::mma_f8_ts_elected(d_tmem, a_tmem + uint32_t(kk * 8), b0 + uint64_t((kk * C::KSTEP * C::RB) >> 4),
                                     C::IDESC_O, (accumulate || kk > 0) ? 1u : 0u);
        else
            sm100::mma_bf16_ts_elected(d_tmem, a_tmem + uint32_t(kk * 8), b0 + uint64_t((kk * 16 * C::RB) >> 4),
                                       C::IDESC_O, (accumulate || kk > 0) ? 1u : 0u);
    }
}

template <class C>
__device__ void mma_role(const FwdParams &p, uint32_t sbase, uint32_t tmem, const Ctl &ctl) {
    auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
    // K/V loads arrive in the order K_0, V_0, K_1, V_1, ...: load n sits in slot n % NS
    // with phase (n / NS) & 1; kv_base is the first load index of the current unit.
    uint32_t kv_base = 0;
    uint32_t qcnt[2] = {0, 0};
    uint32_t s_iss[2] = {0, 0};      // S tiles issued per query tile (S buffer = count % SB)
    uint32_t p_got[2] = {0, 0};      // P tiles consumed per query tile (= P V MMAs issued)
    uint32_t u_count = 0;            // units of this CTA so far (each releases O_EMPTY once)
    uint32_t s_total = 0;            // SSHARE: S tiles issued into the shared buffer so far
    bool ok = true;
    auto wait_load = [&](uint32_t n, int &slot) -> bool {
        slot = int(n % C::NS);
        return warp_wait_bar<kRoleControl>(bar(C::B_FULL + slot), (n / C::NS) & 1u, ctl, kSiteKvFull);
    };
    // An S MMA must not overwrite TMEM columns that an earlier P V MMA is still reading as
    // its A operand (P lives in the S buffer it was computed from): the tensor core does
    // not order one MMA's operand reads before a later MMA's accumulator writes.  S number
    // n of a tile goes into buffer n % SB, which P V number n - SB read: wait for that one
    // (each completion of the buffer's PVDONE barrier is waited for once, in order).
    auto wait_buffer_free = [&](int t) -> bool {
        const uint32_t n = s_iss[t];
        // With P in columns of its own, S never overwrites an operand still being read;
        // the softmax writes the next P only after the next S's commit, which completes
        // after every earlier MMA of this thread (the previous P V included).
        if (C::PSEP || n < uint32_t(C::SB)) return true;
        const int b = int(n % C::SB);
        return warp_wait_bar<kRoleControl>(bar(C::B_PVDONE + t * C::SB + b), ((n / C::SB) - 1u) & 1u, ctl,
                                           kSitePvDone);
    };
    for (int r = 0; ok && r * int(gridDim.x) < p.num_units; ++r) {
        const int u = sched_unit(r);
        if (u >= p.num_units) continue;
        const uint32_t u_local = u_count++;
        const UnitInfo w = decode_unit<C>(u, p);
        if (w.j_hi == w.j_lo) continue;
        int qbuf[2] = {0, 0};
        auto visits = [&](int t, int j) { return w.js[t] <= j && j < w.je[t]; };
        // S_t,j for query tile t, from the K tile in `slot`.
        auto issue_s = [&](int t, int j, int slot) -> bool {
            if (!wait_buffer_free(t)) return false;
            if constexpr (C::SSHARE) {
                // the shared buffer's previous S (of either tile) has been read by its softmax
                if (s_total > 0 && !warp_wait_bar<kRoleControl>(bar(C::B_SEMPTY), (s_total - 1u) & 1u, ctl, kSiteSEmpty))
                    return false;
                ++s_total;
            }
            sm100::tc_fence_after_sync();
            const int sb = int(s_iss[t] % C::SB);
            issue_qk<C>(sbase, tmem, t, qbuf[t], slot, sb);
            sm100::tc_commit_elected(bar(C::B_SFULL + t * C::SB + sb));
            ++s_iss[t];
            if (j == w.je[t] - 1) sm100::tc_commit_elected(bar(C::B_QEMPTY + t * C::NQB + qbuf[t]));
            return true;
        };
        // O_t += P_t,j V_j from the V tile in `slot`.
        auto issue_o = [&](int t, int j, int slot) -> bool {
            const int sb = int(p_got[t] % C::SB);
            if (!C::PSPLIT && !warp_wait_bar<kRoleControl>(bar(C::B_PFULL + t * C::SB + sb), (p_got[t] / C::SB) & 1u,
                                                            ctl, kSitePFull))
                return false;
            if (j == w.js[t] && u_local > 0 &&
                !warp_wait_bar<kRoleControl>(bar(C::B_OEMPTY + t), (u_local - 1) & 1u, ctl, kSiteOEmpty))
                return false;
            if constexpr (C::PSPLIT) {
                // the first 64 keys of P are in TMEM
                if (!warp_wait_bar<kRoleControl>(bar(C::B_PHALF + t * C::SB + sb), (p_got[t] / C::SB) & 1u, ctl,
                                                 kSitePFull))
                    return false;
                sm100::tc_fence_after_sync();
                issue_pv<C, 0, C::BC / C::KSTEP / 2>(sbase, tmem, t, slot, sb, j > w.js[t]);
                if (!warp_wait_bar<kRoleControl>(bar(C::B_PFULL + t * C::SB + sb), (p_got[t] / C::SB) & 1u, ctl,
                                                 kSitePFull))
                    return false;
                sm100::tc_fence_after_sync();
                issue_pv<C, C::BC / C::KSTEP / 2>(sbase, tmem, t, slot, sb, true);
            } else {
                sm100::tc_fence_after_sync();
                issue_pv<C>(sbase, tmem, t, slot, sb, j > w.js[t]);
            }
            if (C::PSEP || C::SB != 1) sm100::tc_commit_elected(bar(C::B_ODONE + t));
            if (!C::PSEP) sm100::tc_commit_elected(bar(C::B_PVDONE + t * C::SB + sb));
            if (j == w.je[t] - 1) sm100::tc_commit_elected(bar(C::B_OFINAL + t));
            ++p_got[t];
            return true;
        };

        // Q tiles of this unit
#pragma unroll
        for (int t = 0; t < C::NQT; ++t) {
            if (!ok || w.je[t] == w.js[t]) continue;
            qbuf[t] = int(qcnt[t] % C::NQB);
            if (!warp_wait_bar<kRoleControl>(bar(C::B_QFULL + t * C::NQB + qbuf[t]), (qcnt[t] / C::NQB) & 1u, ctl,
                                             kSiteQFull))
                ok = false;
            ++qcnt[t];
        }
        if (!ok) break;
        sm100::tc_fence_after_sync();
        int slot_k = 0, slot_v = 0;
        // S for the first SB key tiles (K/V tile j is load pair j - j_lo of the unit)
        for (int j = w.j_lo; ok && j < w.j_lo + C::SB && j < w.j_hi; ++j) {
            if (!wait_load(kv_base + 2u * (j - w.j_lo), slot_k)) { ok = false; break; }
#pragma unroll
            for (int t = 0; t < C::NQT; ++t)
                if (ok && visits(t, j) && !issue_s(t, j, slot_k)) ok = false;
            sm100::tc_commit_elected(bar(C::B_EMPTY + slot_k));
        }
        if (!ok) break;
        for (int j = w.j_lo; ok && j < w.j_hi; ++j) {
            if (!wait_load(kv_base + 2u * (j - w.j_lo) + 1u, slot_v)) { ok = false; break; }
            const int jn = j + C::SB;
            bool k_ready = false;
            if constexpr (C::SB == 2) {
                // P V for both tiles first (keeps the tensor core busy while the S for key
                // tile j + 2 waits for them), then S_{j+2}, which is not needed until the
                // softmax has finished S_{j+1}.
#pragma unroll
                for (int t = 0; t < C::NQT; ++t)
                    if (ok && visits(t, j) && !issue_o(t, j, slot_v)) ok = false;
                if (!ok) break;
                sm100::tc_commit_elected(bar(C::B_EMPTY + slot_v));
                if (jn < w.j_hi) {
                    if (!wait_load(kv_base + 2u * (jn - w.j_lo), slot_k)) { ok = false; break; }
                    k_ready = true;
#pragma unroll
                    for (int t = 0; t < C::NQT; ++t)
                        if (ok && visits(t, jn) && !issue_s(t, jn, slot_k)) ok = false;
                    if (!ok) break;
                }
            } else if constexpr (C::SSHARE) {
                // Per tile, the next S (as soon as the shared buffer is free) then this
                // P V: S_0(j+1), P_0(j) V_j, S_1(j+1), P_1(j) V_j.
#pragma unroll
                for (int t = 0; t < C::NQT; ++t) {
                    if (!ok) break;
                    if (visits(t, jn)) {
                        if (!k_ready) {
                            if (!wait_load(kv_base + 2u * (jn - w.j_lo), slot_k)) { ok = false; break; }
                            k_ready = true;
                        }
                        if (!issue_s(t, jn, slot_k)) { ok = false; break; }
                    }
                    if (visits(t, j) && !issue_o(t, j, slot_v)) { ok = false; break; }
                }
                if (!ok) break;
                sm100::tc_commit_elected(bar(C::B_EMPTY + slot_v));
            } else {
                // One S buffer: per tile, P V then (once it is done) the next S.
#pragma unroll
                for (int t = 0; t < C::NQT; ++t) {
                    if (!ok) break;
                    if (visits(t, j) && !issue_o(t, j, slot_v)) { ok = false; break; }
                    if (visits(t, jn)) {
                        if (!k_ready) {
                            if (!wait_load(kv_base + 2u * (jn - w.j_lo), slot_k)) { ok = false; break; }
                            k_ready = true;
                        }
                        if (!issue_s(t, jn, slot_k)) { ok = false; break; }
                    }
                }
                if (!ok) break;
                sm100::tc_commit_elected(bar(C::B_EMPTY + slot_v));
            }
            if (k_ready) sm100::tc_commit_elected(bar(C::B_EMPTY + slot_k));
        }
        if (!ok) break;
        kv_base += 2u * uint32_t(w.j_hi - w.j_lo);
    }
    // Every MMA this thread issued is complete before the CTA may free TMEM.
    sm100::tc_commit_elected(bar(C::B_DRAIN));
    wait_slow<kRoleControl>(bar(C::B_DRAIN), 0u, ctl, kSiteDrain, ctl.limit_ns, true);
}

// ------------------------------------------------------------------ softmax / epilogue

// p = 2^(s * c_log2 - m) for one row of a score tile, packed to bf16 (F16: fp16) pairs and stored
// to BC/2 TMEM columns at p_taddr (over the S tile itself, or P's own columns); returns
// the fp32 row sum of p.  On unmasked tiles SOFT_EXP of every 8 pairs take the FMA-pipe
// exponential to relieve the special-function unit (worth it where the exponentials
// dominate, i.e. small head dims); masked tiles (which may hold -inf scores) use the
// hardware ex2 throughout.
// FP8 P: four exponentials per 32-bit TMEM column (E4M3 bytes), 128 keys per store of
// 32 columns; the row sum is taken over the unrounded fp32 values, like the LSE.
template <int BC, bool DEFER = false>
__device__ __forceinline__ float exp_pack_store_e4m3(const uint32_t (&s)[BC], float c_log2, float neg_m,
                                                     uint32_t p_taddr, uint32_t (*pk_all)[32] = nullptr) {
    const uint64_t c2 = sm100::pack2(c_log2, c_log2);
    const uint64_t nm2 = sm100::pack2(neg_m, neg_m);
    uint64_t acc0 = sm100::pack2(0.f, 0.f), acc1 = acc0;
#pragma unroll
    for (int c = 0; c < BC / 128; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int e = 128 * c + 4 * i;
            const uint64_t x01 = sm100::fma2(sm100::pack2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2, nm2);
            const uint64_t x23 = sm100::fma2(sm100::pack2(__uint_as_float(s[e + 2]), __uint_as_float(s[e + 3])), c2, nm2);
            float a, b, cc, d;
            sm100::unpack2(x01, a, b);
            sm100::unpack2(x23, cc, d);
            const float p0 = sm100::ex2_approx(a), p1 = sm100::ex2_approx(b);
            const float p2 = sm100::ex2_approx(cc), p3 = sm100::ex2_approx(d);
            acc0 = sm100::add2(acc0, sm100::pack2(p0, p1));
            acc1 = sm100::add2(acc1, sm100::pack2(p2, p3));
            pk[i] = sm100::pack_e4m3x4(p0, p1, p2, p3);
        }
        if constexpr (DEFER) {
#pragma unroll
            for (int i = 0; i < 32; ++i) pk_all[c][i] = pk[i];
            continue;
        }
        sm100::tmem_st32(p_taddr + uint32_t(32 * c), pk);
    }
    float a0, a1, b0, b1;
    sm100::unpack2(acc0, a0, a1);
    sm100::unpack2(acc1, b0, b1);
    return (a0 + a1) + (b0 + b1);
}

// DEFER: nothing is stored; the packed P is left in pk_all for the caller to store once the
// P V MMA still reading this tile's P buffer has completed.
template <int BC, int SOFT_EXP, bool MIXED, bool F16, bool SPLIT = false, bool DEFER = false>
__device__ __forceinline__ float exp_pack_store(const uint32_t (&s)[BC], float c_log2, float neg_m,
                                                uint32_t p_taddr, uint32_t half_bar = 0,
                                                uint32_t (*pk_all)[32] = nullptr) {
    const uint64_t c2 = sm100::pack2(c_log2, c_log2);
    const uint64_t nm2 = sm100::pack2(neg_m, neg_m);
    uint64_t acc0 = sm100::pack2(0.f, 0.f), acc1 = acc0;
#pragma unroll
    for (int c = 0; c < BC / 64; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int e = 64 * c + 2 * i;
            const float s0 = __uint_as_float(s[e]), s1 = __uint_as_float(s[e + 1]);
            const uint64_t x2 = sm100::fma2(sm100::pack2(s0, s1), c2, nm2);
            uint64_t p2;
            if (MIXED && (i % 8) >= 8 - SOFT_EXP) {
                p2 = sm100::ex2_poly_pair(x2);
            } else {
                float a, b;
                sm100::unpack2(x2, a, b);
                p2 = sm100::pack2(sm100::ex2_approx(a), sm100::ex2_approx(b));
            }
            if (i & 1) acc1 = sm100::add2(acc1, p2);
            else acc0 = sm100::add2(acc0, p2);
            float lo, hi;
            sm100::unpack2(p2, lo, hi);
            pk[i] = sm100::pack_x2<F16>(lo, hi);
        }
        if constexpr (DEFER) {
#pragma unroll
            for (int i = 0; i < 32; ++i) pk_all[c][i] = pk[i];
            continue;
        }
        sm100::tmem_st32(p_taddr + uint32_t(32 * c), pk);
        if constexpr (SPLIT) {
            if (c == 0) {   // first 64 keys of P (and any rescale of O before it) are in TMEM
                sm100::tmem_st_wait();
                sm100::tc_fence_before_sync();
                sm100::mbar_arrive(half_bar);
            }
        }
    }
    float a0, a1, b0, b1;
    sm100::unpack2(acc0, a0, a1);
    sm100::unpack2(acc1, b0, b1);
    return (a0 + a1) + (b0 + b1);
}

template <class C>
__device__ void softmax_role(const FwdParams &p, const CUtensorMap *tm_o, uint32_t sbase, uint32_t tmem,
                             const Ctl &ctl, int warp, int lane) {
    constexpr int BC = C::BC;
    auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
    const int t = warp / 4;
    const int quarter = warp % 4;                  // TMEM lanes 32*quarter .. +31
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t s_taddr0 = tmem + lane_off + uint32_t(C::SSHARE ? 0 : t * C::SB * BC);   // S buffer 0 of this tile
    const uint32_t p_taddr_sep = tmem + lane_off + uint32_t(C::P_COL0 + t * C::PCOLS);
    const uint32_t o_taddr = tmem + lane_off + uint32_t(C::O_COL0 + t * C::OST);
    const float c_log2 = p.scale_log2;
    uint32_t scnt = 0, ocnt = 0, ofin = 0;
    // Lazy rescale: O_t holds the sum up to block j-1 at the old reference max; wait for
    // that MMA (completion number `odone`), then scale this warp's rows by alpha (1 where
    // the max held).
    auto rescale_o = [&](bool need, float alpha, uint32_t odone) -> bool {
        if (!__any_sync(0xffffffffu, need)) return true;
        if (!warp_wait_bar(bar((C::PSEP || C::SB != 1) ? C::B_ODONE + t : C::B_PVDONE + t * C::SB), odone & 1u, ctl, kSiteODone)) return false;
        sm100::tc_fence_after_sync();
#pragma unroll
        for (int c = 0; c < C::O_CHUNKS; ++c) {
            uint32_t o[32];
            sm100::tmem_ld32_sync(o_taddr + uint32_t(32 * c), o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            sm100::tmem_st32(o_taddr + uint32_t(32 * c), o);
        }
        return true;
    };

    for (int r = 0; r * int(gridDim.x) < p.num_units; ++r) {
        const int u = sched_unit(r);
        if (u >= p.num_units) continue;
        const UnitInfo w = decode_unit<C>(u, p);
        const int js = w.js[t], je = w.je[t];
        const int nk = je - js;
        const int f_lo = w.q0 + (p.hpair ? 0 : t * kBlockQ);   // flat row f = i * pack + (hq - w.hq)
        const int q_lo = f_lo / p.pack;            // the tile's first query
        const int f_row = f_lo + row_in_tile;
        const int row = f_row / p.pack;            // this thread's query i and head hq
        const int hq = w.hq + (p.hpair ? t : f_row - row * p.pack);
        const int diag = p.diag;                   // causal: key j visible to row i iff j <= i + diag
        const int row_lim = p.causal ? row + diag : 0x7fffffff;
        // sliding window: keys j > i + diag - W; the tile's first row has the lowest bound
        const int row_lo = p.window > 0 ? row + diag - p.window + 1 : -0x7fffffff;
        const int tile_lo_hi = p.window > 0 ? q_lo + kBlockQ / p.pack - 1 + diag - p.window + 1 : -0x7fffffff;
        float m_ref = -INFINITY;                   // reference max, log2 units (scaled)
        float l = 0.f;                             // running sum of 2^(s*c - m_ref)

        for (int j = js; j < je; ++j) {
            const int sb = int(scnt % C::SB);
            const uint32_t s_taddr = s_taddr0 + uint32_t(sb * BC);
            const uint32_t p_taddr = C::PSEP ? p_taddr_sep : s_taddr;
            if (!warp_wait_bar(bar(C::B_SFULL + t * C::SB + sb), (scnt / C::SB) & 1u, ctl, kSiteSFull)) goto unwind;
            ++scnt;
            sm100::tc_fence_after_sync();
            uint32_t s[BC];
            if constexpr (BC == 128) sm100::tmem_ld128_sync(s_taddr, s);
            else sm100::tmem_ld64_sync(s_taddr, s);
            if constexpr (C::SSHARE) {
                // S is in registers: the shared buffer may take the next S (either tile's)
                sm100::tc_fence_before_sync();
                sm100::mbar_arrive(bar(C::B_SEMPTY));
            }

            const int k_lo = j * BC;
            // boundary tiles: the key tail, the causal diagonal, the window's lower edge
            const bool need_mask = (k_lo + BC > p.Nk) || (p.causal && k_lo + BC - 1 > q_lo + diag) ||
                                   (k_lo < tile_lo_hi);
            float alpha = 1.f;
            bool need_rescale = false;
            float row_sum;
            {
                if (need_mask) {
#pragma unroll
                    for (int i = 0; i < BC; ++i) {
                        const int key = k_lo + i;
                        if (key > row_lim || key >= p.Nk || key < row_lo) s[i] = __float_as_uint(-INFINITY);
                    }
                }
                // Row max: eight independent 3-input-max chains, then a short tree, so
                // the dependency depth stays small.
                float mx[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) mx[c] = fmaxf(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]));
#pragma unroll
                for (int i = 16; i < BC; i += 16)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        mx[c] = sm100::max3(mx[c], __uint_as_float(s[i + 2 * c]), __uint_as_float(s[i + 2 * c + 1]));
                const float mx_s = fmaxf(sm100::max3(mx[0], mx[1], mx[2]), sm100::max3(mx[3], mx[4], sm100::max3(mx[5], mx[6], mx[7]))) * c_log2;
                if (j == js) {
                    m_ref = mx_s;
                } else if (mx_s > m_ref + kRescaleLog2) {
                    alpha = sm100::ex2_approx(m_ref - mx_s);
                    m_ref = mx_s;
                    need_rescale = true;
                }
                // with a split hand-off, O is rescaled before any of P is handed over (the
                // first P V MMAs accumulate into O while the rest of P is computed)
                if constexpr (C::PSPLIT)
                    if (!rescale_o(need_rescale, alpha, ocnt + uint32_t(j - js) - 1u)) goto unwind;
                const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;
                const uint32_t half_bar = bar(C::B_PHALF + t * C::SB + sb);
                if constexpr (C::SSHARE) {
                    // P_t's columns are free once the previous P_t V has completed (the
                    // first P of a unit: the epilogue's wait for the unit's last P V)
                    constexpr int kChunks = C::PCOLS / 32;
                    uint32_t pk_all[kChunks][32];
                    if constexpr (C::FP8)
                        row_sum = exp_pack_store_e4m3<BC, true>(s, c_log2, neg_m, p_taddr, pk_all);
                    else
                        row_sum = need_mask
                                      ? exp_pack_store<BC, C::SOFT_EXP, false, C::F16, false, true>(s, c_log2, neg_m, p_taddr, 0, pk_all)
                                      : exp_pack_store<BC, C::SOFT_EXP, true, C::F16, false, true>(s, c_log2, neg_m, p_taddr, 0, pk_all);
                    if (j > js && !warp_wait_bar(bar(C::B_ODONE + t), (ocnt + uint32_t(j - js) - 1u) & 1u, ctl, kSiteODone))
                        goto unwind;
                    sm100::tc_fence_after_sync();
#pragma unroll
                    for (int c = 0; c < kChunks; ++c) sm100::tmem_st32(p_taddr + uint32_t(32 * c), pk_all[c]);
                } else if constexpr (C::FP8)
                    row_sum = exp_pack_store_e4m3<BC>(s, c_log2, neg_m, p_taddr);
                else
                    row_sum = need_mask
                                  ? exp_pack_store<BC, C::SOFT_EXP, false, C::F16, C::PSPLIT>(s, c_log2, neg_m, p_taddr, half_bar)
                                  : exp_pack_store<BC, C::SOFT_EXP, true, C::F16, C::PSPLIT>(s, c_log2, neg_m, p_taddr, half_bar);
            }
            l = l * alpha + row_sum;
            if constexpr (!C::PSPLIT)
                if (!rescale_o(need_rescale, alpha, ocnt + uint32_t(j - js) - 1u)) goto unwind;
            sm100::tmem_st_wait();
            sm100::tc_fence_before_sync();
            sm100::mbar_arrive(bar(C::B_PFULL + t * C::SB + sb));
        }

        // epilogue: O / l -> bf16 -> out, LSE -> lse
        if (nk > 0) {
            if (!warp_wait_bar(bar(C::B_OFINAL + t), ofin & 1u, ctl, kSiteOFinal)) goto unwind;
            ++ofin;
            sm100::tc_fence_after_sync();
        }
        ocnt += uint32_t(nk);
        {
            float inv_l = l > 0.f ? 1.f / l : 0.f;
            if constexpr (C::FP8) inv_l *= p.o_scale;
            const bool store = row < p.Nq;
            const size_t row_off = (size_t(w.b) * p.Nq + size_t(row)) * p.Hq + hq;   // [b][row][hq]
            const bool split_mode = p.num_splits > 1 || p.partial;
            uint16_t *orow = static_cast<uint16_t *>(p.out) + row_off * C::D;
            float *prow = split_mode ? p.o_part + (size_t(w.split) * p.B * p.Nq * p.Hq + row_off) * C::D : nullptr;
            if (C::OSTAGE && p.o_tma && !split_mode) {
                // 64 columns per pass: this warp's 32 rows (lane = row) into its staging
                // buffer as one 128-byte-swizzled TMA box (16-byte unit i of row r at unit
                // i ^ (r % 8)), then one TMA store; rows past Nq and columns past d lie
                // outside the tensor and are not written.
                const uint32_t stage = sbase + uint32_t(C::SMEM_OST + warp * C::OST_BYTES);
                const int row0 = (f_lo + quarter * 32) / p.pack;   // first query of the box
#pragma unroll
                for (int c2 = 0; c2 < (C::D + 63) / 64; ++c2) {
                    uint32_t pk[32];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t o[32];
                        if (nk > 0) {
                            sm100::tmem_ld32_sync(o_taddr + uint32_t(64 * c2 + 32 * h), o);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] = 0u;
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            pk[16 * h + i] = sm100::pack_x2<C::F16>(__uint_as_float(o[2 * i]) * inv_l,
                                                                    __uint_as_float(o[2 * i + 1]) * inv_l);
                    }
#pragma unroll
                    for (int u16 = 0; u16 < 8; ++u16)
                        sm100::st_shared_v4(stage + uint32_t(lane * 128 + ((u16 ^ (lane & 7)) * 16)), pk[4 * u16],
                                            pk[4 * u16 + 1], pk[4 * u16 + 2], pk[4 * u16 + 3]);
                    sm100::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && row0 < p.Nq) {   // (a box wholly past Nq has nothing to write)
                        sm100::tma_store_4d(tm_o, stage, 64 * c2, w.hq + (p.hpair ? t : 0), row0, w.b);
                        sm100::bulk_commit_group();
                        sm100::bulk_wait_group_read0();   // the staging buffer may be rewritten
                    }
                    __syncwarp();
                }
            } else {
#pragma unroll
            for (int c = 0; c < C::O_CHUNKS; ++c) {
                uint32_t o[32];
                if (nk > 0) {
                    sm100::tmem_ld32_sync(o_taddr + uint32_t(32 * c), o);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                if (split_mode) {
                    // fp32 partial for the merge (normalised by this split's own l)
                    if (store) {
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4) {
                            const int col = 32 * c + 4 * v4;
                            if (col < C::D)
                                *reinterpret_cast<float4 *>(prow + col) =
                                    make_float4(__uint_as_float(o[4 * v4]) * inv_l, __uint_as_float(o[4 * v4 + 1]) * inv_l,
                                                __uint_as_float(o[4 * v4 + 2]) * inv_l, __uint_as_float(o[4 * v4 + 3]) * inv_l);
                        }
                    }
                    continue;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = sm100::pack_x2<C::F16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
                if (store) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        const int col = 32 * c + 8 * v4;
                        if (col < C::D)
                            *reinterpret_cast<uint4 *>(orow + col) =
                                make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                    }
                }
            }
            }
            sm100::tc_fence_before_sync();
            sm100::mbar_arrive(bar(C::B_OEMPTY + t));
            const float lse_row = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
            const size_t lse_off = (size_t(w.b) * p.Hq + hq) * p.Nq + row;
            if (split_mode) {
                if (store) p.lse_part[size_t(w.split) * p.B * p.Hq * p.Nq + lse_off] = lse_row;
            } else if (p.lse != nullptr && store) {
                p.lse[lse_off] = lse_row;
            }
        }
    }
unwind:
    sm100::tmem_st_wait();
    if (C::OSTAGE && lane == 0) sm100::bulk_wait_group0();   // this warp's O stores are complete
}

// ------------------------------------------------------------------ kernel

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
              const __grid_constant__ FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = sm100::smem_u32(smem);
    const int warp = int(threadIdx.x) / 32;
    const int lane = int(threadIdx.x) % 32;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::SMEM_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::SMEM_MISC + 4);
    const Ctl ctl{abort_flag, p.status, C::FAULT ? uint64_t(p.wait_limit_ns) : kWaitLimitNs};

    if (threadIdx.x == 0) {
        auto bar = [&](int i) { return sbase + C::SMEM_BAR + 8u * uint32_t(i); };
        for (int s = 0; s < C::NS; ++s) {
            sm100::mbar_init(bar(C::B_FULL + s), 1);
            sm100::mbar_init(bar(C::B_EMPTY + s), 1);
        }
        for (int i = 0; i < C::NQT * C::NQB; ++i) {
            sm100::mbar_init(bar(C::B_QFULL + i), 1);
            sm100::mbar_init(bar(C::B_QEMPTY + i), 1);
        }
        for (int i = 0; i < C::NQT * C::SB; ++i) {
            sm100::mbar_init(bar(C::B_SFULL + i), 1);
            sm100::mbar_init(bar(C::B_PFULL + i), 128);
            sm100::mbar_init(bar(C::B_PHALF + i), 128);
            sm100::mbar_init(bar(C::B_PVDONE + i), 1);
        }
        for (int t = 0; t < C::NQT; ++t) {
            sm100::mbar_init(bar(C::B_ODONE + t), 1);
            sm100::mbar_init(bar(C::B_OFINAL + t), 1);
            sm100::mbar_init(bar(C::B_OEMPTY + t), 128);
        }
        sm100::mbar_init(bar(C::B_DRAIN), 1);
        sm100::mbar_init(bar(C::B_SEMPTY), 128);
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

    if (warp < C::SOFTMAX_WARPS) {
        if constexpr (C::REALLOC_REGS) sm100::regs_increase<C::SOFTMAX_REGS>();
        softmax_role<C>(p, &tm_o, sbase, tmem, ctl, warp, lane);
    } else {
        if constexpr (C::REALLOC_REGS) sm100::regs_decrease<C::CONTROL_REGS>();
        if (warp == C::TMA_WARP) {
            producer_role<C>(&tm_q, &tm_k, &tm_v, p, sbase, ctl);
        } else if (warp == C::MMA_WARP) {
            mma_role<C>(p, sbase, tmem, ctl);
        }
    }
    __syncwarp();

    sm100::tc_fence_before_sync();
    __syncthreads();
    sm100::tc_fence_after_sync();
    if (warp == 0) sm100::tmem_dealloc(tmem, C::TMEM_COLS);
}

// Split-KV merge: one warp per output row (b, i, hq).  With m = max_s LSE_s, the weights
// w_s = e^(LSE_s - m) combine the per-split normalised outputs O = sum_s w_s O_s / sum_s w_s,
// and LSE = m + ln sum_s w_s; a row no split saw (all LSE_s = -inf) gets O = 0, LSE = -inf.
// The lanes read 32 splits' LSEs at once and pass the weights around by shuffle, so the
// loads of the partial rows do not wait on one another.
template <int D, bool F16>
__global__ void __launch_bounds__(256) fa_splitkv_merge_kernel(const float *o_part, const float *lse_part,
                                                               uint16_t *out, float *lse, int B, int Hq,
                                                               int Nq, int num_splits) {
    constexpr int PER_LANE = (D + 31) / 32;
    const long rows = long(B) * Nq * Hq;
    const long split_stride_o = rows * D, split_stride_l = rows;
    const int lane = int(threadIdx.x) % 32;
    for (long r = (long(blockIdx.x) * blockDim.x + threadIdx.x) / 32; r < rows;
         r += long(gridDim.x) * blockDim.x / 32) {
        const int hq = int(r % Hq);
        const long bi = r / Hq;                 // b * Nq + i
        const int i = int(bi % Nq);
        const int b = int(bi / Nq);
        const long lse_off = (long(b) * Hq + hq) * Nq + i;
        float m = -INFINITY;
        for (int base = 0; base < num_splits; base += 32) {
            const int sp = base + lane;
            if (sp < num_splits) m = fmaxf(m, lse_part[sp * split_stride_l + lse_off]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float acc[PER_LANE];
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) acc[e] = 0.f;
        float wsum = 0.f;
        if (m != -INFINITY) {
            for (int base = 0; base < num_splits; base += 32) {
                const int sp = base + lane;
                const float ls = sp < num_splits ? lse_part[sp * split_stride_l + lse_off] : -INFINITY;
                const float wl = ls == -INFINITY ? 0.f : __expf(ls - m);
                wsum += wl;
                const int n = min(32, num_splits - base);
#pragma unroll 4
                for (int t = 0; t < n; ++t) {
                    const float wgt = __shfl_sync(0xffffffffu, wl, t);
                    const float *src = o_part + (base + t) * split_stride_o + r * D;
#pragma unroll
                    for (int e = 0; e < PER_LANE; ++e) {
                        const int col = lane + 32 * e;
                        if (col < D) acc[e] = fmaf(wgt, src[col], acc[e]);
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
        for (int e = 0; e < PER_LANE; ++e) {
            const int col = lane + 32 * e;
            if (col < D) {
                if constexpr (F16) out[r * D + col] = __half_as_ushort(__float2half_rn(acc[e] * inv));
                else out[r * D + col] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[e] * inv));
            }
        }
        if (lse != nullptr && lane == 0) lse[lse_off] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
    }
}

// Nk == 0: no key at all, so every output row is 0 and every LSE is -inf.
__global__ void fa_no_keys_kernel(uint4 *out, size_t n_vec16, float *lse, size_t n_lse) {
    const size_t stride = size_t(gridDim.x) * blockDim.x;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec16; i += stride)
        out[i] = make_uint4(0u, 0u, 0u, 0u);
    if (lse != nullptr)
        for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n_lse; i += stride)
            lse[i] = -INFINITY;
}

}  // namespace fa

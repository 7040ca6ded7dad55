/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention forward library (libfa.so).
 *
 * The operation (exact attention, forward):
 *
 *     S = scale * Q K^T               (per batch b and query head h)
 *     S_ij = -inf where masked        (causal: key j hidden from query i iff j > i + Nk - Nq)
 *     P = softmax(S) row by row,      O = P V
 *     LSE_i = ln sum_j exp(S_ij)      (natural log; -inf for a row with no visible key)
 *
 * is the formula softmax(Q K^T / sqrt(d_k)) V with its optional causal mask, as stated
 * on the hwcomputing.csdn.net article "FlashAttention in CANN ops-transformer"
 * (sections "where the memory black hole of standard attention comes from" and
 * "performance tuning", item 3 mask modes).  It is computed tile by tile with the
 * online softmax of the same article (section "online softmax": running row max m,
 * running sum l, rescale by exp(m_old - m_new), final O /= l), so S and P never
 * reach device memory.  Query head h reads key/value head h / (Hq / Hkv): the
 * repeat_interleave expansion of grouped-query attention ("Transformer efficient
 * attention: Flash Attention vs GQA", yunthe.com, section "GQA principle").
 * The head dimensions are those listed on the datacanvas.csdn.net head-dim article
 * (32, 64, 96, 128, 192, 256, plus 80 added by the custom-compile workaround).
 *
 * With fewer than 128 queries and n_rep = Hq / Hkv > 1 dividing 128, the n_rep query heads
 * of one KV head share a work unit (their rows stacked in one 128-row tile), so decode-sized
 * Nq keeps the tiles full; the results are the same.
 *
 * Conventions for every entry point:
 *  - All tensors are dense, row-major (C-contiguous), owned by the caller; the library
 *    allocates no device memory per call (scratch is the caller's workspace, or the
 *    static array of fa_fwd_splitkv_static) and keeps no pointer after it returns.
 *  - Pointers to tensors are DEVICE pointers on the calling thread's current CUDA device.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Work is enqueued asynchronously on `stream`; no host synchronisation happens,
 *    except in fa_device_status.
 *  - A non-zero return means nothing was launched.
 *  - Per device, the library looks up once (cudaGetSymbolAddress) and caches the addresses
 *    of its device status word and of the static scratch of fa_fwd_splitkv_static.  A
 *    cudaDeviceReset unloads the module behind them, so the library must not be called on a
 *    device after cudaDeviceReset in the same process.
 */
#ifndef EXACT_ATTENTION_FA_H
#define EXACT_ATTENTION_FA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by the entry points. */
enum fa_status_code {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,          /* null pointer, negative size, Hq % Hkv != 0, scale <= 0 or
                                        not finite, causal not 0/1, sizes beyond 32-bit indexing */
    FA_ERR_UNSUPPORTED_HEAD_DIM = 2, /* d not in {32, 64, 80, 96, 128, 192, 256} */
    FA_ERR_MISALIGNED = 3,           /* q/k/v/out not 16-byte aligned, or lse not 4-byte aligned */
    FA_ERR_UNSUPPORTED_DEVICE = 4,   /* no CUDA device, or the current device is not sm_100 */
    FA_ERR_CUDA = 5,                 /* a CUDA runtime/driver call failed (launch, tensor-map encode) */
    FA_ERR_DEVICE_TIMEOUT = 6,       /* reported by fa_device_status: a pipeline wait in the kernel
                                        gave up after its time limit; outputs are undefined */
    FA_ERR_NOT_DEVICE_MEMORY = 7,    /* a tensor pointer is not device memory of the current device,
                                        or its extent runs past the end of its allocation */
    FA_ERR_OVERLAP = 8,              /* out or lse overlaps an input or each other */
    FA_ERR_SCRATCH_LIMIT = 9         /* fa_fwd_splitkv_static: the partials need more than the
                                        library's static scratch (FA_SPLITKV_STATIC_SCRATCH_BYTES) */
};

/*
 * fa_fwd -- exact attention forward.
 *
 *   q    [B, Nq, Hq,  d] bf16, read only
 *   k    [B, Nk, Hkv, d] bf16, read only
 *   v    [B, Nk, Hkv, d] bf16, read only
 *   out  [B, Nq, Hq,  d] bf16, written (O, rounded to nearest-even from fp32)
 *   lse  [B, Hq, Nq]     fp32, written, or NULL to skip it
 *   B >= 0, Hq >= 1, Hkv >= 1 with Hq % Hkv == 0, Nq >= 0, Nk >= 0
 *   d in {32, 64, 80, 96, 128, 192, 256}
 *   scale > 0 and finite (the usual choice is 1/sqrt(d)); applied to Q K^T as given
 *   causal in {0, 1}
 *
 * B == 0 or Nq == 0: nothing to do, returns FA_OK.  Nk == 0: every row has no key,
 * so out is zero and lse is -inf.  Pointers of empty tensors may be NULL.
 * Errors are returned synchronously (see fa_status_code); a device-side pipeline
 * timeout is reported later by fa_device_status.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
           int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
           void *stream);

/*
 * fa_fwd_f16 -- fa_fwd on IEEE fp16 tensors: q, k, v and out are fp16 instead of bf16
 * (lse stays fp32).  The dtype choice between fp16 and bf16 is the one the
 * hwcomputing.csdn.net FlashAttention article weighs ("performance tuning", item on data
 * types: fp16 has the finer mantissa, bf16 the range).  The tensor cores multiply fp16 x
 * fp16 with fp32 accumulation; P is rounded to fp16 before P V and O to fp16 at the end
 * (|O| <= max |V|, so O cannot overflow when V is finite).  Arguments, layouts, ownership
 * and errors as fa_fwd.
 */
int fa_fwd_f16(const void *q, const void *k, const void *v, void *out, float *lse,
               int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
               void *stream);

/*
 * fa_fwd_fp8 -- fa_fwd on FP8 inputs: q, k, v are OCP E4M3 bytes with one dequantisation
 * factor per tensor (Q = descale_q * q8, K = descale_k * k8, V = descale_v * v8), the FP8
 * forward the datacanvas.csdn.net head-dim page attributes to FlashAttention-3.  The tensor
 * cores multiply E4M3 x E4M3 (kind::f8f6f4) with fp32 accumulation; P is rounded to E4M3
 * (relative error <= 2^-4) before P V; out is bf16 [B, Nq, Hq, d], lse fp32 as in fa_fwd
 * (the LSE of the dequantised logits).  d must be 64, 128 or 256 (FA_ERR_UNSUPPORTED_HEAD_DIM
 * otherwise); the descales must be finite and > 0.  Layouts, ownership and the other
 * errors as fa_fwd (q, k, v one byte per element, 16-byte aligned).
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, void *out, float *lse,
               int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
               float descale_q, float descale_k, float descale_v, int causal, void *stream);

/*
 * fa_fwd_window -- exact attention forward with a sliding-window (local) causal mask:
 * query row i sees the `window` keys ending at its causal diagonal,
 *
 *     i + (Nk - Nq) - window < j <= i + (Nk - Nq),
 *
 * the third mask mode of the hwcomputing.csdn.net FlashAttention article ("performance
 * tuning", item 3: only the most recent positions, for long texts).  Arguments, layouts,
 * ownership and errors as fa_fwd, with window >= 1 (FA_ERR_INVALID_ARG otherwise); a
 * window of at least Nk keys is the causal mask.  Key tiles wholly outside a query tile's
 * window are not visited.
 */
int fa_fwd_window(const void *q, const void *k, const void *v, void *out, float *lse,
                  int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                  void *stream);
/* fa_fwd_window_f16: the same on IEEE fp16 q, k, v and out (P rounded to fp16), as fa_fwd_f16
 * is to fa_fwd (the data-type option of the hwcomputing.csdn.net article's "performance
 * tuning" is independent of the mask mode). */
int fa_fwd_window_f16(const void *q, const void *k, const void *v, void *out, float *lse,
                      int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                      void *stream);

/*
 * Split-KV forward, for shapes with too few (batch, head, query block) units to fill the
 * GPU, e.g. decoding (Nq much smaller than Nk).  The key range is cut into num_splits
 * slices of whole key tiles; each (unit, slice) runs the same tiled online softmax and
 * writes its own normalised output O_s and log-sum-exp LSE_s (fp32) into the workspace;
 * a merge kernel on the same stream then writes
 *
 *     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
 *
 * which is exactly the softmax over the whole key range (the same identity the online
 * softmax's running rescale applies block by block; slices that see no key have
 * LSE_s = -inf and weight 0).  Results equal fa_fwd up to rounding.
 *
 * fa_splitkv_workspace_bytes: device bytes the workspace needs (0 for num_splits == 1);
 *   0 also for invalid sizes.
 * fa_splitkv_default_splits: a split count for sm_count SMs: 1 when the plain forward
 *   already has a unit per SM, else the count with the fewest key-tile steps on the busiest
 *   SM (waves x tiles per slice, plus one step per unit), keeping >= 4 key tiles per slice.
 * fa_fwd_splitkv: as fa_fwd (causal in {0, 1}), plus 1 <= num_splits <= 256 and a
 *   caller-owned device workspace of at least fa_splitkv_workspace_bytes bytes, 256-byte
 *   aligned, not overlapping any tensor (FA_ERR_INVALID_ARG / FA_ERR_MISALIGNED /
 *   FA_ERR_OVERLAP / FA_ERR_NOT_DEVICE_MEMORY otherwise).  The workspace is scratch: its
 *   contents are undefined afterwards, and two calls must not share one concurrently.
 *   num_splits == 1 needs no workspace and is fa_fwd.
 */
size_t fa_splitkv_workspace_bytes(int B, int Hq, int Nq, int d, int num_splits);
int fa_splitkv_default_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d, int sm_count);
int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *out, float *lse,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   int num_splits, void *workspace, size_t workspace_bytes, void *stream);
/* fa_fwd_splitkv_f16: the same on fp16 q, k, v and out (the merge writes fp16). */
int fa_fwd_splitkv_f16(const void *q, const void *k, const void *v, void *out, float *lse,
                       int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                       int num_splits, void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_fwd_splitkv_static -- fa_fwd_splitkv without a caller workspace and without any
 * allocation: the per-split partials go to a scratch array the library holds in static
 * device memory, FA_SPLITKV_STATIC_SCRATCH_BYTES (16 MiB) per device.  The paper has no
 * counterpart; it exists for callers that cannot allocate device memory around the call:
 * a plain C host program that embeds the library with no device allocator of its own, or a
 * serving loop whose device memory is planned up front, where a cudaMalloc in the middle
 * of a step would synchronise the device and could fail under memory pressure.
 *
 * Arguments, layouts, ownership and errors as fa_fwd_splitkv minus the workspace.  A problem
 * whose partials (fa_splitkv_workspace_bytes) exceed the static scratch returns
 * FA_ERR_SCRATCH_LIMIT and launches nothing; use fa_fwd_splitkv or fewer splits then.
 * Nothing in the scratch has to start at zero: each call writes every partial the merge
 * reads before the merge reads it.
 * The first call on each device does one-time set-up there (looks up the scratch address,
 * the same device probes as fa_fwd); make that first call before any stream capture.
 * All calls on one device share the one scratch array: two calls that may run at the same
 * time (different streams or threads, no ordering between them) race and corrupt each
 * other's results.  Calls ordered on one stream are safe.
 */
#define FA_SPLITKV_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
int fa_fwd_splitkv_static(const void *q, const void *k, const void *v, void *out, float *lse,
                          int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                          int num_splits, void *stream);

/*
 * fa_bwd -- exact attention backward: the gradients dQ, dK, dV of L = sum O (.) dO, with
 * S and P recomputed from Q, K, V and the forward's LSE instead of being stored (the
 * lpnh.cn YOLO11 / FlashAttention-2 article, section 2.3 "reverse recomputation"; the hwcomputing.csdn.net
 * FlashAttention article, "performance tuning"):
 *
 *     P = exp(scale Q K^T - LSE)  (masked),   dV = P^T dO,   dP = dO V^T,
 *     dS = P (.) (dP - D) with D_i = dO_i . O_i,   dQ = scale dS K,   dK = scale dS^T Q,
 *
 * dK and dV of a KV head summed over the query heads that share it (GQA).
 *
 *   q, out, dout [B, Nq, Hq, d] bf16, read only (out and lse from fa_fwd on the same q, k, v,
 *                scale and mask)
 *   k, v         [B, Nk, Hkv, d] bf16, read only
 *   lse          [B, Hq, Nq] fp32 (natural log), read only
 *   dq           [B, Nq, Hq, d] bf16, written;  dk, dv [B, Nk, Hkv, d] bf16, written
 *   d in {32, 64, 80, 96, 128} (FA_ERR_UNSUPPORTED_HEAD_DIM otherwise: S^T, dP^T, dV and dK
 *   share the 512 TMEM columns); causal in {0, 1}; the other sizes and the scale as fa_fwd
 *   workspace    caller-owned device scratch of at least fa_bwd_workspace_bytes bytes,
 *                256-byte aligned (fp32 dQ accumulator and D); no initial contents are
 *                needed (the call zeroes what it accumulates into); contents undefined
 *                afterwards; two calls must not share one concurrently.
 *
 * Three kernels run on `stream`: D and the zeroed accumulator, the main kernel (one unit per
 * (batch, KV head, 128-key tile); dQ accumulated with fp32 reductions), and dQ = bf16(scale
 * acc).  Errors as fa_fwd; the outputs must not overlap any input, each other or the
 * workspace (FA_ERR_OVERLAP).  With Nq == 0 or Nk == 0 the existing gradients are zero.
 */
size_t fa_bwd_workspace_bytes(int B, int Hq, int Nq, int d);
int fa_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
           void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
           void *workspace, size_t workspace_bytes, void *stream);
/* fa_bwd_f16: the same with fp16 q, k, v, out, dout, dq, dk, dv (P and dS rounded to fp16).
 * fa_bwd_window: fa_bwd for the sliding-window mask of fa_fwd_window (window >= 1; out and
 *   lse from fa_fwd_window with the same W); query tiles outside a key tile's band are skipped. */
int fa_bwd_f16(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
               void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
               void *workspace, size_t workspace_bytes, void *stream);
int fa_bwd_window(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
                  void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Key-sharded attention, for one sequence too long for one GPU: each GPU holds a shard of
 * K and V (keys key_offset .. key_offset + Nk - 1 of a sequence of Nk_total keys) and all of
 * Q, computes the partial (O_r, LSE_r) of its shard, the partials are exchanged (one
 * all-gather), and every GPU merges them with the log-sum-exp identity of the split-KV
 * forward (LSE = ln sum_r exp(LSE_r), O = sum_r exp(LSE_r - LSE) O_r).  The pages promise
 * sequence-dimension parallelism (the yunthe.com attention-variants page, closing paragraph of
 * its section "Flash Attention IO optimisation principle and code practice", on FlashAttention-2
 * parallelising over the sequence dimension; the lpnh.cn article, section 2.4, on FA-2's grid);
 * the exchange is the caller's (e.g. an NCCL all-gather of o_part and lse_part).
 *
 * fa_fwd_partial: q [B, Nq, Hq, d] bf16; k, v [B, Nk, Hkv, d] bf16 (the shard); o_part
 *   [B, Nq, Hq, d] fp32 (16-byte aligned) and lse_part [B, Hq, Nq] fp32, written: O of this
 *   shard's keys normalised by its own sum, and the natural-log LSE of those keys (rows that
 *   see none of them: O = 0, LSE = -inf).  causal: key g (global index) is visible to query
 *   i iff g <= i + Nk_total - Nq.  0 <= key_offset, key_offset + Nk <= Nk_total.  Other
 *   arguments and errors as fa_fwd.
 * fa_merge_partials: o_parts [R, B, Nq, Hq, d] fp32 and lse_parts [R, B, Hq, Nq] fp32 (R >= 1
 *   partials, stacked) -> out [B, Nq, Hq, d] bf16 and lse [B, Hq, Nq] fp32 (NULL: skipped).
 */
int fa_fwd_partial(const void *q, const void *k, const void *v, float *o_part, float *lse_part,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   int key_offset, int Nk_total, void *stream);
int fa_merge_partials(const float *o_parts, const float *lse_parts, int R, void *out, float *lse,
                      int B, int Hq, int Nq, int d, void *stream);

/* Human-readable text of a status code (static storage; never NULL). */
/*
 * fa_test_withheld_load -- the failure path of the forward kernel, for tests (no counterpart
 * on the pages: it exercises this library's own bounded waits).  Runs the d = 64 bf16 forward
 * (arguments, layouts and checks as fa_fwd with d = 64) in a build whose pipeline waits give
 * up after wait_limit_us microseconds (1 .. 1000000) and whose TMA producer leaves out one
 * K/V tile load: number `withheld_load` (>= 0) of its CTA, counted in issue order K_0, V_0,
 * K_1, V_1, ...  Nothing ever fills that slot, so the consumer's wait for it runs out: the
 * kernel records FA_ERR_DEVICE_TIMEOUT in the status word, every role unwinds (the producer
 * waits for its copies in flight, the MMA thread for its MMAs, TMEM is freed) and the kernel
 * returns.  fa_device_status then reports it; out and lse are undefined.  A later call runs
 * normally.  If the withheld load is past the last load a CTA issues, the call is an ordinary
 * forward.  Returns FA_ERR_INVALID_ARG for a negative index or a limit out of range.
 */
int fa_test_withheld_load(const void *q, const void *k, const void *v, void *out, float *lse,
                          int B, int Hq, int Hkv, int Nq, int Nk, float scale, int causal,
                          int withheld_load, unsigned int wait_limit_us, void *stream);

const char *fa_status_string(int status);

/*
 * fa_device_status -- synchronises `stream`, then returns and clears the current
 * device's kernel status word: FA_OK, or FA_ERR_DEVICE_TIMEOUT if a pipeline wait in a
 * forward or backward kernel ran out of time.  FA_ERR_CUDA if the synchronisation itself
 * failed.  If `detail` is not NULL it receives the raw status word (bits 8..15 name the
 * wait: 1-12 forward, 21-34 backward; bits 16.. the CTA).
 */
int fa_device_status(void *stream, int *detail);

/*
 * fa_tile_config -- the tiling fa_fwd uses for head dimension d (host only, no GPU):
 * rows per query tile, rows per key/value tile, query tiles per work unit, and the
 * number of key/value tile slots in the shared-memory ring.  Any output may be NULL.
 * Returns FA_ERR_UNSUPPORTED_HEAD_DIM for an unsupported d.
 */
int fa_tile_config(int d, int *block_q, int *block_k, int *q_tiles_per_unit, int *kv_slots);

/* Library ABI version (major * 100 + minor). */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_FA_H */

/*
 * attention_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.
 *
 * A plain, slow, obviously correct CPU implementation of the exact attention forward
 *
 *     O = softmax(scale * Q K^T  [+ causal mask]) V ,   LSE_i = ln sum_j exp(S_ij)
 *
 * in IEEE fp64, written straight from the definition.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or helper with the CUDA library; the two only see the same seeded
 * bf16 inputs.
 *
 * Where each step comes from:
 *  - the formula softmax(Q K^T / sqrt(d_k)) V and its three-step listing (scores,
 *    softmax, weighted sum), with S and P materialised as full N x N matrices:
 *    hwcomputing.csdn.net article on FlashAttention in CANN ops-transformer, section
 *    "where the memory black hole of standard attention comes from";
 *  - the softmax definition softmax(x_i) = e^{x_i} / sum_j e^{x_j}: same article,
 *    section "online softmax: keeping block-wise computation exact";
 *  - causal mask ("only see content before the current position"), sliding-window mask
 *    ("only look at the most recent positions") and no mask: same article,
 *    "performance tuning" item 3 (mask modes);
 *  - GQA: query head h uses KV head floor(h / n_rep), n_rep = Hq / Hkv, i.e. the
 *    repeat_interleave(n_rep, dim=1) expansion of K and V: "Transformer efficient
 *    attention: Flash Attention vs GQA" (yunthe.com), section "GQA principle and
 *    implementation";
 *  - tensor layout [batch, seq, heads, head_dim]: same yunthe.com page, the
 *    flash_attn_func call in section "Flash Attention IO optimisation".
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - the causal mask keeps the diagonal (key j visible to query i iff j <= i) and,
 *    for Nq != Nk, is aligned to the bottom-right: j <= i + (Nk - Nq);
 *  - the sliding window of W >= 1 keys is causal and ends at that diagonal:
 *    i + (Nk - Nq) - W < j <= i + (Nk - Nq);
 *  - a row with no visible key (only possible when Nq > Nk under the causal mask,
 *    or Nk == 0) has O = 0 and LSE = -inf, the limit of an empty sum;
 *  - LSE is the natural-log log-sum-exp of the scaled, masked logits;
 *  - inputs are bf16 (or, for the fp16 variant of the "performance tuning" data-type
 *    item of the same article, IEEE binary16) bit patterns, widened exactly to fp64;
 *    nothing is rounded in between;
 *  - FP8 inputs (the FlashAttention-3 FP8 forward of the datacanvas.csdn.net head-dim
 *    page) are OCP E4M3 bytes with one dequantisation factor per tensor: Q = dq * q8,
 *    K = dk * k8, V = dv * v8, after which the definition is unchanged.
 *
 * Softmax is taken in two passes over the materialised row (row max M_i first,
 * then exp(S_ij - M_i)), the textbook way to keep exp() in range.
 *
 * The backward pass (oracle_attention_bwd) is the gradient of L = sum O (.) dO through
 * the same definition: the pages ask for it by recomputation from Q, K, V (hwcomputing
 * article, "performance tuning"; the lpnh.cn YOLO11 / FlashAttention-2 article,
 * section 2.3 "reverse recomputation", on recomputing S and P in the backward pass).  With P the probability
 * matrix of the forward, the chain rule through O = P V and the row softmax gives
 *     dV = P^T dO,  dP = dO V^T,  dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
 *     dQ = scale dS K,  dK = scale dS^T Q,
 * with dK and dV of a KV head summed over the query heads that share it (GQA).
 *
 * Compile-time ORACLE_PLANT_* macros build deliberately wrong variants; the test
 * suite uses them to show that its pins catch each kind of mistake.  A normal build
 * defines none of them.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL -1
#define ORACLE_ENOMEM -2
#define ORACLE_ETHREAD -3

static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; exponent 0 is
 * subnormal (fraction * 2^-9); S.1111.111 is NaN; there is no infinity (max 448). */
static double e4m3_bits_to_double(uint8_t bits) {
    const int e = (bits >> 3) & 0xf, frac = bits & 0x7;
    double mag;
    if (e == 0xf && frac == 0x7) return NAN;
    if (e == 0) mag = ldexp((double)frac, -9);
#ifdef ORACLE_PLANT_E4M3_BIAS
    else mag = ldexp((double)(8 + frac), e - 11);
#else
    else mag = ldexp((double)(8 + frac), e - 10);
#endif
    return (bits & 0x80) ? -mag : mag;
}

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits;
 * exponent 0 is subnormal (fraction * 2^-24), exponent 31 is inf/NaN. */
static double f16_bits_to_double(uint16_t bits) {
    const int e = (bits >> 10) & 0x1f, frac = bits & 0x3ff;
    double mag;
    if (e == 0) mag = ldexp((double)frac, -24);
    else if (e == 31) mag = frac ? NAN : INFINITY;
#ifdef ORACLE_PLANT_F16_BIAS
    else mag = ldexp((double)(1024 + frac), e - 24);
#else
    else mag = ldexp((double)(1024 + frac), e - 25);
#endif
    return (bits & 0x8000) ? -mag : mag;
}

typedef struct {
    const uint16_t *q, *k, *v;
    int B, Hq, Hkv, Nq, Nk, d;
    double scale;
    int causal;
    int window;     /* 0: no window; W >= 1: sliding window of W keys (implies causal) */
    int elem_f16;   /* inputs are fp16 (1) or bf16 (0) bit patterns */
    const uint8_t *q8, *k8, *v8;   /* non-NULL: E4M3 inputs (q, k, v unused) */
    double dq, dk, dv;             /* dequantisation factors of the E4M3 inputs */
} problem_t;

static double elem(const problem_t *p, uint16_t bits) {
    return p->elem_f16 ? f16_bits_to_double(bits) : bf16_bits_to_double(bits);
}

static int kv_head_of(const problem_t *p, int hq) {
#ifdef ORACLE_PLANT_GQA_MODULO
    return hq % p->Hkv;
#else
    return hq / (p->Hq / p->Hkv);
#endif
}

static int key_visible(const problem_t *p, int i, int j) {
    const long diag = (long)i + (long)(p->Nk - p->Nq);   /* last key row i may see */
    if (p->window > 0) {
#ifdef ORACLE_PLANT_WINDOW_OFF_BY_ONE
        if ((long)j < diag - p->window) return 0;
#else
        if ((long)j <= diag - p->window) return 0;
#endif
    }
    if (!p->causal && p->window == 0) return 1;
#ifdef ORACLE_PLANT_CAUSAL_STRICT
    return (long)j < diag;
#else
    return (long)j <= diag;
#endif
}

static double q_at(const problem_t *p, int b, int i, int h, int c) {
    const size_t at = (((size_t)b * p->Nq + i) * p->Hq + h) * p->d + c;
    return p->q8 ? p->dq * e4m3_bits_to_double(p->q8[at]) : elem(p, p->q[at]);
}
static double k_at(const problem_t *p, int b, int j, int g, int c) {
    const size_t at = (((size_t)b * p->Nk + j) * p->Hkv + g) * p->d + c;
    return p->k8 ? p->dk * e4m3_bits_to_double(p->k8[at]) : elem(p, p->k[at]);
}
static double v_at(const problem_t *p, int b, int j, int g, int c) {
#ifdef ORACLE_PLANT_TRANSPOSE_V
    c = p->d - 1 - c;
#endif
    const size_t at = (((size_t)b * p->Nk + j) * p->Hkv + g) * p->d + c;
    return p->v8 ? p->dv * e4m3_bits_to_double(p->v8[at]) : elem(p, p->v[at]);
}

/*
 * One query row of one (b, hq): fills srow[0..Nk) with S_i. (scores, then masked),
 * turns it into the probability row P_i. in place, and writes O_i. (d values) and
 * LSE_i.  Step numbers follow the three-step standard listing.
 */
static void attention_row(const problem_t *p, int b, int hq, int i, double *srow,
                          double *o_row, double *lse_out) {
    const int g = kv_head_of(p, hq);
    const int Nk = p->Nk, d = p->d;

    /* step 1: scores S_ij = scale * sum_c Q[i,c] K[j,c]; masked entries -> -inf */
    for (int j = 0; j < Nk; ++j) {
        if (!key_visible(p, i, j)) { srow[j] = -INFINITY; continue; }
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += q_at(p, b, i, hq, c) * k_at(p, b, j, g, c);
#ifdef ORACLE_PLANT_NO_SCALE
        srow[j] = acc;
#else
        srow[j] = p->scale * acc;
#endif
    }

    /* step 2: softmax over the row, two passes: M = max_j S_ij, Z = sum_j exp(S_ij - M) */
    double M = -INFINITY;
    for (int j = 0; j < Nk; ++j) if (srow[j] > M) M = srow[j];
    if (M == -INFINITY) {               /* no visible key: empty sum */
        for (int c = 0; c < d; ++c) o_row[c] = 0.0;
        for (int j = 0; j < Nk; ++j) srow[j] = 0.0;
        *lse_out = -INFINITY;
        return;
    }
    double Z = 0.0;
    for (int j = 0; j < Nk; ++j) {
        srow[j] = exp(srow[j] - M);     /* exp(-inf) = 0 for masked keys */
        Z += srow[j];
    }
#ifndef ORACLE_PLANT_NO_NORMALIZE
    for (int j = 0; j < Nk; ++j) srow[j] /= Z;
#endif
#ifdef ORACLE_PLANT_LSE_NO_MAX
    *lse_out = log(Z);
#else
    *lse_out = M + log(Z);
#endif

    /* step 3: weighted sum O_i. = sum_j P_ij V_j. */
    for (int c = 0; c < d; ++c) o_row[c] = 0.0;
    for (int j = 0; j < Nk; ++j) {
        const double pij = srow[j];
        if (pij == 0.0) continue;
        for (int c = 0; c < d; ++c) o_row[c] += pij * v_at(p, b, j, g, c);
    }
}

/* ---- full forward: S and P materialised per (b, hq), rows split across threads ---- */

typedef struct {
    const problem_t *p;
    int b, hq, i0, i1;
    double *S;          /* Nq x Nk for this (b, hq), shared; each thread owns its rows */
    double *out, *lse;  /* whole outputs */
    double *probs;      /* optional [B,Hq,Nq,Nk] copy of P */
} head_job_t;

static void *head_rows_worker(void *arg) {
    head_job_t *jb = (head_job_t *)arg;
    const problem_t *p = jb->p;
    for (int i = jb->i0; i < jb->i1; ++i) {
        double *srow = jb->S + (size_t)i * p->Nk;
        double *o_row = jb->out + (((size_t)jb->b * p->Nq + i) * p->Hq + jb->hq) * p->d;
        double *l = jb->lse + ((size_t)jb->b * p->Hq + jb->hq) * p->Nq + i;
        attention_row(p, jb->b, jb->hq, i, srow, o_row, l);
        if (jb->probs) {
            double *dst = jb->probs + (((size_t)jb->b * p->Hq + jb->hq) * p->Nq + i) * p->Nk;
            memcpy(dst, srow, sizeof(double) * (size_t)p->Nk);
        }
    }
    return NULL;
}

static int check_problem(const problem_t *p) {
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->Nq < 0 || p->Nk < 0 || p->d <= 0) return 0;
    if (p->Hq % p->Hkv != 0) return 0;
    if (p->window < 0) return 0;
    if (!isfinite(p->scale)) return 0;
    return 1;
}

static int run_full(const problem_t *p, double *out, double *lse, double *probs, int nthreads) {
    if (!check_problem(p)) return ORACLE_EINVAL;
    if (nthreads < 1) nthreads = 1;
    if (p->B == 0 || p->Nq == 0) return ORACLE_OK;
    const size_t nk_alloc = p->Nk > 0 ? (size_t)p->Nk : 1;
    double *S = (double *)malloc(sizeof(double) * (size_t)p->Nq * nk_alloc);
    if (!S) return ORACLE_ENOMEM;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    head_job_t *jobs = (head_job_t *)malloc(sizeof(head_job_t) * (size_t)nthreads);
    if (!tid || !jobs) { free(S); free(tid); free(jobs); return ORACLE_ENOMEM; }
    int rc = ORACLE_OK;
    for (int b = 0; b < p->B && rc == ORACLE_OK; ++b) {
        for (int hq = 0; hq < p->Hq && rc == ORACLE_OK; ++hq) {
            int nt = nthreads < p->Nq ? nthreads : p->Nq;
            int started = 0;
            for (int t = 0; t < nt; ++t) {
                jobs[t] = (head_job_t){p, b, hq, (int)((long)p->Nq * t / nt),
                                       (int)((long)p->Nq * (t + 1) / nt), S, out, lse, probs};
                if (nt == 1) { head_rows_worker(&jobs[t]); continue; }
                if (pthread_create(&tid[t], NULL, head_rows_worker, &jobs[t]) != 0) {
                    rc = ORACLE_ETHREAD;
                    break;
                }
                ++started;
            }
            for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
        }
    }
    free(S);
    free(tid);
    free(jobs);
    return rc;
}

/*
 * oracle_attention_fwd: the whole forward.
 *   q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d]: bf16 (elem_f16 = 0) or fp16 (1) bit patterns (host memory).
 *   causal in {0,1}; window = 0 (none) or W >= 1 keys (sliding window, causal).
 *   out [B,Nq,Hq,d] fp64, lse [B,Hq,Nq] fp64 (natural log).
 * Returns 0, or a negative code (bad sizes, no memory, thread failure).
 */
int oracle_attention_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         double *out, double *lse, int B, int Hq, int Hkv, int Nq, int Nk,
                         int d, double scale, int causal, int window, int elem_f16, int nthreads) {
    problem_t p = {q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal ? 1 : 0, window, elem_f16 ? 1 : 0, NULL, NULL, NULL, 1.0, 1.0, 1.0};
    return run_full(&p, out, lse, NULL, nthreads);
}

/*
 * oracle_attention_probs: as oracle_attention_fwd, and also copies the
 * probability matrix P into probs [B,Hq,Nq,Nk] (tiny problems only).
 */
int oracle_attention_probs(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           double *out, double *lse, double *probs, int B, int Hq, int Hkv,
                           int Nq, int Nk, int d, double scale, int causal, int window, int elem_f16) {
    problem_t p = {q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal ? 1 : 0, window, elem_f16 ? 1 : 0, NULL, NULL, NULL, 1.0, 1.0, 1.0};
    return run_full(&p, out, lse, probs, 1);
}

/* ---- selected rows: the same definition evaluated only for listed (b, hq, i) ---- */

typedef struct {
    const problem_t *p;
    const int32_t *rows;   /* triples (b, hq, i) */
    long r0, r1;
    double *out_rows;      /* [nrows, d] */
    double *lse_rows;      /* [nrows] */
    int rc;
} rows_job_t;

static void *rows_worker(void *arg) {
    rows_job_t *jb = (rows_job_t *)arg;
    const problem_t *p = jb->p;
    double *srow = (double *)malloc(sizeof(double) * (size_t)(p->Nk > 0 ? p->Nk : 1));
    if (!srow) { jb->rc = ORACLE_ENOMEM; return NULL; }
    for (long r = jb->r0; r < jb->r1; ++r) {
        int b = jb->rows[3 * r], hq = jb->rows[3 * r + 1], i = jb->rows[3 * r + 2];
        attention_row(p, b, hq, i, srow, jb->out_rows + r * p->d, jb->lse_rows + r);
    }
    free(srow);
    return NULL;
}

/* O and LSE of the listed rows only (shared by the bit-pattern and E4M3 entry points). */
static int run_rows(const problem_t *pp, const int32_t *rows, long nrows, double *out_rows, double *lse_rows,
                    int nthreads) {
    const problem_t p = *pp;
    const int B = p.B, Hq = p.Hq, Nq = p.Nq;
    if (!check_problem(&p) || nrows < 0) return ORACLE_EINVAL;
    for (long r = 0; r < nrows; ++r) {
        int b = rows[3 * r], hq = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || hq < 0 || hq >= Hq || i < 0 || i >= Nq) return ORACLE_EINVAL;
    }
    if (nthreads < 1) nthreads = 1;
    if (nrows == 0) return ORACLE_OK;
    int nt = (long)nthreads < nrows ? nthreads : (int)nrows;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    rows_job_t *jobs = (rows_job_t *)malloc(sizeof(rows_job_t) * (size_t)nt);
    if (!tid || !jobs) { free(tid); free(jobs); return ORACLE_ENOMEM; }
    int started = 0, rc = ORACLE_OK;
    for (int t = 0; t < nt; ++t) {
        jobs[t] = (rows_job_t){&p, rows, nrows * t / nt, nrows * (t + 1) / nt, out_rows, lse_rows, 0};
        if (nt == 1) { rows_worker(&jobs[t]); continue; }
        if (pthread_create(&tid[t], NULL, rows_worker, &jobs[t]) != 0) { rc = ORACLE_ETHREAD; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    for (int t = 0; t < nt && rc == ORACLE_OK; ++t) if (jobs[t].rc) rc = jobs[t].rc;
    free(tid);
    free(jobs);
    return rc;
}

/*
 * oracle_attention_rows: O and LSE of the listed rows only.
 *   rows: nrows triples (b, hq, i), each in range; out_rows [nrows, d]; lse_rows [nrows].
 */
int oracle_attention_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int32_t *rows, long nrows, double *out_rows, double *lse_rows,
                          int B, int Hq, int Hkv, int Nq, int Nk, int d, double scale,
                          int causal, int window, int elem_f16, int nthreads) {
    problem_t p = {q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal ? 1 : 0, window, elem_f16 ? 1 : 0,
                   NULL, NULL, NULL, 1.0, 1.0, 1.0};
    return run_rows(&p, rows, nrows, out_rows, lse_rows, nthreads);
}

/* oracle_attention_rows_fp8: the same for E4M3 inputs with dequantisation factors. */
int oracle_attention_rows_fp8(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8, const int32_t *rows,
                              long nrows, double *out_rows, double *lse_rows, int B, int Hq, int Hkv, int Nq, int Nk,
                              int d, double scale, double dq, double dk, double dv, int causal, int window,
                              int nthreads) {
    problem_t p = {NULL, NULL, NULL, B, Hq, Hkv, Nq, Nk, d, scale, causal ? 1 : 0, window, 0, q8, k8, v8, dq, dk, dv};
    if (!q8 || !k8 || !v8) return ORACLE_EINVAL;
    return run_rows(&p, rows, nrows, out_rows, lse_rows, nthreads);
}

/* ---- backward: gradients of L = sum_{b,i,h,c} O[b,i,h,c] dO[b,i,h,c] ---- */

typedef struct {
    const problem_t *p;
    const uint16_t *dout;     /* dO bit patterns, [B,Nq,Hq,d] */
    double *dq, *dk, *dv;     /* [B,Nq,Hq,d], [B,Nk,Hkv,d], [B,Nk,Hkv,d] */
    int t, nt;                /* this worker takes (b, g) pairs t, t + nt, ... */
    int rc;
} bwd_job_t;

static double do_at(const bwd_job_t *jb, int b, int i, int h, int c) {
    const problem_t *p = jb->p;
    return elem(p, jb->dout[(((size_t)b * p->Nq + i) * p->Hq + h) * p->d + c]);
}

static void *bwd_worker(void *arg) {
    bwd_job_t *jb = (bwd_job_t *)arg;
    const problem_t *p = jb->p;
    const int Nk = p->Nk, d = p->d, n_rep = p->Hq / p->Hkv;
    const size_t nk = Nk > 0 ? (size_t)Nk : 1;
    double *prow = (double *)malloc(sizeof(double) * nk);
    double *dprow = (double *)malloc(sizeof(double) * nk);
    double *orow = (double *)malloc(sizeof(double) * (size_t)d);
    if (!prow || !dprow || !orow) { free(prow); free(dprow); free(orow); jb->rc = ORACLE_ENOMEM; return NULL; }
    for (long pair = jb->t; pair < (long)p->B * p->Hkv; pair += jb->nt) {
        const int b = (int)(pair / p->Hkv), g = (int)(pair % p->Hkv);
        for (int r = 0; r < n_rep; ++r) {
            const int hq = g * n_rep + r;    /* the query heads that read KV head g */
            if (kv_head_of(p, hq) != g) continue;
            for (int i = 0; i < p->Nq; ++i) {
                double lse;
                attention_row(p, b, hq, i, prow, orow, &lse);   /* prow = P_i. */
                /* dP_ij = dO_i . V_j ; D_i = sum_j P_ij dP_ij */
                double D = 0.0;
                for (int j = 0; j < Nk; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += do_at(jb, b, i, hq, c) * v_at(p, b, j, g, c);
                    dprow[j] = acc;
                    D += prow[j] * acc;
                }
                double *dqi = jb->dq + (((size_t)b * p->Nq + i) * p->Hq + hq) * d;
                for (int j = 0; j < Nk; ++j) {
                    const double pij = prow[j];
                    if (pij == 0.0) continue;
#ifdef ORACLE_PLANT_BWD_NO_D
                    const double dsij = pij * dprow[j];
#else
                    const double dsij = pij * (dprow[j] - D);
#endif
#ifdef ORACLE_PLANT_BWD_DQ_NO_SCALE
                    const double sq = 1.0;
#else
                    const double sq = p->scale;
#endif
                    double *dkj = jb->dk + (((size_t)b * Nk + j) * p->Hkv + g) * d;
                    double *dvj = jb->dv + (((size_t)b * Nk + j) * p->Hkv + g) * d;
                    for (int c = 0; c < d; ++c) {
                        dqi[c] += sq * dsij * k_at(p, b, j, g, c);
                        dkj[c] += p->scale * dsij * q_at(p, b, i, hq, c);
#ifdef ORACLE_PLANT_BWD_DV_NO_P
                        dvj[c] += do_at(jb, b, i, hq, c);
#else
                        dvj[c] += pij * do_at(jb, b, i, hq, c);
#endif
                    }
                }
            }
        }
    }
    free(prow); free(dprow); free(orow);
    return NULL;
}

/*
 * oracle_attention_bwd: dQ, dK, dV of L = sum O (.) dO.
 *   q/k/v as oracle_attention_fwd; dout [B,Nq,Hq,d] bit patterns of the same element type.
 *   dq [B,Nq,Hq,d], dk/dv [B,Nk,Hkv,d] fp64, overwritten.
 */
int oracle_attention_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                         double *dq, double *dk, double *dv, int B, int Hq, int Hkv, int Nq, int Nk,
                         int d, double scale, int causal, int window, int elem_f16, int nthreads) {
    problem_t p = {q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal ? 1 : 0, window, elem_f16 ? 1 : 0, NULL, NULL, NULL, 1.0, 1.0, 1.0};
    if (!check_problem(&p)) return ORACLE_EINVAL;
    memset(dq, 0, sizeof(double) * (size_t)B * Nq * Hq * d);
    memset(dk, 0, sizeof(double) * (size_t)B * Nk * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)B * Nk * Hkv * d);
    if (nthreads < 1) nthreads = 1;
    const long pairs = (long)B * Hkv;
    if (pairs == 0 || Nq == 0 || Nk == 0) return ORACLE_OK;
    int nt = (long)nthreads < pairs ? nthreads : (int)pairs;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    bwd_job_t *jobs = (bwd_job_t *)malloc(sizeof(bwd_job_t) * (size_t)nt);
    if (!tid || !jobs) { free(tid); free(jobs); return ORACLE_ENOMEM; }
    int started = 0, rc = ORACLE_OK;
    for (int t = 0; t < nt; ++t) {
        jobs[t] = (bwd_job_t){&p, dout, dq, dk, dv, t, nt, 0};
        if (nt == 1) { bwd_worker(&jobs[t]); continue; }
        if (pthread_create(&tid[t], NULL, bwd_worker, &jobs[t]) != 0) { rc = ORACLE_ETHREAD; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    for (int t = 0; t < nt && rc == ORACLE_OK; ++t) if (jobs[t].rc) rc = jobs[t].rc;
    free(tid);
    free(jobs);
    return rc;
}

/*
 * oracle_attention_fwd_fp8 / oracle_attention_rows_fp8: the same forward (all rows, or
 * listed rows) for E4M3 inputs q8, k8, v8 (one byte per element, layouts as above) with
 * dequantisation factors dq, dk, dv: Q = dq * q8 and so on.
 */
int oracle_attention_fwd_fp8(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8, double *out, double *lse,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d, double scale, double dq, double dk,
                             double dv, int causal, int window, int nthreads) {
    problem_t p = {NULL, NULL, NULL, B, Hq, Hkv, Nq, Nk, d, scale, causal ? 1 : 0, window, 0, q8, k8, v8, dq, dk, dv};
    if (!q8 || !k8 || !v8 || !isfinite(dq) || !isfinite(dk) || !isfinite(dv)) return ORACLE_EINVAL;
    return run_full(&p, out, lse, NULL, nthreads);
}

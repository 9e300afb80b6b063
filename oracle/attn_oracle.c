/*
 * attn_oracle.c -- plain fp64 CPU attention. TEST INFRASTRUCTURE ONLY.
 *
 * This is the oracle that the CUDA path is checked against. It is slow and
 * literal on purpose. For every query row it materialises that row of scores,
 * applies the mask, takes a two-pass softmax (max, then sum of exponentials),
 * and forms the probability-weighted sum of value rows. Nothing is tiled,
 * fused or reordered. Only the tests, the smoke check and the benchmark's CPU
 * baseline may call it. The library never does, and the two share no code.
 *
 * What it computes, and where that is defined:
 *  - Scores = Q K^T / sqrt(d_k), a row-wise softmax whose rows are
 *    probabilities summing to 1, and Attention(Q,K,V) = softmax(Scores) V:
 *    "Self-attention, CUDA kernels and FlashAttention" (russian.itimpress.au),
 *    section 1, the Scores and Attention(Q,K,V) formulas. The scale is passed
 *    in explicitly; callers use 1/sqrt(D) unless a workload fixes another.
 *  - Several heads run the same computation independently: same page,
 *    section 1, last paragraph.
 *  - causal=True "for autoregressive models": "Flash Attention" skill page
 *    (hermes-agent-app.ru), Scenario 2, step 2. Reading taken: key j is
 *    visible to query i iff j <= i + (Lk - Lq) (bottom-right alignment; the
 *    same as top-left when Lq == Lk, and a single decode query sees all keys).
 *  - Sliding-window (local) attention, window_size = (left, right): same page,
 *    Scenario 2, step 3 ("attention only to a window of tokens before/after").
 *    Reading taken: with i' = i + (Lk - Lq), key j is visible iff
 *    i' - left <= j <= i' + right, a negative bound meaning unbounded on that
 *    side; causal=True caps the right side at i' (right = 0).
 *  - Fewer K/V heads than query heads (multi-query / grouped-query): same
 *    page, Scenario 2, step 3. Reading taken: consecutive query heads share a
 *    K/V head, h_kv = h_q / (H_q / H_kv).
 *  - Only small normalisation statistics are kept for the backward pass:
 *    "Self-attention, CUDA kernels and FlashAttention", section 3. Reading
 *    taken: lse = m + ln(sum_j exp(s_j - m)), natural log, over the scaled,
 *    masked scores of the row.
 *  - A row with no visible key has no softmax. Reading taken: O = 0 and
 *    lse = -inf.
 *  - Backward pass: only the normalisation statistics are kept from the forward
 *    pass, and the attention tiles are recomputed during backpropagation: "Self-
 *    attention, CUDA kernels and FlashAttention", section 3 (recomputation). The
 *    pages print no gradient formulas. What the backward pass computes is the
 *    gradient of a scalar loss through the section 1 definition, given dO =
 *    dLoss/dO. Here it is written out by the chain rule for one query row i:
 *    P_ij are the row's probabilities, dV_j += P_ij dO_i, dP_ij = dO_i . v_j,
 *    delta_i = sum_j P_ij dP_ij (the softmax Jacobian applied to the row of dP),
 *    dS_ij = P_ij (dP_ij - delta_i), dQ_i = scale sum_j dS_ij k_j and dK_j +=
 *    scale dS_ij q_i. Masked keys have P_ij = 0 and so take no part. Grouped K/V
 *    heads collect the gradients of every query head that reads them.
 *  - Paged KV cache: storage in fixed-size blocks plus a table from logical
 *    position to physical block, resolved for every position inside the
 *    attention: "Fast attention kernels and operator fusion" (the-ai.news),
 *    section "FlashAttention-style attention and paged attention". Layout
 *    taken: cache[num_blocks][H_kv][block_size][D]; token t of sequence s is
 *    row t % block_size of physical block block_table[s][t / block_size].
 *  - Prefill over a paged cache: the same page says the kernel translates every
 *    position through the block table, and that long prefill is where the T x T
 *    score matrix hurts. Reading taken: a chunk of q_len queries per sequence
 *    occupies its last q_len positions (causal alignment bottom-right, as for
 *    dense attention with Lq = q_len, Lk = seq_len).
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared -pthread (no fast-math, so
 * every operation is the IEEE double operation written here).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_INDEX (-2)
#define ORACLE_ERR_NOMEM (-3)

/*
 * One query row of attention.
 *   qi      : the query row, D values
 *   K, V    : Lk rows of D values each
 *   lo, hi  : keys lo .. hi-1 are visible (the mask is one contiguous range)
 *   s       : scratch for the Lk scores
 *   o       : output row, D values
 *   lse     : output log-sum-exp of the row (may be NULL)
 *   p_out   : if not NULL, receives the Lk softmax probabilities
 */
static void attention_row(const double* qi, const double* K, const double* V,
                          int64_t Lk, int64_t lo, int64_t hi, int64_t D, double scale,
                          double* s, double* o, double* lse, double* p_out) {
    int64_t j, d;
    /* Scores: scale * (q_i . k_j); masked keys get -inf. */
    for (j = 0; j < Lk; ++j) {
        if (j >= lo && j < hi) {
            double dot = 0.0;
            for (d = 0; d < D; ++d) dot += qi[d] * K[j * D + d];
            s[j] = scale * dot;
        } else {
            s[j] = -INFINITY;
        }
    }
    /* Pass 1: the row maximum. */
    double m = -INFINITY;
    for (j = 0; j < Lk; ++j)
        if (s[j] > m) m = s[j];
    for (d = 0; d < D; ++d) o[d] = 0.0;
    if (m == -INFINITY) { /* no visible key */
        if (lse) *lse = -INFINITY;
        if (p_out)
            for (j = 0; j < Lk; ++j) p_out[j] = 0.0;
        return;
    }
    /* Pass 2: the normaliser l = sum_j exp(s_j - m). */
    double l = 0.0;
    for (j = 0; j < Lk; ++j) l += exp(s[j] - m);
    /* Probabilities P_j = exp(s_j - m) / l and O = sum_j P_j v_j. */
    for (j = 0; j < Lk; ++j) {
        double p = exp(s[j] - m) / l;
        if (p_out) p_out[j] = p;
        for (d = 0; d < D; ++d) o[d] += p * V[j * D + d];
    }
    if (lse) *lse = m + log(l);
}

/*
 * Keys visible to query row i: [*lo, *hi). With i' = i + (Lk - Lq) (bottom-right
 * alignment), key j is visible iff i' - left <= j <= i' + right; a negative left or
 * right leaves that side unbounded, and causal sets right = 0.
 */
static void visible_range(int64_t i, int64_t Lq, int64_t Lk, int causal, int64_t left,
                          int64_t right, int64_t* lo, int64_t* hi) {
    int64_t last = i + (Lk - Lq); /* i' */
    int64_t a = 0, b = Lk;
    if (causal) right = 0;
    if (left >= 0 && last - left > a) a = last - left;
    if (right >= 0 && last + right + 1 < b) b = last + right + 1;
    if (b < a) b = a;
    *lo = a;
    *hi = b;
}

/* ------------------------------------------------------------------------ */
/* Dense attention over [B, H, L, D] tensors.                               */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *q, *k, *v;
    double *out, *lse, *probs;
    int64_t B, Hq, Hkv, Lq, Lk, D;
    double scale;
    int causal;
    int64_t win_left, win_right; /* -1: unbounded */
    const int64_t* rows; /* NULL: every row, in order */
    int64_t n_rows;
    int64_t next; /* shared work counter */
    int status;
} dense_job;

static void* dense_worker(void* arg) {
    dense_job* J = (dense_job*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)(J->Lk > 0 ? J->Lk : 1));
    if (!s) {
        __atomic_store_n(&J->status, ORACLE_ERR_NOMEM, __ATOMIC_RELAXED);
        return NULL;
    }
    const int64_t group = J->Hq / J->Hkv;
    for (;;) {
        int64_t r = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (r >= J->n_rows) break;
        /* Flattened row id = (b * Hq + h) * Lq + i. */
        int64_t id = J->rows ? J->rows[r] : r;
        int64_t i = id % J->Lq;
        int64_t bh = id / J->Lq;
        int64_t h = bh % J->Hq;
        int64_t b = bh / J->Hq;
        int64_t hkv = h / group;
        const double* qi = J->q + id * J->D;
        const double* K = J->k + (b * J->Hkv + hkv) * J->Lk * J->D;
        const double* V = J->v + (b * J->Hkv + hkv) * J->Lk * J->D;
        double* o = J->out + r * J->D;
        double* lse = J->lse ? J->lse + r : NULL;
        double* p = J->probs ? J->probs + r * J->Lk : NULL;
        int64_t lo, hi;
        visible_range(i, J->Lq, J->Lk, J->causal, J->win_left, J->win_right, &lo, &hi);
        attention_row(qi, K, V, J->Lk, lo, hi, J->D, J->scale, s, o, lse, p);
    }
    free(s);
    return NULL;
}

static int run_dense(dense_job* J, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (J->n_rows < nthreads) nthreads = (int)(J->n_rows > 0 ? J->n_rows : 1);
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&tid[started], NULL, dense_worker, J) == 0) ++started;
    }
    dense_worker(J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return J->status;
}

static int check_dims(int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk, int64_t D) {
    if (B < 0 || Hq < 1 || Hkv < 1 || Lq < 0 || Lk < 0 || D < 1) return ORACLE_ERR_ARG;
    if (Hq % Hkv != 0) return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

/*
 * out[B,Hq,Lq,D], lse[B,Hq,Lq] (lse may be NULL) from q[B,Hq,Lq,D],
 * k[B,Hkv,Lk,D], v[B,Hkv,Lk,D].
 */
int oracle_attn_fwd(const double* q, const double* k, const double* v, double* out,
                    double* lse, int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                    int64_t D, double scale, int causal, int nthreads) {
    int rc = check_dims(B, Hq, Hkv, Lq, Lk, D);
    if (rc) return rc;
    dense_job J = {q, k, v, out, lse, NULL, B, Hq, Hkv, Lq, Lk, D, scale, causal, -1, -1,
                   NULL, B * Hq * Lq, 0, ORACLE_OK};
    return run_dense(&J, nthreads);
}

/* Sliding-window attention: as oracle_attn_fwd with window (left, right), -1 = unbounded. */
int oracle_attn_fwd_window(const double* q, const double* k, const double* v, double* out,
                           double* lse, int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq,
                           int64_t Lk, int64_t D, double scale, int causal, int64_t left,
                           int64_t right, int nthreads) {
    int rc = check_dims(B, Hq, Hkv, Lq, Lk, D);
    if (rc) return rc;
    if (left < -1 || right < -1) return ORACLE_ERR_ARG;
    dense_job J = {q, k, v, out, lse, NULL, B, Hq, Hkv, Lq, Lk, D, scale, causal, left, right,
                   NULL, B * Hq * Lq, 0, ORACLE_OK};
    return run_dense(&J, nthreads);
}

/*
 * Selected rows only. rows[r] is a flattened row id (b*Hq + h)*Lq + i;
 * out[r, D] and lse[r] receive that row's result.
 */
int oracle_attn_fwd_rows(const double* q, const double* k, const double* v,
                         const int64_t* rows, int64_t n_rows, double* out, double* lse,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                         int64_t D, double scale, int causal, int nthreads) {
    int rc = check_dims(B, Hq, Hkv, Lq, Lk, D);
    if (rc) return rc;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= B * Hq * Lq) return ORACLE_ERR_INDEX;
    dense_job J = {q, k, v, out, lse, NULL, B, Hq, Hkv, Lq, Lk, D, scale, causal, -1, -1,
                   rows, n_rows, 0, ORACLE_OK};
    return run_dense(&J, nthreads);
}

/* The softmax matrix itself: probs[B,Hq,Lq,Lk] (small problems only). */
int oracle_attn_probs(const double* q, const double* k, const double* v, double* probs,
                      int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk, int64_t D,
                      double scale, int causal) {
    int rc = check_dims(B, Hq, Hkv, Lq, Lk, D);
    if (rc) return rc;
    double* out = (double*)malloc(sizeof(double) * (size_t)(B * Hq * Lq * D + 1));
    if (!out) return ORACLE_ERR_NOMEM;
    dense_job J = {q, k, v, out, NULL, probs, B, Hq, Hkv, Lq, Lk, D, scale, causal, -1, -1,
                   NULL, B * Hq * Lq, 0, ORACLE_OK};
    rc = run_dense(&J, 1);
    free(out);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Paged decode: one query per sequence, keys resolved through a table.     */
/* ------------------------------------------------------------------------ */

typedef struct {
    const double *q, *kc, *vc;
    const int32_t *block_table, *seq_lens;
    double *out, *lse;
    int64_t block_size, num_seqs, Hq, Hkv, D, max_blocks, num_blocks;
    double scale;
    int64_t next;
    int status;
} paged_job;

static void* paged_worker(void* arg) {
    paged_job* J = (paged_job*)arg;
    const int64_t cap = J->max_blocks * J->block_size;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)(cap * J->D + 1));
    double* Vd = (double*)malloc(sizeof(double) * (size_t)(cap * J->D + 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)(cap + 1));
    if (!Kd || !Vd || !s) {
        __atomic_store_n(&J->status, ORACLE_ERR_NOMEM, __ATOMIC_RELAXED);
        free(Kd); free(Vd); free(s);
        return NULL;
    }
    const int64_t group = J->Hq / J->Hkv;
    for (;;) {
        int64_t u = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (u >= J->num_seqs * J->Hkv) break;
        int64_t sq = u / J->Hkv, hkv = u % J->Hkv;
        int64_t len = J->seq_lens[sq];
        /* Gather this sequence's keys and values in logical order. */
        for (int64_t t = 0; t < len; ++t) {
            int64_t phys = J->block_table[sq * J->max_blocks + t / J->block_size];
            if (phys < 0 || phys >= J->num_blocks) {
                __atomic_store_n(&J->status, ORACLE_ERR_INDEX, __ATOMIC_RELAXED);
                len = 0;
                break;
            }
            const int64_t row = ((phys * J->Hkv + hkv) * J->block_size + t % J->block_size) * J->D;
            memcpy(Kd + t * J->D, J->kc + row, sizeof(double) * (size_t)J->D);
            memcpy(Vd + t * J->D, J->vc + row, sizeof(double) * (size_t)J->D);
        }
        /* The query heads of this K/V head attend over all len keys. */
        for (int64_t g = 0; g < group; ++g) {
            int64_t h = hkv * group + g;
            const double* qi = J->q + (sq * J->Hq + h) * J->D;
            attention_row(qi, Kd, Vd, len, 0, len, J->D, J->scale, s,
                          J->out + (sq * J->Hq + h) * J->D,
                          J->lse ? J->lse + sq * J->Hq + h : NULL, NULL);
        }
    }
    free(Kd); free(Vd); free(s);
    return NULL;
}

/*
 * q[num_seqs,Hq,D]; k_cache, v_cache [num_blocks,Hkv,block_size,D];
 * block_table[num_seqs,max_blocks]; seq_lens[num_seqs];
 * out[num_seqs,Hq,D]; lse[num_seqs,Hq] (may be NULL).
 */
int oracle_attn_paged(const double* q, const double* k_cache, const double* v_cache,
                      const int32_t* block_table, const int32_t* seq_lens, int64_t block_size,
                      double* out, double* lse, int64_t num_seqs, int64_t Hq, int64_t Hkv,
                      int64_t D, int64_t max_blocks, int64_t num_blocks, double scale,
                      int nthreads) {
    if (num_seqs < 0 || Hq < 1 || Hkv < 1 || D < 1 || block_size < 1 || max_blocks < 0 ||
        num_blocks < 0 || Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    for (int64_t s = 0; s < num_seqs; ++s)
        if (seq_lens[s] < 0 || seq_lens[s] > max_blocks * block_size) return ORACLE_ERR_INDEX;
    paged_job J = {q, k_cache, v_cache, block_table, seq_lens, out, lse, block_size,
                   num_seqs, Hq, Hkv, D, max_blocks, num_blocks, scale, 0, ORACLE_OK};
    int64_t units = num_seqs * Hkv;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (units < nthreads) nthreads = (int)(units > 0 ? units : 1);
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&tid[started], NULL, paged_worker, &J) == 0) ++started;
    paged_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return J.status;
}

/* ------------------------------------------------------------------------ */
/* Backward pass: gradients of a scalar loss through dense attention.       */
/* ------------------------------------------------------------------------ */

/*
 * Rounding sensitivity of the gradients, for the tests' tolerances (not part of the
 * gradient arithmetic). A kernel that rounds P and dS to a 16-bit type (relative
 * error u each) and computes delta_i from the rounded O (an error of at most
 * u A_i, A_i = sum_d |do_id o_id|) perturbs dS_ij by at most u (|dS_ij| + P_ij A_i)
 * and P_ij by u P_ij. To first order the gradient errors are then bounded by u times
 *   mQ_i = scale sum_j (|dS_ij| + P_ij A_i) |k_j|
 *   mK_j = scale sum_i (|dS_ij| + P_ij A_i) |q_i|
 *   mV_j = sum_i P_ij |do_i|        (elementwise over d)
 */

/*
 * One query row of the backward pass. Recomputes the row's probabilities p (with
 * attention_row), then the row of dP_ij = do_i . v_j over the visible keys, the
 * row's delta = sum_j P_ij dP_ij, and dS_ij = P_ij (dP_ij - delta).
 *   dqi      : receives dQ_i = scale sum_j dS_ij k_j (may be NULL)
 *   dK, dV   : Lk rows each, accumulated into (may be NULL):
 *              dV_j += P_ij do_i and dK_j += scale dS_ij q_i
 *   mq, mK, mV : the sensitivities mQ_i (D values) and mK_j, mV_j (Lk rows each,
 *              accumulated into); each may be NULL
 *   s, p, ds : scratch of Lk values; o : scratch of D values
 * Returns the row's delta (0 for a row with no visible key).
 */
static double backward_row(const double* qi, const double* doi, const double* K,
                           const double* V, int64_t Lk, int64_t lo, int64_t hi, int64_t D,
                           double scale, double* s, double* p, double* ds, double* o,
                           double* dqi, double* dK, double* dV, double* mq, double* mK,
                           double* mV) {
    int64_t j, d;
    attention_row(qi, K, V, Lk, lo, hi, D, scale, s, o, NULL, p);
    /* dP_ij = do_i . v_j (kept in ds for now) and delta = sum_j P_ij dP_ij. */
    double delta = 0.0;
    for (j = lo; j < hi; ++j) {
        double dot = 0.0;
        for (d = 0; d < D; ++d) dot += doi[d] * V[j * D + d];
        ds[j] = dot;
        delta += p[j] * dot;
    }
    /* dS_ij = P_ij (dP_ij - delta). */
    for (j = lo; j < hi; ++j) ds[j] = p[j] * (ds[j] - delta);
    if (dqi) {
        for (d = 0; d < D; ++d) dqi[d] = 0.0;
        for (j = lo; j < hi; ++j)
            for (d = 0; d < D; ++d) dqi[d] += ds[j] * K[j * D + d];
        for (d = 0; d < D; ++d) dqi[d] *= scale;
    }
    for (j = lo; j < hi; ++j) {
        if (dV)
            for (d = 0; d < D; ++d) dV[j * D + d] += p[j] * doi[d];
        if (dK)
            for (d = 0; d < D; ++d) dK[j * D + d] += scale * ds[j] * qi[d];
    }
    if (mq || mK || mV) {
        double A = 0.0;
        for (d = 0; d < D; ++d) A += fabs(doi[d] * o[d]);
        if (mq)
            for (d = 0; d < D; ++d) mq[d] = 0.0;
        for (j = lo; j < hi; ++j) {
            const double w = fabs(ds[j]) + p[j] * A;
            for (d = 0; d < D; ++d) {
                if (mq) mq[d] += scale * w * fabs(K[j * D + d]);
                if (mK) mK[j * D + d] += scale * w * fabs(qi[d]);
                if (mV) mV[j * D + d] += p[j] * fabs(doi[d]);
            }
        }
    }
    return delta;
}

typedef struct {
    const double *q, *k, *v, *dout;
    double *dq, *dk, *dv;
    double *mq, *mk, *mv; /* sensitivities, all NULL or all set */
    int64_t B, Hq, Hkv, Lq, Lk, D;
    double scale;
    int causal;
    int64_t win_left, win_right;
    int64_t next; /* shared work counter over (b, h_kv) units */
    int status;
} bwd_job;

/* One unit = one (batch, K/V head): every query row of every query head that reads it,
 * so the unit's dK and dV rows are written by this worker alone. */
static void* bwd_worker(void* arg) {
    bwd_job* J = (bwd_job*)arg;
    const size_t n = (size_t)(J->Lk > 0 ? J->Lk : 1);
    double* s = (double*)malloc(sizeof(double) * n);
    double* p = (double*)malloc(sizeof(double) * n);
    double* ds = (double*)malloc(sizeof(double) * n);
    double* o = (double*)malloc(sizeof(double) * (size_t)J->D);
    if (!s || !p || !ds || !o) {
        __atomic_store_n(&J->status, ORACLE_ERR_NOMEM, __ATOMIC_RELAXED);
        free(s); free(p); free(ds); free(o);
        return NULL;
    }
    const int64_t group = J->Hq / J->Hkv;
    for (;;) {
        int64_t u = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (u >= J->B * J->Hkv) break;
        const int64_t b = u / J->Hkv, hkv = u % J->Hkv;
        const double* K = J->k + u * J->Lk * J->D;
        const double* V = J->v + u * J->Lk * J->D;
        double* dK = J->dk + u * J->Lk * J->D;
        double* dV = J->dv + u * J->Lk * J->D;
        double* mK = J->mk ? J->mk + u * J->Lk * J->D : NULL;
        double* mV = J->mv ? J->mv + u * J->Lk * J->D : NULL;
        for (int64_t x = 0; x < J->Lk * J->D; ++x) dK[x] = dV[x] = 0.0;
        if (mK)
            for (int64_t x = 0; x < J->Lk * J->D; ++x) mK[x] = mV[x] = 0.0;
        for (int64_t g = 0; g < group; ++g) {
            const int64_t h = hkv * group + g;
            for (int64_t i = 0; i < J->Lq; ++i) {
                const int64_t id = (b * J->Hq + h) * J->Lq + i;
                int64_t lo, hi;
                visible_range(i, J->Lq, J->Lk, J->causal, J->win_left, J->win_right, &lo, &hi);
                backward_row(J->q + id * J->D, J->dout + id * J->D, K, V, J->Lk, lo, hi, J->D,
                             J->scale, s, p, ds, o, J->dq + id * J->D, dK, dV,
                             J->mq ? J->mq + id * J->D : NULL, mK, mV);
            }
        }
    }
    free(s); free(p); free(ds); free(o);
    return NULL;
}

/*
 * Gradients of attention: dq[B,Hq,Lq,D], dk[B,Hkv,Lk,D], dv[B,Hkv,Lk,D] from
 * q[B,Hq,Lq,D], k/v[B,Hkv,Lk,D] and dout[B,Hq,Lq,D] = dLoss/dO, with the mask of
 * oracle_attn_fwd_window (left = right = -1 and causal = 0: no mask). mq, mk, mv
 * (shaped like dq, dk, dv) receive the rounding sensitivities when all three are
 * given; pass NULL for none.
 */
int oracle_attn_bwd(const double* q, const double* k, const double* v, const double* dout,
                    double* dq, double* dk, double* dv, double* mq, double* mk, double* mv,
                    int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk, int64_t D,
                    double scale, int causal, int64_t left, int64_t right, int nthreads) {
    int rc = check_dims(B, Hq, Hkv, Lq, Lk, D);
    if (rc) return rc;
    if (left < -1 || right < -1) return ORACLE_ERR_ARG;
    if (!mq || !mk || !mv) mq = mk = mv = NULL;
    bwd_job J = {q, k, v, dout, dq, dk, dv, mq, mk, mv, B, Hq, Hkv, Lq, Lk, D, scale, causal,
                 left, right, 0, ORACLE_OK};
    int64_t units = B * Hkv;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (units < nthreads) nthreads = (int)(units > 0 ? units : 1);
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&tid[started], NULL, bwd_worker, &J) == 0) ++started;
    bwd_worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return J.status;
}

/* Selected outputs of the backward pass, for problems too large to run whole. */
typedef struct {
    const double *q, *k, *v, *dout;
    int64_t B, Hq, Hkv, Lq, Lk, D;
    double scale;
    int causal;
    const int64_t* ids; /* query rows (dq) or keys (dk, dv), flattened */
    int64_t n;
    double *dq, *dk, *dv;  /* n rows of D each */
    double *mq, *mk, *mv;  /* their sensitivities (may be NULL) */
    int64_t unit;          /* keys: the (b * Hkv + h_kv) unit the row statistics are for */
    double *lse, *delta, *absdo; /* keys: per query row of the unit's group, [group * Lq];
                                    absdo = sum_d |do_id o_id| */
    int64_t next;
    int status;
} sel_job;

/* dQ of selected query rows: each row by backward_row on its own. */
static void* dq_rows_worker(void* arg) {
    sel_job* J = (sel_job*)arg;
    const size_t n = (size_t)(J->Lk > 0 ? J->Lk : 1);
    double* s = (double*)malloc(sizeof(double) * n);
    double* p = (double*)malloc(sizeof(double) * n);
    double* ds = (double*)malloc(sizeof(double) * n);
    double* o = (double*)malloc(sizeof(double) * (size_t)J->D);
    if (!s || !p || !ds || !o) {
        __atomic_store_n(&J->status, ORACLE_ERR_NOMEM, __ATOMIC_RELAXED);
        free(s); free(p); free(ds); free(o);
        return NULL;
    }
    const int64_t group = J->Hq / J->Hkv;
    for (;;) {
        int64_t r = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (r >= J->n) break;
        const int64_t id = J->ids[r];
        const int64_t i = id % J->Lq, bh = id / J->Lq;
        const int64_t h = bh % J->Hq, b = bh / J->Hq;
        const int64_t u = b * J->Hkv + h / group;
        int64_t lo, hi;
        visible_range(i, J->Lq, J->Lk, J->causal, -1, -1, &lo, &hi);
        backward_row(J->q + id * J->D, J->dout + id * J->D, J->k + u * J->Lk * J->D,
                     J->v + u * J->Lk * J->D, J->Lk, lo, hi, J->D, J->scale, s, p, ds, o,
                     J->dq + r * J->D, NULL, NULL, J->mq ? J->mq + r * J->D : NULL, NULL, NULL);
    }
    free(s); free(p); free(ds); free(o);
    return NULL;
}

/* Row statistics of one unit's query rows: lse_i (attention_row) and delta_i. */
static void* unit_stats_worker(void* arg) {
    sel_job* J = (sel_job*)arg;
    const size_t n = (size_t)(J->Lk > 0 ? J->Lk : 1);
    double* s = (double*)malloc(sizeof(double) * n);
    double* p = (double*)malloc(sizeof(double) * n);
    double* o = (double*)malloc(sizeof(double) * (size_t)J->D);
    if (!s || !p || !o) {
        __atomic_store_n(&J->status, ORACLE_ERR_NOMEM, __ATOMIC_RELAXED);
        free(s); free(p); free(o);
        return NULL;
    }
    const int64_t group = J->Hq / J->Hkv;
    const int64_t b = J->unit / J->Hkv, hkv = J->unit % J->Hkv;
    const double* K = J->k + J->unit * J->Lk * J->D;
    const double* V = J->v + J->unit * J->Lk * J->D;
    for (;;) {
        int64_t r = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (r >= group * J->Lq) break;
        const int64_t g = r / J->Lq, i = r % J->Lq;
        const int64_t id = (b * J->Hq + hkv * group + g) * J->Lq + i;
        const double* doi = J->dout + id * J->D;
        int64_t lo, hi;
        visible_range(i, J->Lq, J->Lk, J->causal, -1, -1, &lo, &hi);
        attention_row(J->q + id * J->D, K, V, J->Lk, lo, hi, J->D, J->scale, s, o, &J->lse[r], p);
        double delta = 0.0;
        for (int64_t j = lo; j < hi; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < J->D; ++d) dot += doi[d] * V[j * J->D + d];
            delta += p[j] * dot;
        }
        J->delta[r] = delta;
        double A = 0.0;
        for (int64_t d = 0; d < J->D; ++d) A += fabs(doi[d] * o[d]);
        J->absdo[r] = A;
    }
    free(s); free(p); free(o);
    return NULL;
}

/* dK_j, dV_j of the selected keys of the current unit, as sums over the query rows
 * that see key j: P_ij = exp(s_ij - lse_i), dS_ij = P_ij (do_i . v_j - delta_i). */
static void* dkv_keys_worker(void* arg) {
    sel_job* J = (sel_job*)arg;
    const int64_t group = J->Hq / J->Hkv;
    const int64_t b = J->unit / J->Hkv, hkv = J->unit % J->Hkv;
    const double* K = J->k + J->unit * J->Lk * J->D;
    const double* V = J->v + J->unit * J->Lk * J->D;
    for (;;) {
        int64_t r = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (r >= J->n) break;
        if (J->ids[r] / J->Lk != J->unit) continue;
        const int64_t j = J->ids[r] % J->Lk;
        double* dk = J->dk + r * J->D;
        double* dv = J->dv + r * J->D;
        double* mk = J->mk ? J->mk + r * J->D : NULL;
        double* mv = J->mv ? J->mv + r * J->D : NULL;
        for (int64_t d = 0; d < J->D; ++d) dk[d] = dv[d] = 0.0;
        if (mk)
            for (int64_t d = 0; d < J->D; ++d) mk[d] = mv[d] = 0.0;
        for (int64_t g = 0; g < group; ++g) {
            for (int64_t i = 0; i < J->Lq; ++i) {
                int64_t lo, hi;
                visible_range(i, J->Lq, J->Lk, J->causal, -1, -1, &lo, &hi);
                if (j < lo || j >= hi) continue;
                const int64_t id = (b * J->Hq + hkv * group + g) * J->Lq + i;
                const double* qi = J->q + id * J->D;
                const double* doi = J->dout + id * J->D;
                double dot = 0.0, dpv = 0.0;
                for (int64_t d = 0; d < J->D; ++d) dot += qi[d] * K[j * J->D + d];
                for (int64_t d = 0; d < J->D; ++d) dpv += doi[d] * V[j * J->D + d];
                const double pij = exp(J->scale * dot - J->lse[g * J->Lq + i]);
                const double dsij = pij * (dpv - J->delta[g * J->Lq + i]);
                for (int64_t d = 0; d < J->D; ++d) {
                    dv[d] += pij * doi[d];
                    dk[d] += J->scale * dsij * qi[d];
                }
                if (mk) {
                    const double w = fabs(dsij) + pij * J->absdo[g * J->Lq + i];
                    for (int64_t d = 0; d < J->D; ++d) {
                        mk[d] += J->scale * w * fabs(qi[d]);
                        mv[d] += pij * fabs(doi[d]);
                    }
                }
            }
        }
    }
    return NULL;
}

static int run_workers(void* (*fn)(void*), void* job, int64_t work, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (work < nthreads) nthreads = (int)(work > 0 ? work : 1);
    pthread_t tid[256];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&tid[started], NULL, fn, job) == 0) ++started;
    fn(job);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    return 0;
}

/* dq[n,D] of the query rows ids[r] = (b*Hq + h)*Lq + i (causal or no mask); mq[n,D]
 * receives their sensitivities if not NULL. */
int oracle_attn_bwd_dq_rows(const double* q, const double* k, const double* v,
                            const double* dout, const int64_t* rows, int64_t n, double* dq,
                            double* mq, int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq,
                            int64_t Lk, int64_t D, double scale, int causal, int nthreads) {
    int rc = check_dims(B, Hq, Hkv, Lq, Lk, D);
    if (rc) return rc;
    for (int64_t r = 0; r < n; ++r)
        if (rows[r] < 0 || rows[r] >= B * Hq * Lq) return ORACLE_ERR_INDEX;
    sel_job J = {q, k, v, dout, B, Hq, Hkv, Lq, Lk, D, scale, causal, rows, n, dq, NULL, NULL,
                 mq, NULL, NULL, 0, NULL, NULL, NULL, 0, ORACLE_OK};
    run_workers(dq_rows_worker, &J, n, nthreads);
    return J.status;
}

/* dk[n,D], dv[n,D] of the keys ids[r] = (b*Hkv + h_kv)*Lk + j (causal or no mask);
 * mk, mv [n,D] receive their sensitivities when both are given. */
int oracle_attn_bwd_dkv_keys(const double* q, const double* k, const double* v,
                             const double* dout, const int64_t* keys, int64_t n, double* dk,
                             double* dv, double* mk, double* mv, int64_t B, int64_t Hq,
                             int64_t Hkv, int64_t Lq, int64_t Lk, int64_t D, double scale,
                             int causal, int nthreads) {
    int rc = check_dims(B, Hq, Hkv, Lq, Lk, D);
    if (rc) return rc;
    for (int64_t r = 0; r < n; ++r)
        if (keys[r] < 0 || keys[r] >= B * Hkv * Lk) return ORACLE_ERR_INDEX;
    const int64_t group = Hq / Hkv;
    if (!mk || !mv) mk = mv = NULL;
    double* lse = (double*)malloc(sizeof(double) * (size_t)(group * Lq + 1));
    double* delta = (double*)malloc(sizeof(double) * (size_t)(group * Lq + 1));
    double* absdo = (double*)malloc(sizeof(double) * (size_t)(group * Lq + 1));
    if (!lse || !delta || !absdo) {
        free(lse); free(delta); free(absdo);
        return ORACLE_ERR_NOMEM;
    }
    int status = ORACLE_OK;
    /* One pass per distinct unit among the keys: its rows' statistics, then its keys. */
    for (int64_t r0 = 0; r0 < n && status == ORACLE_OK; ++r0) {
        const int64_t unit = keys[r0] / Lk;
        int seen = 0;
        for (int64_t r = 0; r < r0; ++r)
            if (keys[r] / Lk == unit) seen = 1;
        if (seen) continue;
        sel_job J = {q, k, v, dout, B, Hq, Hkv, Lq, Lk, D, scale, causal, keys, n, NULL, dk, dv,
                     NULL, mk, mv, unit, lse, delta, absdo, 0, ORACLE_OK};
        run_workers(unit_stats_worker, &J, group * Lq, nthreads);
        J.next = 0;
        run_workers(dkv_keys_worker, &J, n, nthreads);
        status = J.status;
    }
    free(lse); free(delta); free(absdo);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Paged prefill: a chunk of queries per sequence over its paged cache.     */
/* ------------------------------------------------------------------------ */

/*
 * Each sequence s has seq_lens[s] tokens in the paged cache (resolved through
 * block_table exactly as in oracle_attn_paged) and a chunk of q_lens[s] queries,
 * which are its last q_lens[s] positions: query i sits at position
 * seq_lens[s] - q_lens[s] + i, the bottom-right alignment of the dense causal mask
 * (Lq = q_lens[s], Lk = seq_lens[s]). Without causal every query sees all
 * seq_lens[s] keys. Rows i >= q_lens[s] of the [num_seqs, Hq, Lq, D] output are
 * written as rows with no key (O = 0, lse = -inf).
 */
typedef struct {
    const double *q, *kc, *vc;
    const int32_t *block_table, *seq_lens, *q_lens;
    double *out, *lse;
    int64_t block_size, num_seqs, Hq, Hkv, Lq, D, max_blocks, num_blocks;
    double scale;
    int causal;
    int64_t next;
    int status;
} paged_prefill_job;

static void* paged_prefill_worker(void* arg) {
    paged_prefill_job* J = (paged_prefill_job*)arg;
    const int64_t cap = J->max_blocks * J->block_size;
    double* Kd = (double*)malloc(sizeof(double) * (size_t)(cap * J->D + 1));
    double* Vd = (double*)malloc(sizeof(double) * (size_t)(cap * J->D + 1));
    double* s = (double*)malloc(sizeof(double) * (size_t)(cap + 1));
    if (!Kd || !Vd || !s) {
        __atomic_store_n(&J->status, ORACLE_ERR_NOMEM, __ATOMIC_RELAXED);
        free(Kd); free(Vd); free(s);
        return NULL;
    }
    const int64_t group = J->Hq / J->Hkv;
    for (;;) {
        int64_t u = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
        if (u >= J->num_seqs * J->Hkv) break;
        int64_t sq = u / J->Hkv, hkv = u % J->Hkv;
        int64_t len = J->seq_lens[sq];
        int64_t ql = J->q_lens ? J->q_lens[sq] : J->Lq;
        /* Gather this sequence's keys and values in logical order. */
        for (int64_t t = 0; t < len; ++t) {
            int64_t phys = J->block_table[sq * J->max_blocks + t / J->block_size];
            if (phys < 0 || phys >= J->num_blocks) {
                __atomic_store_n(&J->status, ORACLE_ERR_INDEX, __ATOMIC_RELAXED);
                len = 0;
                break;
            }
            const int64_t row = ((phys * J->Hkv + hkv) * J->block_size + t % J->block_size) * J->D;
            memcpy(Kd + t * J->D, J->kc + row, sizeof(double) * (size_t)J->D);
            memcpy(Vd + t * J->D, J->vc + row, sizeof(double) * (size_t)J->D);
        }
        for (int64_t g = 0; g < group; ++g) {
            const int64_t h = hkv * group + g;
            for (int64_t i = 0; i < J->Lq; ++i) {
                const int64_t id = (sq * J->Hq + h) * J->Lq + i;
                double* o = J->out + id * J->D;
                double* l = J->lse ? J->lse + id : NULL;
                int64_t lo = 0, hi = 0; /* rows past the chunk see no key */
                if (i < ql) visible_range(i, ql, len, J->causal, -1, -1, &lo, &hi);
                attention_row(J->q + id * J->D, Kd, Vd, len, lo, hi, J->D, J->scale, s, o, l, NULL);
            }
        }
    }
    free(Kd); free(Vd); free(s);
    return NULL;
}

/*
 * q[num_seqs,Hq,Lq,D]; k_cache, v_cache [num_blocks,Hkv,block_size,D];
 * block_table[num_seqs,max_blocks]; seq_lens[num_seqs]; q_lens[num_seqs] (NULL: all
 * Lq); out[num_seqs,Hq,Lq,D]; lse[num_seqs,Hq,Lq] (may be NULL).
 */
int oracle_attn_paged_prefill(const double* q, const double* k_cache, const double* v_cache,
                              const int32_t* block_table, const int32_t* seq_lens,
                              const int32_t* q_lens, int64_t block_size, double* out,
                              double* lse, int64_t num_seqs, int64_t Hq, int64_t Hkv, int64_t Lq,
                              int64_t D, int64_t max_blocks, int64_t num_blocks, double scale,
                              int causal, int nthreads) {
    if (num_seqs < 0 || Hq < 1 || Hkv < 1 || Lq < 0 || D < 1 || block_size < 1 ||
        max_blocks < 0 || num_blocks < 0 || Hq % Hkv != 0)
        return ORACLE_ERR_ARG;
    for (int64_t s = 0; s < num_seqs; ++s) {
        if (seq_lens[s] < 0 || seq_lens[s] > max_blocks * block_size) return ORACLE_ERR_INDEX;
        if (q_lens && (q_lens[s] < 0 || q_lens[s] > Lq)) return ORACLE_ERR_INDEX;
    }
    paged_prefill_job J = {q, k_cache, v_cache, block_table, seq_lens, q_lens, out, lse,
                           block_size, num_seqs, Hq, Hkv, Lq, D, max_blocks, num_blocks, scale,
                           causal, 0, ORACLE_OK};
    run_workers(paged_prefill_worker, &J, num_seqs * Hkv, nthreads);
    return J.status;
}

/*
 * attn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of exact scaled dot-product
 * attention in fp64.  Only the test suite, the smoke entry and the bench's
 * CPU-baseline leg may load this library; the CUDA product path never does,
 * and this file shares no source with it.
 *
 * What it computes (one batch b, one query head h, kv head g = h / (Hq/Hkv)):
 *
 *   S[i][j] = scale * sum_t q[i][t] * k[j][t]            (the score matrix)
 *   S[i][j] = -inf  where key j is masked for query i      (additive 0/-inf mask)
 *   P[i][j] = exp(S[i][j] - m_i) / l_i,  m_i = max_j S[i][j],
 *             l_i = sum_j exp(S[i][j] - m_i)              (row softmax)
 *   O[i][:] = sum_j P[i][j] * v[j][:]
 *   LSE[i]  = m_i + log(l_i)                              (natural log)
 *
 * Sources, as printed on the pages:
 *  - ai6s.net "ops-transformer FlashAttention" article, section "标准注意力的
 *    致命伤不在算力，在搬运" (the flaw of standard attention is data movement):
 *    the four steps Q·Kᵀ -> scale -> softmax -> ·V and the N×N matrix S, which
 *    this oracle materialises on purpose.
 *  - same article, section "FlashAttention 拆的不是算法，是数据流": the method
 *    is exact, i.e. its result is this plain definition.
 *  - same article, section "ops-transformer 里的 FlashAttention 做了什么额外
 *    的事", points 2 and 3: the causal mask and the variable-length KV cache
 *    whose real length bounds the keys.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - the mask is additive 0/-inf, so a masked key gets exactly zero weight and
 *    is never multiplied (a NaN stored in a masked slot cannot leak);
 *  - causal alignment is bottom-right: query i of Nq attends key j iff
 *    j <= i + (Lk - Nq), which is the usual top-left rule when Nq == Lk and
 *    makes the newest query tokens the last rows of a growing KV cache;
 *  - a row with no visible key gives O = 0 and LSE = -inf;
 *  - grouped-query heads map contiguously: g = h / (Hq / Hkv);
 *  - a sliding window (window_left >= 0) also masks keys more than
 *    window_left positions before the query's own position i + (Lk - Nq)
 *    (the "extensions for masks" the pages list as a direction); -1 = none;
 *  - a block mask (the other mask extension: block-sparse attention) cuts
 *    the (query, key) plane into blocks of block_m rows by block_n keys and
 *    masks every key of a block whose entry is 0, on top of the other rules.
 *
 * Arithmetic: every input is fp64 (the caller widens the bf16/fp16 bits
 * exactly).  Row sums and output sums use Neumaier compensated summation so
 * that a softmax row sums to 1 within 1e-12 even over 32K keys.  Build with
 * -O2 -ffp-contract=off and without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- compensated summation (Neumaier's variant of Kahan) ---------------- */
typedef struct {
    double sum;
    double comp;
} csum_t;

static void csum_add(csum_t* a, double x) {
    double t = a->sum + x;
    if (fabs(a->sum) >= fabs(x))
        a->comp += (a->sum - t) + x;
    else
        a->comp += (x - t) + a->sum;
    a->sum = t;
}

static double csum_value(const csum_t* a) { return a->sum + a->comp; }

/* ---- the mask: is key j visible to query row i? --------------------------
 * causal: j <= i + (Lk - Nq); window_left >= 0: j >= i + (Lk - Nq) - window_left */
static int key_visible(int i, int j, int Nq, int Lk, int causal, int window_left) {
    const int pos = i + (Lk - Nq); /* the query's own position among the keys */
    if (causal && j > pos) return 0;
    if (window_left >= 0 && j < pos - window_left) return 0;
    return 1;
}

/* ---- the block mask of one (batch, head) ---------------------------------
 * m == NULL: no block mask.  Otherwise block (i / bm, j / bn) is
 * m[(i / bm) * nkb + j / bn]; 0 masks every key of the block. */
typedef struct {
    const unsigned char* m;
    int nkb, bm, bn;
} bmask_t;

static const bmask_t nomask = {NULL, 0, 1, 1};

static int block_on(const bmask_t* mk, int i, int j) {
    if (!mk->m) return 1;
    return mk->m[(size_t)(i / mk->bm) * (size_t)mk->nkb + (size_t)(j / mk->bn)] != 0;
}

/* the block mask of (b, h) inside a [B?, H?, nqb, nkb] array with strides sb, sh */
static bmask_t head_mask(const unsigned char* mask, long sb, long sh, int nkb, int bm, int bn,
                         int b, int h) {
    bmask_t r = {NULL, nkb, bm, bn};
    if (mask) r.m = mask + (size_t)b * (size_t)sb + (size_t)h * (size_t)sh;
    return r;
}

/* mask arguments: NULL mask, or block sizes > 0, rows and columns of blocks
 * that cover Nq x Nk, non-negative strides */
static int mask_args_ok(const unsigned char* mask, long sb, long sh, int nqb, int nkb, int bm,
                        int bn, int Nq, int Nk) {
    if (!mask) return 1;
    if (bm <= 0 || bn <= 0 || sb < 0 || sh < 0) return 0;
    if ((long)nqb * bm < Nq || (long)nkb * bn < Nk) return 0;
    return 1;
}

/* ---- one query head against one key/value head --------------------------
 * q_rows[r]   : pointer to the d values of the r-th requested query row
 * row_index[r]: that row's index i in [0, Nq), used by the causal rule
 * k, v        : key/value row j at k + j*kv_stride (j in [0, Lk))
 * S           : scratch of nrows*Lk doubles, the materialised score rows
 * o_rows[r]   : output row (d doubles), lse_out[r]: its log-sum-exp
 */
static void attend_head(int nrows, const double* const* q_rows, const int* row_index,
                        const double* k, const double* v, long kv_stride, int Nq, int Lk,
                        int d, double scale, int causal, int window_left, const bmask_t* mk,
                        double* const* o_rows, double* const* lse_out, double* S) {
    for (int r = 0; r < nrows; ++r) {
        const double* qi = q_rows[r];
        const int i = row_index[r];
        double* Srow = S + (size_t)r * (size_t)(Lk > 0 ? Lk : 1);
        /* step 1 + 2: scores, then the additive 0 / -inf mask */
        for (int j = 0; j < Lk; ++j) {
            const int visible = key_visible(i, j, Nq, Lk, causal, window_left) &&
                                block_on(mk, i, j);
            if (!visible) {
                Srow[j] = -INFINITY;
                continue;
            }
            const double* kj = k + (size_t)j * (size_t)kv_stride;
            double dot = 0.0;
            for (int t = 0; t < d; ++t) dot += qi[t] * kj[t];
            Srow[j] = scale * dot;
        }
        /* step 3: row softmax */
        double m = -INFINITY;
        for (int j = 0; j < Lk; ++j)
            if (Srow[j] > m) m = Srow[j];
        double* oi = o_rows[r];
        if (m == -INFINITY) { /* no visible key */
            for (int t = 0; t < d; ++t) oi[t] = 0.0;
            *lse_out[r] = -INFINITY;
            continue;
        }
        csum_t l = {0.0, 0.0};
        for (int j = 0; j < Lk; ++j) {
            if (Srow[j] == -INFINITY) {
                Srow[j] = 0.0; /* exp(-inf) */
                continue;
            }
            Srow[j] = exp(Srow[j] - m);
            csum_add(&l, Srow[j]);
        }
        const double lsum = csum_value(&l);
        for (int j = 0; j < Lk; ++j) Srow[j] = Srow[j] / lsum; /* P row */
        /* step 4: O = P·V, masked keys skipped (their weight is exactly 0) */
        for (int t = 0; t < d; ++t) {
            csum_t acc = {0.0, 0.0};
            for (int j = 0; j < Lk; ++j) {
                if (Srow[j] == 0.0) continue;
                csum_add(&acc, Srow[j] * v[(size_t)j * (size_t)kv_stride + t]);
            }
            oi[t] = csum_value(&acc);
        }
        *lse_out[r] = m + log(lsum);
    }
}

static int pick_threads(size_t scratch_bytes_per_thread) {
#ifdef _OPENMP
    int n = omp_get_max_threads();
    const size_t budget = (size_t)8 << 30; /* keep the materialised S under 8 GiB */
    if (scratch_bytes_per_thread > 0) {
        size_t cap = budget / scratch_bytes_per_thread;
        if (cap < 1) cap = 1;
        if ((size_t)n > cap) n = (int)cap;
    }
    return n;
#else
    (void)scratch_bytes_per_thread;
    return 1;
#endif
}

/* Threads the oracle will use (OpenMP), for reporting. */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Dense (optionally key-padded) attention.
 *   q   [B, Nq, Hq, d]   k, v [B, Nk, Hkv, d]   (row-major, fp64)
 *   o   [B, Nq, Hq, d]   lse  [B, Hq, Nq]
 *   seqlens_k: NULL, or [B] real key lengths (<= Nk); keys at or beyond the
 *              length are masked (the variable-length reading of the KV-cache
 *              point on the ai6s.net page).
 *   rows, nrows: NULL/0 computes every query row; otherwise only the listed
 *              row indices, for every (b, h); other outputs are left alone.
 *   window_left: -1, or the sliding window described at the top.
 *   block_mask: NULL, or the block mask of (b, h) at
 *              block_mask + b * mask_sb + h * mask_sh, mask_nqb rows of
 *              mask_nkb entries (blocks of block_m queries by block_n keys;
 *              a zero stride shares one mask across batches or heads).
 * Returns 0, or -1 on bad arguments.
 */
int oracle_attn_fwd_mask(const double* q, const double* k, const double* v, double* o,
                         double* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         double scale, int causal, const int* seqlens_k, const int* rows,
                         int nrows, int window_left, const unsigned char* block_mask,
                         long mask_sb, long mask_sh, int mask_nqb, int mask_nkb, int block_m,
                         int block_n) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || d <= 0 || Hq % Hkv != 0) return -1;
    if (!mask_args_ok(block_mask, mask_sb, mask_sh, mask_nqb, mask_nkb, block_m, block_n, Nq, Nk))
        return -1;
    if (seqlens_k)
        for (int b = 0; b < B; ++b)
            if (seqlens_k[b] < 0 || seqlens_k[b] > Nk) return -1;
    const int nr = rows ? nrows : Nq;
    if (rows)
        for (int r = 0; r < nrows; ++r)
            if (rows[r] < 0 || rows[r] >= Nq) return -1;
    const int G = Hq / Hkv;
    const size_t s_bytes = (size_t)(nr > 0 ? nr : 1) * (size_t)(Nk > 0 ? Nk : 1) * sizeof(double);
    const int nthreads = pick_threads(s_bytes);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        const int Lk = seqlens_k ? seqlens_k[b] : Nk;
        double* S = (double*)malloc(s_bytes);
        const double** qp = (const double**)malloc(sizeof(double*) * (size_t)(nr > 0 ? nr : 1));
        double** op = (double**)malloc(sizeof(double*) * (size_t)(nr > 0 ? nr : 1));
        double** lp = (double**)malloc(sizeof(double*) * (size_t)(nr > 0 ? nr : 1));
        int* ri = (int*)malloc(sizeof(int) * (size_t)(nr > 0 ? nr : 1));
        if (!S || !qp || !op || !lp || !ri) {
#pragma omp atomic write
            err = 1;
        } else {
            for (int r = 0; r < nr; ++r) {
                const int i = rows ? rows[r] : r;
                ri[r] = i;
                qp[r] = q + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                op[r] = o + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                lp[r] = lse + ((size_t)b * Hq + h) * (size_t)Nq + i;
            }
            const double* kb = k + ((size_t)b * Nk * Hkv + g) * (size_t)d;
            const double* vb = v + ((size_t)b * Nk * Hkv + g) * (size_t)d;
            const bmask_t mk =
                head_mask(block_mask, mask_sb, mask_sh, mask_nkb, block_m, block_n, b, h);
            attend_head(nr, qp, ri, kb, vb, (long)Hkv * d, Nq, Lk, d, scale, causal, window_left,
                        &mk, op, lp, S);
        }
        free(S);
        free(qp);
        free(op);
        free(lp);
        free(ri);
    }
    return err ? -2 : 0;
}

/* oracle_attn_fwd_mask without a block mask */
int oracle_attn_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
                    int B, int Hq, int Hkv, int Nq, int Nk, int d, double scale, int causal,
                    const int* seqlens_k, const int* rows, int nrows, int window_left) {
    return oracle_attn_fwd_mask(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, seqlens_k,
                                rows, nrows, window_left, NULL, 0, 0, 0, 0, 1, 1);
}

/*
 * Attention of new query tokens against a packed, variable-length KV cache.
 *   q        [B, Nq, Hq, d]          (Nq new tokens per sequence)
 *   k_cache, v_cache [slots, Hkv, d] sequence b owns slots
 *            cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1, of which the first
 *            seqlens_k[b] are filled (the cache is pre-allocated and grows by
 *            one row per token: ai6s.net article, adaptation point 3)
 *   o        [B, Nq, Hq, d]          lse [B, Hq, Nq]
 * Causal means bottom-right: token i of Nq sees keys j <= i + Lk - Nq.
 */
int oracle_attn_kvcache(const double* q, const double* k_cache, const double* v_cache,
                        const int* cu_seqlens_k, const int* seqlens_k, double* o, double* lse,
                        int B, int Hq, int Hkv, int Nq, int d, double scale, int causal) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || d <= 0 || Hq % Hkv != 0) return -1;
    int maxlen = 0;
    for (int b = 0; b < B; ++b) {
        const int cap = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        if (cu_seqlens_k[b] < 0 || cap < 0 || seqlens_k[b] < 0 || seqlens_k[b] > cap) return -1;
        if (seqlens_k[b] > maxlen) maxlen = seqlens_k[b];
    }
    const int G = Hq / Hkv;
    const size_t s_bytes = (size_t)Nq * (size_t)(maxlen > 0 ? maxlen : 1) * sizeof(double);
    const int nthreads = pick_threads(s_bytes);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        const int Lk = seqlens_k[b];
        double* S = (double*)malloc(s_bytes);
        const double** qp = (const double**)malloc(sizeof(double*) * (size_t)Nq);
        double** op = (double**)malloc(sizeof(double*) * (size_t)Nq);
        double** lp = (double**)malloc(sizeof(double*) * (size_t)Nq);
        int* ri = (int*)malloc(sizeof(int) * (size_t)Nq);
        if (!S || !qp || !op || !lp || !ri) {
#pragma omp atomic write
            err = 1;
        } else {
            for (int i = 0; i < Nq; ++i) {
                ri[i] = i;
                qp[i] = q + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                op[i] = o + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                lp[i] = lse + ((size_t)b * Hq + h) * (size_t)Nq + i;
            }
            const double* kb = k_cache + ((size_t)cu_seqlens_k[b] * Hkv + g) * (size_t)d;
            const double* vb = v_cache + ((size_t)cu_seqlens_k[b] * Hkv + g) * (size_t)d;
            attend_head(Nq, qp, ri, kb, vb, (long)Hkv * d, Nq, Lk, d, scale, causal, -1, &nomask,
                        op, lp,
                        S);
        }
        free(S);
        free(qp);
        free(op);
        free(lp);
        free(ri);
    }
    return err ? -2 : 0;
}

/*
 * Merge of attention results computed over disjoint key sets (the online
 * softmax correction of the ai6s.net article, section "FlashAttention 拆的不是
 * 算法，是数据流", applied to whole partial results instead of tiles):
 *   LSE = log sum_p exp(LSE_p)
 *   O   = sum_p exp(LSE_p - LSE) * O_p
 * o_parts [nparts][nrows][d], lse_parts [nparts][nrows]; a part whose LSE is
 * -inf saw no key and has weight 0.  Rows with no key anywhere: O = 0,
 * LSE = -inf.
 */
int oracle_lse_combine(const double* o_parts, const double* lse_parts, int nparts, int nrows,
                       int d, double* o, double* lse) {
    if (nparts <= 0 || nrows < 0 || d <= 0) return -1;
    for (int r = 0; r < nrows; ++r) {
        double m = -INFINITY;
        for (int p = 0; p < nparts; ++p)
            if (lse_parts[(size_t)p * nrows + r] > m) m = lse_parts[(size_t)p * nrows + r];
        if (m == -INFINITY) {
            for (int t = 0; t < d; ++t) o[(size_t)r * d + t] = 0.0;
            lse[r] = -INFINITY;
            continue;
        }
        csum_t s = {0.0, 0.0};
        for (int p = 0; p < nparts; ++p) {
            const double lp = lse_parts[(size_t)p * nrows + r];
            if (lp != -INFINITY) csum_add(&s, exp(lp - m));
        }
        const double total = m + log(csum_value(&s));
        for (int t = 0; t < d; ++t) {
            csum_t acc = {0.0, 0.0};
            for (int p = 0; p < nparts; ++p) {
                const double lp = lse_parts[(size_t)p * nrows + r];
                if (lp == -INFINITY) continue;
                csum_add(&acc, exp(lp - total) * o_parts[((size_t)p * nrows + r) * d + t]);
            }
            o[(size_t)r * d + t] = csum_value(&acc);
        }
        lse[r] = total;
    }
    return 0;
}

/*
 * Gradients of exact attention (the backward pass) -- the chain rule applied
 * to the definition at the top of this file.  The pages report training
 * speed-ups (effectstory.com article, "訓練性能量化提升" table) but print no
 * backward algorithm, so this states the plain derivative of
 *
 *   L = sum_{b,i,h,t} dO[b,i,h,t] * O[b,i,h,t]
 *
 * for one (b, h) with kv head g and the row softmax P of the definition:
 *
 *   dV[j]    += sum_i P[i][j] * dO[i]                (summed over the G heads of g)
 *   dP[i][j]  = dO[i] . V[j]
 *   dS[i][j]  = P[i][j] * (dP[i][j] - sum_j' P[i][j'] * dP[i][j'])   (softmax Jacobian)
 *   dQ[i]     = scale * sum_j dS[i][j] * K[j]
 *   dK[j]    += scale * sum_i dS[i][j] * Q[i]       (summed over the G heads of g)
 *
 * Masked keys have P = 0 and therefore dS = 0; a row with no visible key
 * contributes nothing.  P is recomputed here from q, k, v (no forward output
 * or LSE is taken from the caller).  Every sum is compensated (Neumaier).
 *   q, dout, dq [B, Nq, Hq, d]   k, v, dk, dv [B, Nk, Hkv, d]   seqlens_k: NULL or [B]
 *   window_left, block_mask and its layout: as in oracle_attn_fwd_mask.
 * Work is split over (b, g) so that the sums over the heads of a group are
 * done by one thread in head order.  Returns 0, -1 (bad arguments) or -2.
 */
int oracle_attn_bwd_mask(const double* q, const double* k, const double* v, const double* dout,
                         double* dq, double* dk, double* dv, int B, int Hq, int Hkv, int Nq,
                         int Nk, int d, double scale, int causal, const int* seqlens_k,
                         int window_left, const unsigned char* block_mask, long mask_sb,
                         long mask_sh, int mask_nqb, int mask_nkb, int block_m, int block_n) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq < 0 || Nk < 0 || d <= 0 || Hq % Hkv != 0) return -1;
    if (!mask_args_ok(block_mask, mask_sb, mask_sh, mask_nqb, mask_nkb, block_m, block_n, Nq, Nk))
        return -1;
    if (seqlens_k)
        for (int b = 0; b < B; ++b)
            if (seqlens_k[b] < 0 || seqlens_k[b] > Nk) return -1;
    const int G = Hq / Hkv;
    const size_t nq1 = (size_t)(Nq > 0 ? Nq : 1), nk1 = (size_t)(Nk > 0 ? Nk : 1);
    const size_t per_thread = (2 * nq1 * nk1 + 2 * nk1 * (size_t)d) * sizeof(double) +
                              2 * nk1 * (size_t)d * sizeof(csum_t);
    const int nthreads = pick_threads(per_thread);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bg = 0; bg < (long)B * Hkv; ++bg) {
        const int b = (int)(bg / Hkv), g = (int)(bg % Hkv);
        const int Lk = seqlens_k ? seqlens_k[b] : Nk;
        double* P = (double*)malloc(nq1 * nk1 * sizeof(double));
        double* dS = (double*)malloc(nq1 * nk1 * sizeof(double));
        csum_t* dk_acc = (csum_t*)calloc(nk1 * (size_t)d, sizeof(csum_t));
        csum_t* dv_acc = (csum_t*)calloc(nk1 * (size_t)d, sizeof(csum_t));
        if (!P || !dS || !dk_acc || !dv_acc) {
#pragma omp atomic write
            err = 1;
        } else {
            const long kv_stride = (long)Hkv * d;
            const double* kb = k + ((size_t)b * Nk * Hkv + g) * (size_t)d;
            const double* vb = v + ((size_t)b * Nk * Hkv + g) * (size_t)d;
            for (int hh = 0; hh < G; ++hh) {
                const int h = g * G + hh;
                const bmask_t mk =
                    head_mask(block_mask, mask_sb, mask_sh, mask_nkb, block_m, block_n, b, h);
                for (int i = 0; i < Nq; ++i) {
                    const double* qi = q + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                    const double* doi = dout + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                    double* Prow = P + (size_t)i * nk1;
                    double* dSrow = dS + (size_t)i * nk1;
                    /* P row: scores, mask, softmax */
                    double m = -INFINITY;
                    for (int j = 0; j < Lk; ++j) {
                        const int visible = key_visible(i, j, Nq, Lk, causal, window_left) &&
                                            block_on(&mk, i, j);
                        if (!visible) {
                            Prow[j] = -INFINITY;
                            continue;
                        }
                        const double* kj = kb + (size_t)j * (size_t)kv_stride;
                        csum_t dot = {0.0, 0.0};
                        for (int t = 0; t < d; ++t) csum_add(&dot, qi[t] * kj[t]);
                        Prow[j] = scale * csum_value(&dot);
                        if (Prow[j] > m) m = Prow[j];
                    }
                    if (m == -INFINITY) { /* no visible key: O = 0 whatever q is */
                        for (int j = 0; j < Lk; ++j) Prow[j] = 0.0, dSrow[j] = 0.0;
                        double* dq0 = dq + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                        for (int t = 0; t < d; ++t) dq0[t] = 0.0;
                        continue;
                    }
                    csum_t l = {0.0, 0.0};
                    for (int j = 0; j < Lk; ++j) {
                        Prow[j] = (Prow[j] == -INFINITY) ? 0.0 : exp(Prow[j] - m);
                        csum_add(&l, Prow[j]);
                    }
                    const double lsum = csum_value(&l);
                    for (int j = 0; j < Lk; ++j) Prow[j] /= lsum;
                    /* dP row and the softmax Jacobian */
                    csum_t pdp = {0.0, 0.0};
                    for (int j = 0; j < Lk; ++j) {
                        if (Prow[j] == 0.0) {
                            dSrow[j] = 0.0;
                            continue;
                        }
                        const double* vj = vb + (size_t)j * (size_t)kv_stride;
                        csum_t dot = {0.0, 0.0};
                        for (int t = 0; t < d; ++t) csum_add(&dot, doi[t] * vj[t]);
                        dSrow[j] = csum_value(&dot); /* dP for now */
                        csum_add(&pdp, Prow[j] * dSrow[j]);
                    }
                    const double Di = csum_value(&pdp);
                    for (int j = 0; j < Lk; ++j)
                        if (Prow[j] != 0.0) dSrow[j] = Prow[j] * (dSrow[j] - Di);
                    /* dQ row */
                    double* dqi = dq + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                    for (int t = 0; t < d; ++t) {
                        csum_t acc = {0.0, 0.0};
                        for (int j = 0; j < Lk; ++j)
                            if (dSrow[j] != 0.0)
                                csum_add(&acc, dSrow[j] * kb[(size_t)j * (size_t)kv_stride + t]);
                        dqi[t] = scale * csum_value(&acc);
                    }
                    /* this row's contributions to dK and dV */
                    for (int j = 0; j < Lk; ++j) {
                        if (Prow[j] == 0.0) continue;
                        for (int t = 0; t < d; ++t) {
                            csum_add(&dv_acc[(size_t)j * d + t], Prow[j] * doi[t]);
                            csum_add(&dk_acc[(size_t)j * d + t], dSrow[j] * qi[t]);
                        }
                    }
                }
                /* rows of dq for queries are complete for this head */
            }
            for (int j = 0; j < Nk; ++j) {
                double* dkj = dk + (((size_t)b * Nk + j) * Hkv + g) * (size_t)d;
                double* dvj = dv + (((size_t)b * Nk + j) * Hkv + g) * (size_t)d;
                for (int t = 0; t < d; ++t) {
                    if (j < Lk) {
                        dkj[t] = scale * csum_value(&dk_acc[(size_t)j * d + t]);
                        dvj[t] = csum_value(&dv_acc[(size_t)j * d + t]);
                    } else { /* keys behind the real length get no gradient */
                        dkj[t] = 0.0;
                        dvj[t] = 0.0;
                    }
                }
            }
        }
        free(P);
        free(dS);
        free(dk_acc);
        free(dv_acc);
    }
    return err ? -2 : 0;
}

/* oracle_attn_bwd_mask without a block mask */
int oracle_attn_bwd(const double* q, const double* k, const double* v, const double* dout,
                    double* dq, double* dk, double* dv, int B, int Hq, int Hkv, int Nq, int Nk,
                    int d, double scale, int causal, const int* seqlens_k, int window_left) {
    return oracle_attn_bwd_mask(q, k, v, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                seqlens_k, window_left, NULL, 0, 0, 0, 0, 1, 1);
}

/*
 * Attention of new query tokens against a PAGED KV cache: the cache is cut
 * into fixed blocks of block_size rows and sequence b's logical key j lives
 * in physical block block_table[b][j / block_size], row j % block_size.
 * (The ai6s.net article, adaptation point 3, has a pre-allocated cache that
 * grows one row per token; paging is the same cache with its rows found
 * through a table instead of one contiguous slice per sequence.)
 *   q        [B, Nq, Hq, d]
 *   k_cache, v_cache [num_blocks, block_size, Hkv, d]
 *   block_table [B, max_blocks]; seqlens_k [B] (<= max_blocks * block_size)
 *   o [B, Nq, Hq, d], lse [B, Hq, Nq]; causal is bottom-right, as above.
 * Each sequence's keys are gathered into a contiguous scratch and attended
 * exactly as in oracle_attn_kvcache.  Returns 0, -1 (bad arguments, or a
 * table entry outside [0, num_blocks) for a filled block) or -2.
 */
int oracle_attn_paged(const double* q, const double* k_cache, const double* v_cache,
                      const int* block_table, int max_blocks, int block_size, int num_blocks,
                      const int* seqlens_k, double* o, double* lse, int B, int Hq, int Hkv, int Nq,
                      int d, double scale, int causal) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || d <= 0 || Hq % Hkv != 0 || block_size <= 0 ||
        max_blocks <= 0 || num_blocks <= 0)
        return -1;
    int maxlen = 0;
    for (int b = 0; b < B; ++b) {
        const int L = seqlens_k[b];
        if (L < 0 || L > max_blocks * block_size) return -1;
        for (int i = 0; i < (L + block_size - 1) / block_size; ++i) {
            const int blk = block_table[(size_t)b * max_blocks + i];
            if (blk < 0 || blk >= num_blocks) return -1;
        }
        if (L > maxlen) maxlen = L;
    }
    const int G = Hq / Hkv;
    const size_t m1 = (size_t)(maxlen > 0 ? maxlen : 1);
    const size_t per_thread = ((size_t)Nq * m1 + 2 * m1 * (size_t)d) * sizeof(double);
    const int nthreads = pick_threads(per_thread);
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        const int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        const int Lk = seqlens_k[b];
        double* S = (double*)malloc((size_t)Nq * m1 * sizeof(double));
        double* kg = (double*)malloc(m1 * (size_t)d * sizeof(double));
        double* vg = (double*)malloc(m1 * (size_t)d * sizeof(double));
        const double** qp = (const double**)malloc(sizeof(double*) * (size_t)Nq);
        double** op = (double**)malloc(sizeof(double*) * (size_t)Nq);
        double** lp = (double**)malloc(sizeof(double*) * (size_t)Nq);
        int* ri = (int*)malloc(sizeof(int) * (size_t)Nq);
        if (!S || !kg || !vg || !qp || !op || !lp || !ri) {
#pragma omp atomic write
            err = 1;
        } else {
            for (int j = 0; j < Lk; ++j) { /* gather the sequence's rows through the table */
                const int blk = block_table[(size_t)b * max_blocks + j / block_size];
                const size_t row = (size_t)blk * block_size + (size_t)(j % block_size);
                memcpy(kg + (size_t)j * d, k_cache + (row * Hkv + g) * (size_t)d,
                       sizeof(double) * (size_t)d);
                memcpy(vg + (size_t)j * d, v_cache + (row * Hkv + g) * (size_t)d,
                       sizeof(double) * (size_t)d);
            }
            for (int i = 0; i < Nq; ++i) {
                ri[i] = i;
                qp[i] = q + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                op[i] = o + (((size_t)b * Nq + i) * Hq + h) * (size_t)d;
                lp[i] = lse + ((size_t)b * Hq + h) * (size_t)Nq + i;
            }
            attend_head(Nq, qp, ri, kg, vg, (long)d, Nq, Lk, d, scale, causal, -1, &nomask, op, lp,
                        S);
        }
        free(S);
        free(kg);
        free(vg);
        free(qp);
        free(op);
        free(lp);
        free(ri);
    }
    return err ? -2 : 0;
}

/*
 * CPU oracle for exact softmax attention, forward and backward, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library.  The GPU library
 * shares no code with it and never calls it.
 *
 * What it computes (the plain definition, no blocking, no fusion):
 *   the pages define attention as S = QK^T, P = softmax(S) row by row,
 *   O = PV ("flash attention io aware", section "The Memory Bandwidth
 *   Bottleneck"), and say the tiled method reaches exactly this
 *   result ("FlashAttention" glossary, online-softmax paragraph: output
 *   identical to the two-pass version).  The statistics kept for the
 *   backward pass are the running max m and sum l ("FlashAttention"
 *   glossary, recomputation paragraph); they are stored here as one
 *   logsumexp per row, lse = m + ln(l), natural log.
 *
 *   For batch b, query head h, kv head g = h / (Hq / Hkv) (contiguous groups,
 *   "Flash Attention" glossary, grouped-query attention paragraph):
 *     s_ij  = scale * sum_c q_ic k_jc,   s_ij = -inf for j > i when causal,
 *             and, with a sliding window of W keys, -inf for j <= i - W
 *             (query i sees keys i-W+1 .. i: the banded pattern is the
 *             plainest instance of the block-sparse attention that the
 *             "FlashAttention" glossary's block-sparse entry describes),
 *             and, with a block mask M of blocks of bq query rows by bk
 *             keys (the general form of that entry: blocks the mask hides
 *             are skipped), -inf where M[h][i / bq][j / bk] = 0
 *     m_i   = max_j s_ij                                (pass 1)
 *     l_i   = sum_j exp(s_ij - m_i)                     (pass 2)
 *     P_ij  = exp(s_ij - m_i) / l_i
 *     O_i   = sum_j P_ij v_j
 *     lse_i = m_i + ln(l_i)
 *   A row that sees no key at all (possible only under a block mask) has
 *   P_i. = 0, O_i = 0 and lse_i = -inf, and contributes nothing to the
 *   gradients.
 *
 *   Backward (the pages print no formula; this is the calculus of
 *   y = softmax(x) applied to the definition above, summed over the query
 *   heads of a group for dK and dV):
 *     dV_j  = sum_i P_ij dO_i
 *     dP_ij = dO_i . v_j
 *     D_i   = sum_j P_ij dP_ij
 *     dS_ij = P_ij (dP_ij - D_i)
 *     dQ_i  = scale * sum_j dS_ij k_j
 *     dK_j  = scale * sum_i dS_ij q_i
 *
 * Dropout (optional; the pages name dropout among the operations the kernel
 * fuses, "Flash Attention" glossary, kernel-fusion paragraph, and give no
 * rule): inverted dropout on the probabilities with an 8-bit threshold t,
 *     P'_ij = P_ij * Z_ij * 256 / (256 - t),   Z_ij = [u8_ij >= t],
 *     O_i   = sum_j P'_ij v_j           (lse_i is that of P, undropped)
 *     dV_j  = sum_i P'_ij dO_i,  dP_ij = (dO_i . v_j) * Z_ij * 256/(256-t),
 *     D_i, dS, dQ, dK as above with this dP (D_i = dO_i . O_i still holds).
 * u8_ij is a byte of Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel
 * random numbers: as easy as 1, 2, 3", SC 2011) with key (seed_lo, seed_hi)
 * and counter (j / 4, i / 4, b * Hq + h, 0): byte j % 4 of output word i % 4.
 *
 * FP8 forward (the FlashAttention-3 paragraph of the "FlashAttention" glossary
 * names FP8 low-precision attention and gives no rule): Q, K and V arrive as
 * 8-bit E4M3 codes with one fp32 dequantisation factor per tensor, and the
 * result is the definition above applied to the dequantised values
 * delta_q * Q8, delta_k * K8, delta_v * V8.  This file supplies the exact
 * decode of the codes (oracle_e4m3_decode); the product delta * x of an E4M3
 * value (4 significant bits) and an fp32 factor (24 bits) is exact in fp64.
 *
 * Layouts: all arrays are dense row-major fp64.
 *   q, o, dout, dq : [B][Hq][N][d]
 *   k, v, dk, dv   : [B][Hkv][N][d]
 *   lse            : [B][Hq][N]
 *
 * Threads: work items are independent (one head, or one kv head with its
 * query group), handed out through an atomic counter; nthreads <= 0 means
 * every online core.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef int64_t i64;

/* ------------------------------------------------------------------------ */
/* E4M3: the 8-bit float with 4 exponent and 3 fraction bits (the E4M3 format
 * of the OCP 8-bit floating point specification, as NVIDIA's FP8 tensor cores
 * take it).  Bit 7 is the sign; bits 6..3 hold the exponent field e with bias
 * 7; bits 2..0 hold the fraction f.  e = 0 gives the subnormals (f / 8) * 2^-6,
 * e = 1..15 gives (1 + f / 8) * 2^(e - 7), except that e = 15 with f = 7 is NaN.
 * There is no infinity; the largest finite magnitude is 1.75 * 2^8 = 448.     */

static double e4m3_value(uint8_t code) {
    const int sign = code >> 7, e = (code >> 3) & 15, f = code & 7;
    double mag;
    if (e == 15 && f == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)f / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)f / 8.0, e - 7);
    return sign ? -mag : mag;
}

void oracle_e4m3_decode(const uint8_t *codes, i64 n, double *out) {
    for (i64 i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
}

/* ------------------------------------------------------------------------ */
/* a minimal thread pool: run fn(ctx, item) for item in [0, n_items)          */

typedef void (*item_fn)(void *ctx, i64 item);

typedef struct {
    item_fn fn;
    void *ctx;
    i64 n_items;
    i64 next; /* accessed with __atomic builtins */
} pool_t;

static void *pool_worker(void *arg) {
    pool_t *p = (pool_t *)arg;
    for (;;) {
        i64 it = __atomic_fetch_add(&p->next, 1, __ATOMIC_RELAXED);
        if (it >= p->n_items) break;
        p->fn(p->ctx, it);
    }
    return NULL;
}

static int resolve_threads(int nthreads) {
    if (nthreads > 0) return nthreads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static void run_pool(item_fn fn, void *ctx, i64 n_items, int nthreads) {
    pool_t p = {fn, ctx, n_items, 0};
    int nt = resolve_threads(nthreads);
    if (nt > n_items) nt = (int)(n_items > 0 ? n_items : 1);
    if (nt <= 1) {
        pool_worker(&p);
        return;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    for (int t = 0; t < nt; ++t) pthread_create(&th[t], NULL, pool_worker, &p);
    for (int t = 0; t < nt; ++t) pthread_join(th[t], NULL);
    free(th);
}

int oracle_num_threads(int nthreads) { return resolve_threads(nthreads); }

/* ------------------------------------------------------------------------ */
/* shared problem description                                                */

typedef struct {
    const double *q, *k, *v, *dout;
    double *o, *lse, *dq, *dk, *dv;
    i64 B, Hq, Hkv, N, d;
    double scale;
    int causal;
    i64 window; /* 0: no window; W > 0: key j hidden from query i when j <= i - W */
    /* dropout: drop_t = 0 means none */
    int drop_t;
    uint32_t seed_lo, seed_hi;
    /* row / column subsets */
    const i64 *rows;
    i64 nrows;
    i64 b_sel, hkv_sel;
    /* online-softmax block size */
    i64 block;
    /* block mask (NULL: none): key j visible to query i of query head h only
     * when bmask[h * bm_hstride + (i / bm_bq) * bm_nbk + j / bm_bk] != 0 */
    const uint8_t *bmask;
    i64 bm_hstride, bm_bq, bm_bk, bm_nbk;
} prob_t;

/* Installs a block mask of bq x bk blocks ([Hq or 1][ceil(N/bq)][ceil(N/bk)]
 * bytes, head stride hstride: 0 shares one mask among the heads).  P->N must
 * be set.  Returns nonzero for an invalid description. */
static int set_block_mask(prob_t *P, const uint8_t *bmask, i64 hstride, i64 bq, i64 bk) {
    P->bmask = bmask;
    if (!bmask) return 0;
    if (bq <= 0 || bk <= 0 || hstride < 0) return 1;
    P->bm_hstride = hstride;
    P->bm_bq = bq;
    P->bm_bk = bk;
    P->bm_nbk = (P->N + bk - 1) / bk;
    return 0;
}

static const double *head_ptr(const double *base, i64 b, i64 h, i64 H, i64 N, i64 d) {
    return base + ((b * H + h) * N) * d;
}

static double dot(const double *a, const double *b, i64 d) {
    double s = 0.0;
    for (i64 c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, as defined by Salmon et al. (SC 2011): ten rounds of
 *   (hi0, lo0) = M0 * c0,  (hi1, lo1) = M1 * c2   (32 x 32 -> 64-bit products)
 *   c = (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)
 * with the key bumped by the Weyl constants (W0, W1) between rounds.        */

void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += W0;
            k1 += W1;
        }
        const uint64_t p0 = (uint64_t)M0 * c0, p1 = (uint64_t)M1 * c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Dropout factor of (query head bh, query i, key j): 0 when dropped, else
 * 256 / (256 - t).  1 when dropout is off. */
static double drop_factor(const prob_t *P, i64 bh, i64 i, i64 j) {
    if (P->drop_t == 0) return 1.0;
    const uint32_t ctr[4] = {(uint32_t)(j >> 2), (uint32_t)(i >> 2), (uint32_t)bh, 0u};
    const uint32_t key[2] = {P->seed_lo, P->seed_hi};
    uint32_t x[4];
    oracle_philox4x32_10(ctr, key, x);
    const uint32_t u8 = (x[i & 3] >> (8 * (j & 3))) & 0xFFu;
    return u8 >= (uint32_t)P->drop_t ? 256.0 / (256.0 - P->drop_t) : 0.0;
}

/* Key j is hidden from query i of query head h: after it under a causal
 * mask, W or more keys before it under a sliding window of W keys, or in a
 * block that the block mask hides. */
static int hidden(const prob_t *P, i64 h, i64 i, i64 j) {
    return (P->causal && j > i) || (P->window > 0 && j <= i - P->window) ||
           (P->bmask && !P->bmask[h * P->bm_hstride + (i / P->bm_bq) * P->bm_nbk + j / P->bm_bk]);
}

/* Scores of one query row against every key: s[j] = scale * q_i . k_j, with
 * -inf for masked keys.  Returns the number of unmasked keys. */
static i64 score_row(const prob_t *P, i64 h, const double *qi, const double *kh, i64 i, double *s) {
    i64 n_valid = 0;
    for (i64 j = 0; j < P->N; ++j) {
        if (hidden(P, h, i, j)) {
            s[j] = -INFINITY;
        } else {
            s[j] = P->scale * dot(qi, kh + j * P->d, P->d);
            ++n_valid;
        }
    }
    return n_valid;
}

/* Two-pass softmax of one row in place: s -> P.  Writes m and l.  A row
 * with every score -inf (no visible key) gives P = 0, m = -inf, l = 0. */
static void softmax_row_two_pass(double *s, i64 N, double *m_out, double *l_out) {
    double m = -INFINITY;
    for (i64 j = 0; j < N; ++j)
        if (s[j] > m) m = s[j]; /* pass 1: max */
    if (m == -INFINITY) {
        for (i64 j = 0; j < N; ++j) s[j] = 0.0;
        *m_out = m;
        *l_out = 0.0;
        return;
    }
    double l = 0.0;
    for (i64 j = 0; j < N; ++j) l += exp(s[j] - m); /* pass 2: sum */
    for (i64 j = 0; j < N; ++j) s[j] = exp(s[j] - m) / l;
    *m_out = m;
    *l_out = l;
}

/* ------------------------------------------------------------------------ */
/* forward, full: materialises the N x N matrix of one head                  */

static void fwd_full_item(void *ctx, i64 item) {
    const prob_t *P = (const prob_t *)ctx;
    const i64 N = P->N, d = P->d, group = P->Hq / P->Hkv;
    const i64 b = item / P->Hq, h = item % P->Hq, g = h / group;
    const double *qh = head_ptr(P->q, b, h, P->Hq, N, d);
    const double *kh = head_ptr(P->k, b, g, P->Hkv, N, d);
    const double *vh = head_ptr(P->v, b, g, P->Hkv, N, d);
    double *oh = P->o + ((b * P->Hq + h) * N) * d;
    double *lseh = P->lse + (b * P->Hq + h) * N;

    double *S = (double *)malloc(sizeof(double) * (size_t)(N * N));
    for (i64 i = 0; i < N; ++i) score_row(P, h, qh + i * d, kh, i, S + i * N);
    for (i64 i = 0; i < N; ++i) {
        double m, l;
        softmax_row_two_pass(S + i * N, N, &m, &l);
        lseh[i] = m + log(l);
    }
    /* O = P' V (P' = P with dropout applied) */
    for (i64 i = 0; i < N; ++i) {
        double *oi = oh + i * d;
        for (i64 c = 0; c < d; ++c) oi[c] = 0.0;
        for (i64 j = 0; j < N; ++j) {
            const double p = S[i * N + j] * drop_factor(P, b * P->Hq + h, i, j);
            const double *vj = vh + j * d;
            for (i64 c = 0; c < d; ++c) oi[c] += p * vj[c];
        }
    }
    free(S);
}

int oracle_fwd(const double *q, const double *k, const double *v, double *o, double *lse,
               i64 B, i64 Hq, i64 Hkv, i64 N, i64 d, double scale, int causal, i64 window,
               int drop_t, uint32_t seed_lo, uint32_t seed_hi,
               const uint8_t *bmask, i64 bm_hstride, i64 bm_bq, i64 bm_bk, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || window < 0 ||
        drop_t < 0 || drop_t > 255) return 1;
    prob_t P = {0};
    P.window = window; P.drop_t = drop_t; P.seed_lo = seed_lo; P.seed_hi = seed_hi;
    P.q = q; P.k = k; P.v = v; P.o = o; P.lse = lse;
    P.B = B; P.Hq = Hq; P.Hkv = Hkv; P.N = N; P.d = d; P.scale = scale; P.causal = causal;
    if (set_block_mask(&P, bmask, bm_hstride, bm_bq, bm_bk)) return 1;
    if (N > 0) run_pool(fwd_full_item, &P, B * Hq, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* forward, selected query rows of every head (row-streamed form of the same
 * formulas: each output row depends on its own query row only)              */

static void fwd_rows_item(void *ctx, i64 item) {
    const prob_t *P = (const prob_t *)ctx;
    const i64 N = P->N, d = P->d, group = P->Hq / P->Hkv;
    const i64 bh = item / P->nrows, r = item % P->nrows;
    const i64 b = bh / P->Hq, h = bh % P->Hq, g = h / group;
    const i64 i = P->rows[r];
    const double *qi = head_ptr(P->q, b, h, P->Hq, N, d) + i * d;
    const double *kh = head_ptr(P->k, b, g, P->Hkv, N, d);
    const double *vh = head_ptr(P->v, b, g, P->Hkv, N, d);
    double *oi = P->o + (bh * P->nrows + r) * d;

    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    score_row(P, h, qi, kh, i, s);
    double m, l;
    softmax_row_two_pass(s, N, &m, &l);
    P->lse[bh * P->nrows + r] = m + log(l);
    for (i64 c = 0; c < d; ++c) oi[c] = 0.0;
    for (i64 j = 0; j < N; ++j) {
        const double *vj = vh + j * d;
        const double pj = s[j] * drop_factor(P, bh, i, j);
        for (i64 c = 0; c < d; ++c) oi[c] += pj * vj[c];
    }
    free(s);
}

/* o_rows: [B][Hq][nrows][d], lse_rows: [B][Hq][nrows] */
int oracle_fwd_rows(const double *q, const double *k, const double *v, const i64 *rows, i64 nrows,
                    double *o_rows, double *lse_rows, i64 B, i64 Hq, i64 Hkv, i64 N, i64 d,
                    double scale, int causal, i64 window, int drop_t,
                    uint32_t seed_lo, uint32_t seed_hi, const uint8_t *bmask, i64 bm_hstride, i64 bm_bq, i64 bm_bk, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || nrows < 0 || window < 0 ||
        drop_t < 0 || drop_t > 255)
        return 1;
    for (i64 r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return 2;
    prob_t P = {0};
    P.window = window; P.drop_t = drop_t; P.seed_lo = seed_lo; P.seed_hi = seed_hi;
    P.q = q; P.k = k; P.v = v; P.o = o_rows; P.lse = lse_rows; P.rows = rows; P.nrows = nrows;
    P.B = B; P.Hq = Hq; P.Hkv = Hkv; P.N = N; P.d = d; P.scale = scale; P.causal = causal;
    if (set_block_mask(&P, bmask, bm_hstride, bm_bq, bm_bk)) return 1;
    if (nrows > 0) run_pool(fwd_rows_item, &P, B * Hq * nrows, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* forward by the online (one-pass, blocked) softmax, the method the pages
 * describe: keep a running max m and running sum l, and rescale the partial
 * sums when the max grows ("FlashAttention" glossary, online-softmax
 * paragraph; "flash attention io aware", section "Online Softmax").  This is
 * NOT the definition; it exists so a test can check, in fp64, that the
 * one-pass recurrence reaches the two-pass result.                          */

static void fwd_online_item(void *ctx, i64 item) {
    const prob_t *P = (const prob_t *)ctx;
    const i64 N = P->N, d = P->d, group = P->Hq / P->Hkv, Bc = P->block;
    const i64 b = item / P->Hq, h = item % P->Hq, g = h / group;
    const double *qh = head_ptr(P->q, b, h, P->Hq, N, d);
    const double *kh = head_ptr(P->k, b, g, P->Hkv, N, d);
    const double *vh = head_ptr(P->v, b, g, P->Hkv, N, d);
    double *oh = P->o + ((b * P->Hq + h) * N) * d;
    double *lseh = P->lse + (b * P->Hq + h) * N;
    double *s = (double *)malloc(sizeof(double) * (size_t)Bc);

    for (i64 i = 0; i < N; ++i) {
        double m = -INFINITY, l = 0.0;
        double *acc = oh + i * d;
        for (i64 c = 0; c < d; ++c) acc[c] = 0.0;
        for (i64 j0 = 0; j0 < N; j0 += Bc) {
            const i64 nb = (j0 + Bc <= N) ? Bc : N - j0;
            double mb = -INFINITY;
            for (i64 t = 0; t < nb; ++t) {
                const i64 j = j0 + t;
                s[t] = hidden(P, h, i, j) ? -INFINITY : P->scale * dot(qh + i * d, kh + j * d, d);
                if (s[t] > mb) mb = s[t];
            }
            if (mb == -INFINITY) continue; /* block fully masked */
            const double m_new = mb > m ? mb : m;
            const double corr = exp(m - m_new); /* 0 when m = -inf */
            l *= corr;
            for (i64 c = 0; c < d; ++c) acc[c] *= corr;
            for (i64 t = 0; t < nb; ++t) {
                const double p = exp(s[t] - m_new);
                l += p;
                const double pd = p * drop_factor(P, b * P->Hq + h, i, j0 + t);
                const double *vj = vh + (j0 + t) * d;
                for (i64 c = 0; c < d; ++c) acc[c] += pd * vj[c];
            }
            m = m_new;
        }
        if (l == 0.0) { /* no visible key: O = 0, lse = -inf */
            lseh[i] = -INFINITY;
            continue;
        }
        for (i64 c = 0; c < d; ++c) acc[c] /= l;
        lseh[i] = m + log(l);
    }
    free(s);
}

int oracle_fwd_online(const double *q, const double *k, const double *v, double *o, double *lse,
                      i64 B, i64 Hq, i64 Hkv, i64 N, i64 d, double scale, int causal, i64 window,
                      int drop_t, uint32_t seed_lo, uint32_t seed_hi, const uint8_t *bmask, i64 bm_hstride, i64 bm_bq, i64 bm_bk, 
                      i64 block, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || block <= 0 || window < 0 ||
        drop_t < 0 || drop_t > 255)
        return 1;
    prob_t P = {0};
    P.window = window; P.drop_t = drop_t; P.seed_lo = seed_lo; P.seed_hi = seed_hi;
    P.q = q; P.k = k; P.v = v; P.o = o; P.lse = lse; P.block = block;
    P.B = B; P.Hq = Hq; P.Hkv = Hkv; P.N = N; P.d = d; P.scale = scale; P.causal = causal;
    if (set_block_mask(&P, bmask, bm_hstride, bm_bq, bm_bk)) return 1;
    if (N > 0) run_pool(fwd_online_item, &P, B * Hq, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* backward, full: one work item = one kv head and all query heads of its
 * group, so that dK and dV are summed without sharing between threads.      */

static void bwd_full_item(void *ctx, i64 item) {
    const prob_t *P = (const prob_t *)ctx;
    const i64 N = P->N, d = P->d, group = P->Hq / P->Hkv;
    const i64 b = item / P->Hkv, g = item % P->Hkv;
    const double *kh = head_ptr(P->k, b, g, P->Hkv, N, d);
    const double *vh = head_ptr(P->v, b, g, P->Hkv, N, d);
    double *dkh = P->dk + ((b * P->Hkv + g) * N) * d;
    double *dvh = P->dv + ((b * P->Hkv + g) * N) * d;
    memset(dkh, 0, sizeof(double) * (size_t)(N * d));
    memset(dvh, 0, sizeof(double) * (size_t)(N * d));

    double *Pm = (double *)malloc(sizeof(double) * (size_t)(N * N));
    double *dP = (double *)malloc(sizeof(double) * (size_t)(N * N));
    for (i64 h = g * group; h < (g + 1) * group; ++h) {
        const double *qh = head_ptr(P->q, b, h, P->Hq, N, d);
        const double *doh = head_ptr(P->dout, b, h, P->Hq, N, d);
        double *dqh = P->dq + ((b * P->Hq + h) * N) * d;
        /* recompute P from the definition */
        for (i64 i = 0; i < N; ++i) {
            double m, l;
            score_row(P, h, qh + i * d, kh, i, Pm + i * N);
            softmax_row_two_pass(Pm + i * N, N, &m, &l);
        }
        /* dP = dO V^T, times the dropout factor (dP of P, not of P') */
        for (i64 i = 0; i < N; ++i)
            for (i64 j = 0; j < N; ++j) dP[i * N + j] = dot(doh + i * d, vh + j * d, d);
        if (P->drop_t)
            for (i64 i = 0; i < N; ++i)
                for (i64 j = 0; j < N; ++j) dP[i * N + j] *= drop_factor(P, b * P->Hq + h, i, j);
        /* dS = P o (dP - D), D_i = sum_j P_ij dP_ij; stored in place of dP */
        for (i64 i = 0; i < N; ++i) {
            double D = 0.0;
            for (i64 j = 0; j < N; ++j) D += Pm[i * N + j] * dP[i * N + j];
            for (i64 j = 0; j < N; ++j) dP[i * N + j] = Pm[i * N + j] * (dP[i * N + j] - D);
        }
        /* dQ = scale dS K ; dK += scale dS^T Q ; dV += P^T dO */
        for (i64 i = 0; i < N; ++i) {
            double *dqi = dqh + i * d;
            for (i64 c = 0; c < d; ++c) dqi[c] = 0.0;
            for (i64 j = 0; j < N; ++j) {
                const double ds = dP[i * N + j];
                const double p = Pm[i * N + j] * drop_factor(P, b * P->Hq + h, i, j); /* P' */
                const double *kj = kh + j * d;
                const double *qi = qh + i * d;
                const double *doi = doh + i * d;
                double *dkj = dkh + j * d;
                double *dvj = dvh + j * d;
                for (i64 c = 0; c < d; ++c) {
                    dqi[c] += P->scale * ds * kj[c];
                    dkj[c] += P->scale * ds * qi[c];
                    dvj[c] += p * doi[c];
                }
            }
        }
    }
    free(Pm);
    free(dP);
}

int oracle_bwd(const double *q, const double *k, const double *v, const double *dout, double *dq,
               double *dk, double *dv, i64 B, i64 Hq, i64 Hkv, i64 N, i64 d, double scale,
               int causal, i64 window, int drop_t, uint32_t seed_lo, uint32_t seed_hi,
               const uint8_t *bmask, i64 bm_hstride, i64 bm_bq, i64 bm_bk, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || window < 0 ||
        drop_t < 0 || drop_t > 255) return 1;
    prob_t P = {0};
    P.window = window; P.drop_t = drop_t; P.seed_lo = seed_lo; P.seed_hi = seed_hi;
    P.q = q; P.k = k; P.v = v; P.dout = dout; P.dq = dq; P.dk = dk; P.dv = dv;
    P.B = B; P.Hq = Hq; P.Hkv = Hkv; P.N = N; P.d = d; P.scale = scale; P.causal = causal;
    if (set_block_mask(&P, bmask, bm_hstride, bm_bq, bm_bk)) return 1;
    if (N > 0) run_pool(bwd_full_item, &P, B * Hkv, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* backward, dQ of selected query rows of every head.  dQ_i depends on query
 * row i only: P_i. and dP_i. over all keys, D_i from the same row.           */

static void bwd_rows_item(void *ctx, i64 item) {
    const prob_t *P = (const prob_t *)ctx;
    const i64 N = P->N, d = P->d, group = P->Hq / P->Hkv;
    const i64 bh = item / P->nrows, r = item % P->nrows;
    const i64 b = bh / P->Hq, h = bh % P->Hq, g = h / group;
    const i64 i = P->rows[r];
    const double *qi = head_ptr(P->q, b, h, P->Hq, N, d) + i * d;
    const double *doi = head_ptr(P->dout, b, h, P->Hq, N, d) + i * d;
    const double *kh = head_ptr(P->k, b, g, P->Hkv, N, d);
    const double *vh = head_ptr(P->v, b, g, P->Hkv, N, d);
    double *dqi = P->dq + (bh * P->nrows + r) * d;

    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    double m, l;
    score_row(P, h, qi, kh, i, p);
    softmax_row_two_pass(p, N, &m, &l);
    double D = 0.0;
    for (i64 j = 0; j < N; ++j) {
        dp[j] = dot(doi, vh + j * d, d);
        dp[j] *= drop_factor(P, bh, i, j);
        D += p[j] * dp[j];
    }
    for (i64 c = 0; c < d; ++c) dqi[c] = 0.0;
    for (i64 j = 0; j < N; ++j) {
        const double ds = p[j] * (dp[j] - D);
        if (ds == 0.0) continue;
        const double *kj = kh + j * d;
        for (i64 c = 0; c < d; ++c) dqi[c] += P->scale * ds * kj[c];
    }
    free(p);
    free(dp);
}

/* dq_rows: [B][Hq][nrows][d] */
int oracle_bwd_rows(const double *q, const double *k, const double *v, const double *dout,
                    const i64 *rows, i64 nrows, double *dq_rows, i64 B, i64 Hq, i64 Hkv, i64 N,
                    i64 d, double scale, int causal, i64 window, int drop_t,
                    uint32_t seed_lo, uint32_t seed_hi, const uint8_t *bmask, i64 bm_hstride, i64 bm_bq, i64 bm_bk, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || nrows < 0 || window < 0 ||
        drop_t < 0 || drop_t > 255)
        return 1;
    for (i64 r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return 2;
    prob_t P = {0};
    P.window = window; P.drop_t = drop_t; P.seed_lo = seed_lo; P.seed_hi = seed_hi;
    P.q = q; P.k = k; P.v = v; P.dout = dout; P.dq = dq_rows; P.rows = rows; P.nrows = nrows;
    P.B = B; P.Hq = Hq; P.Hkv = Hkv; P.N = N; P.d = d; P.scale = scale; P.causal = causal;
    if (set_block_mask(&P, bmask, bm_hstride, bm_bq, bm_bk)) return 1;
    if (nrows > 0) run_pool(bwd_rows_item, &P, B * Hq * nrows, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* backward, dK and dV of selected key rows of one kv head (b_sel, hkv_sel).
 * dK_j and dV_j need P_ij over every query row i of every head in the group,
 * so the per-row statistics (m_i, l_i) and D_i are computed first for every
 * row (one O(N^2 d) pass per head); then each selected column is summed.
 * With a causal mask only rows i >= min(selected j) contribute, so the
 * statistics are computed for those rows only.                              */

typedef struct {
    const prob_t *P;
    i64 h;          /* query head being processed */
    i64 i_lo;       /* first query row that can contribute */
    double *m, *l;  /* [N] per-row max and sum */
    double *D;      /* [N] per-row D_i */
} colstat_t;

static void col_stats_item(void *ctx, i64 item) {
    colstat_t *C = (colstat_t *)ctx;
    const prob_t *P = C->P;
    const i64 N = P->N, d = P->d, g = P->hkv_sel, b = P->b_sel, h = C->h;
    const i64 i = C->i_lo + item;
    const double *qi = head_ptr(P->q, b, h, P->Hq, N, d) + i * d;
    const double *doi = head_ptr(P->dout, b, h, P->Hq, N, d) + i * d;
    const double *kh = head_ptr(P->k, b, g, P->Hkv, N, d);
    const double *vh = head_ptr(P->v, b, g, P->Hkv, N, d);
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double m, l;
    score_row(P, h, qi, kh, i, p);
    softmax_row_two_pass(p, N, &m, &l);
    double D = 0.0;
    for (i64 j = 0; j < N; ++j)
        if (p[j] != 0.0) D += p[j] * dot(doi, vh + j * d, d) * drop_factor(P, b * P->Hq + h, i, j);
    C->m[i] = m;
    C->l[i] = l;
    C->D[i] = D;
    free(p);
}

typedef struct {
    const prob_t *P;
    const colstat_t *stats; /* one per group head */
    i64 group;
} colsum_t;

static void col_sum_item(void *ctx, i64 r) {
    const colsum_t *C = (const colsum_t *)ctx;
    const prob_t *P = C->P;
    const i64 N = P->N, d = P->d, g = P->hkv_sel, b = P->b_sel;
    const i64 j = P->rows[r];
    const double *kj = head_ptr(P->k, b, g, P->Hkv, N, d) + j * d;
    const double *vj = head_ptr(P->v, b, g, P->Hkv, N, d) + j * d;
    double *dkj = P->dk + r * d;
    double *dvj = P->dv + r * d;
    for (i64 c = 0; c < d; ++c) dkj[c] = dvj[c] = 0.0;
    for (i64 t = 0; t < C->group; ++t) {
        const colstat_t *S = &C->stats[t];
        const double *qh = head_ptr(P->q, b, S->h, P->Hq, N, d);
        const double *doh = head_ptr(P->dout, b, S->h, P->Hq, N, d);
        for (i64 i = S->i_lo; i < N; ++i) {
            if (hidden(P, S->h, i, j)) continue;
            const double s = P->scale * dot(qh + i * d, kj, d);
            const double p = exp(s - S->m[i]) / S->l[i];
            const double f = drop_factor(P, b * P->Hq + S->h, i, j);
            const double dp = dot(doh + i * d, vj, d) * f;
            const double ds = p * (dp - S->D[i]);
            for (i64 c = 0; c < d; ++c) {
                dvj[c] += p * f * doh[i * d + c];
                dkj[c] += P->scale * ds * qh[i * d + c];
            }
        }
    }
}

/* dk_cols, dv_cols: [ncols][d] for kv rows cols[] of kv head (b_sel, hkv_sel) */
int oracle_bwd_cols(const double *q, const double *k, const double *v, const double *dout,
                    i64 b_sel, i64 hkv_sel, const i64 *cols, i64 ncols, double *dk_cols,
                    double *dv_cols, i64 B, i64 Hq, i64 Hkv, i64 N, i64 d, double scale,
                    int causal, i64 window, int drop_t, uint32_t seed_lo, uint32_t seed_hi,
                    const uint8_t *bmask, i64 bm_hstride, i64 bm_bq, i64 bm_bk, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || N < 0 || d <= 0 || Hq % Hkv || ncols < 0 || window < 0 ||
        drop_t < 0 || drop_t > 255)
        return 1;
    if (b_sel < 0 || b_sel >= B || hkv_sel < 0 || hkv_sel >= Hkv) return 2;
    i64 j_min = N;
    for (i64 r = 0; r < ncols; ++r) {
        if (cols[r] < 0 || cols[r] >= N) return 2;
        if (cols[r] < j_min) j_min = cols[r];
    }
    if (ncols == 0) return 0;
    const i64 group = Hq / Hkv;
    prob_t P = {0};
    P.q = q; P.k = k; P.v = v; P.dout = dout; P.dk = dk_cols; P.dv = dv_cols;
    P.rows = cols; P.nrows = ncols; P.b_sel = b_sel; P.hkv_sel = hkv_sel; P.window = window; P.drop_t = drop_t; P.seed_lo = seed_lo; P.seed_hi = seed_hi;
    P.B = B; P.Hq = Hq; P.Hkv = Hkv; P.N = N; P.d = d; P.scale = scale; P.causal = causal;
    if (set_block_mask(&P, bmask, bm_hstride, bm_bq, bm_bk)) return 1;

    const i64 i_lo = causal ? j_min : 0;
    colstat_t *stats = (colstat_t *)calloc((size_t)group, sizeof(colstat_t));
    for (i64 t = 0; t < group; ++t) {
        stats[t].P = &P;
        stats[t].h = hkv_sel * group + t;
        stats[t].i_lo = i_lo;
        stats[t].m = (double *)malloc(sizeof(double) * (size_t)N);
        stats[t].l = (double *)malloc(sizeof(double) * (size_t)N);
        stats[t].D = (double *)malloc(sizeof(double) * (size_t)N);
        run_pool(col_stats_item, &stats[t], N - i_lo, nthreads);
    }
    colsum_t C = {&P, stats, group};
    run_pool(col_sum_item, &C, ncols, nthreads);
    for (i64 t = 0; t < group; ++t) {
        free(stats[t].m);
        free(stats[t].l);
        free(stats[t].D);
    }
    free(stats);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode over a paged key/value cache (the serving workload of the pages:
 * "Paper digest: FlashAttention", section "Limits", names decode-time
 * attention over a KV cache; the "Flash Attention" glossary's PagedAttention
 * entry stores that cache in fixed-size blocks found through a table).
 * Sequence b holds seq_lens[b] = L cached tokens, its last Nq being the new
 * queries: query t (position L - Nq + t) sees keys 0 .. L - Nq + t.  Key k of
 * sequence b lives in physical page block_table[b][k / P], slot k % P.
 *   q        [B][Hq][Nq][d]          o [B][Hq][Nq][d], lse [B][Hq][Nq]
 *   k_cache  [num_pages][Hkv][P][d]  v_cache likewise
 *   block_table [B][max_pages] (int64 here), seq_lens [B]
 * Plain definition: gather the visible keys, two-pass softmax, O = P V.     */

typedef struct {
    const double *q, *kc, *vc;
    const i64 *table, *lens;
    double *o, *lse;
    i64 B, Hq, Hkv, Nq, d, P, max_pages, num_pages;
    double scale;
} decode_t;

static void decode_item(void *ctx, i64 item) {
    const decode_t *D = (const decode_t *)ctx;
    const i64 d = D->d, group = D->Hq / D->Hkv;
    const i64 t = item % D->Nq, h = (item / D->Nq) % D->Hq, b = item / (D->Nq * D->Hq);
    const i64 g = h / group, L = D->lens[b];
    const i64 n_vis = L - D->Nq + t + 1; /* keys 0 .. L - Nq + t */
    const double *qi = D->q + ((b * D->Hq + h) * D->Nq + t) * d;
    double *oi = D->o + ((b * D->Hq + h) * D->Nq + t) * d;
    double *s = (double *)malloc(sizeof(double) * (size_t)(n_vis > 0 ? n_vis : 1));
    for (i64 kk = 0; kk < n_vis; ++kk) {
        const i64 page = D->table[b * D->max_pages + kk / D->P], slot = kk % D->P;
        const double *kr = D->kc + ((page * D->Hkv + g) * D->P + slot) * d;
        s[kk] = D->scale * dot(qi, kr, d);
    }
    double m, l;
    softmax_row_two_pass(s, n_vis, &m, &l);
    D->lse[(b * D->Hq + h) * D->Nq + t] = m + log(l);
    for (i64 c = 0; c < d; ++c) oi[c] = 0.0;
    for (i64 kk = 0; kk < n_vis; ++kk) {
        const i64 page = D->table[b * D->max_pages + kk / D->P], slot = kk % D->P;
        const double *vr = D->vc + ((page * D->Hkv + g) * D->P + slot) * d;
        for (i64 c = 0; c < d; ++c) oi[c] += s[kk] * vr[c];
    }
    free(s);
}

int oracle_decode_paged(const double *q, const double *k_cache, const double *v_cache,
                        const i64 *block_table, const i64 *seq_lens, double *o, double *lse,
                        i64 B, i64 Hq, i64 Hkv, i64 Nq, i64 d, i64 page_size, i64 max_pages,
                        i64 num_pages, double scale, int nthreads) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Nq <= 0 || d <= 0 || page_size <= 0 ||
        max_pages < 0 || num_pages < 0)
        return 1;
    for (i64 b = 0; b < B; ++b) {
        const i64 L = seq_lens[b];
        if (L < Nq || L > max_pages * page_size) return 2;
        for (i64 p = 0; p < (L + page_size - 1) / page_size; ++p) {
            const i64 pg = block_table[b * max_pages + p];
            if (pg < 0 || pg >= num_pages) return 2;
        }
    }
    decode_t D = {q, k_cache, v_cache, block_table, seq_lens, o, lse,
                  B, Hq, Hkv, Nq, d, page_size, max_pages, num_pages, scale};
    if (B > 0) run_pool(decode_item, &D, B * Hq * Nq, nthreads);
    return 0;
}

/*
 * fp2_oracle.c -- plain CPU oracle of block-sparse prefill attention with a
 * block-mean score estimator, a max-relative threshold and a mean correction
 * (the method described in "FlashPrefill V2: Block-Sparse Prefill Attention for
 * Long-Context LLM Serving", lode.cx write-up, section "How It Works"; the
 * aimodeling.com write-up, section "From Prototype to Production").
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this file.  It shares no code, header
 * or constant with the CUDA library; the two meet only through the seeded
 * inputs.  All arithmetic is IEEE double (no fast-math), one plain loop per
 * definition below, no blocking or fusion beyond what the definition states.
 * (-DORC_FP32 builds the same code in float: the timed CPU baseline only.)
 * OpenMP only splits independent (q-block, head) rows across host cores.
 *
 * Definitions (the pages give them in words only; where they are silent the
 * plainest reading is taken and named):
 *   D0 blocks   Request b of length L_b is cut into blocks of Bs rows starting
 *               at its first token (blocks of one fixed size: 345tool.com page,
 *               section "Why block-sparse attention for prefill?"; queries and
 *               keys both cut into blocks: stuffinsider page, "Technical
 *               Details").  n_j = rows of block j.  Token r sees tokens c <= r of
 *               the same request (causal prefill).
 *               Chunked form (prefill of the last Lq_b of Lk_b tokens, the first
 *               P_b = Lk_b - Lq_b already in the KV cache; the pages name paged KV
 *               and continuous batching but not this case, so the plainest
 *               extension is taken): key blocks as above over Lk_b; query row t
 *               is position P_b + t; query blocks keep the same absolute grid, so
 *               q-block i holds the positions of [i Bs, i Bs + Bs) that are in
 *               [P_b, Lk_b) and the first one may be partial.  Position p sees
 *               keys c <= p.  With P_b = 0 this is the plain definition.
 *   D1 estimate xbar_j = (1/n_j) sum_{r in j} x_r for x in {q, k, v}
 *               (the lode.cx page, "How It Works", estimates the scores from a
 *               small sample and the aipulsen page does so per block; read here
 *               as block means), and
 *               s[h,i,j] = tau * qbar[h,i] . kbar[g(h),j] for j <= i, g(h) = h / G.
 *   D2 keep     m = max_{j<=i} s[h,i,j]; head h keeps j iff s - m >= ln(alpha)
 *               (lode.cx page, "How It Works": only what clears a threshold
 *               set relative to the maximum estimated score is attended; read in
 *               the probability domain, exp(s - m) >= alpha).  A KV group keeps
 *               the union over its heads plus the diagonal block i.  alpha <= 0
 *               keeps every j <= i.
 *   D3 attend   For row r (head h) of q-block i with kept set K and pruned set
 *               P = {j < i not kept}:
 *               o = [sum_{c in K, c<=r} e^{l_c} v_c + sum_{j in P} n_j e^{lbar_j} vbar_j]
 *                 / [sum_{c in K, c<=r} e^{l_c}     + sum_{j in P} n_j e^{lbar_j}],
 *               l_c = tau q_r . k_c, lbar_j = tau q_r . kbar_j (reading of the
 *               correction term of the lode.cx page, "How It Works", which offsets
 *               the bias that dropping blocks introduces: every pruned block
 *               replaced by n_j copies of its mean key and mean value).
 *               LSE = ln(denominator).
 *   D4 e4m3     inputs are codes times a per-(tensor, head) scale; the oracle
 *               dequantises them exactly in double.
 *   D3 variants (not the method as the pages give it; compared on approximation
 *               error only): correction mode 2 adds the Gaussian second-order
 *               term to every pruned block's logit, lbar_j + (tau^2 / 2)
 *               sum_c q_c^2 var_j[c], with var_j the per-dimension key variance
 *               inside block j (the logit variance when the dimensions are
 *               uncorrelated inside the block; by Jensen the plain form
 *               undercounts a block's mass by about e^{var / 2}).  Mode 3 uses the
 *               block-pooled logit tau qbar_i . kbar_j, shared by all rows of
 *               q-block i, instead of the row's own.  Mode 4 is mode 2 with the
 *               key variance averaged over the dimensions, (tau^2 / 2) |q|^2
 *               mean_c var_j[c]: one scalar per row times one per block.
 *
 * Pins (tests/oracle_pins.py), each against a fact outside this file:
 *   D0, D3 core   torch scaled_dot_product_attention in fp64 at alpha <= 0
 *                 (plain and chunked, ragged lengths, an empty request);
 *   D1            numpy means; the score equals the brute-force mean token logit;
 *   D2            hand-derived golden cases; forced diagonal; nesting in alpha;
 *                 packed heads equal each head alone;
 *   D3 correction exact on block-constant K/V (plain and chunked); weights sum to 1;
 *   D4            power-of-two scaled inputs;
 *   D3 variants   numpy variance of the token logits; the pooled form reduces to
 *                 the row-wise one.
 * The pages print no worked example or value, so the readings named above
 * (mean pooling, the threshold in the exp domain, the form of the correction,
 * the chunked block grid) are parity unpinned by the pages themselves: the pins
 * fix the arithmetic given each reading.
 *
 * Build with -DORC_MUTANT=n to plant one deliberate mistake (see the MUT()
 * sites); the oracle self-tests check that every such mistake is caught.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORC_MUTANT
#define ORC_MUTANT 0
#endif

/* The arithmetic type: IEEE double for the parity reference; the same code
 * built with -DORC_FP32 runs in float (the timed CPU baseline only; parity is
 * always checked against the double build). */
#ifdef ORC_FP32
typedef float real;
#define EXP expf
#define LOG logf
#else
typedef double real;
#define EXP exp
#define LOG log
#endif
#define MUT(n) (ORC_MUTANT == (n))

/* D0: number of blocks of a request of length L. */
static int64_t nblocks(int64_t L, int64_t Bs) { return (L + Bs - 1) / Bs; }

/* D0 (chunked form): rows at request positions pos0 .. pos0 + L - 1 lie in the
 * blocks floor(pos0 / Bs) .. ceil((pos0 + L) / Bs) - 1. */
static int64_t first_block(int64_t pos0, int64_t Bs) { return pos0 / Bs; }
static int64_t blocks_at(int64_t pos0, int64_t L, int64_t Bs) {
    return L > 0 ? nblocks(pos0 + L, Bs) - first_block(pos0, Bs) : 0;
}

/* D0: first global block id of every request (cb[B] = total blocks); the rows
 * of request b start at position pos0[b] (pos0 NULL: at 0). */
static void block_offsets(const int32_t* cu, const int64_t* pos0, int B, int Bs, int64_t* cb) {
    cb[0] = 0;
    for (int b = 0; b < B; ++b) cb[b + 1] = cb[b] + blocks_at(pos0 ? pos0[b] : 0, cu[b + 1] - cu[b], Bs);
}

/* D0 (chunked form): P_b = Lk_b - Lq_b, the position of the first query row.
 * NULL when a request has Lq_b < 0 or Lq_b > Lk_b.  The caller frees it. */
static int64_t* chunk_starts(const int32_t* cu_q, const int32_t* cu_k, int B) {
    int64_t* P = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    for (int b = 0; b < B; ++b) {
        int64_t Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
        if (Lq < 0 || Lq > Lk) { free(P); return NULL; }
        P[b] = Lk - Lq;
    }
    return P;
}

/* Total blocks of a batch whose request b starts at position pos0[b] (NULL: 0). */
int64_t orc_total_blocks(const int32_t* cu, const int64_t* pos0, int B, int Bs) {
    int64_t t = 0;
    for (int b = 0; b < B; ++b) t += blocks_at(pos0 ? pos0[b] : 0, cu[b + 1] - cu[b], Bs);
    return t;
}

/* D1: block means of a dequantised input x[T, H, d] (value * scale[h]).  Row
 * t of request b is at position pos0[b] + t (pos0 NULL: 0); the mean of a
 * block runs over its positions that hold rows.  out: [total_blocks, H, d]. */
void orc_block_means(const float* x, const real* scale, const int32_t* cu, const int64_t* pos0,
                     int B, int H, int d, int Bs, real* out) {
    int64_t* cb = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    block_offsets(cu, pos0, B, Bs, cb);
    for (int b = 0; b < B; ++b) {
        int64_t L = cu[b + 1] - cu[b];
        int64_t p0 = pos0 ? pos0[b] : 0;
        int64_t i0 = first_block(p0, Bs);
        int64_t nb = blocks_at(p0, L, Bs);
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < nb; ++t) {
            int64_t i = i0 + t;
            int64_t lo = i * Bs > p0 ? i * Bs : p0;                       /* first position */
            int64_t hi = (i + 1) * Bs < p0 + L ? (i + 1) * Bs : p0 + L;   /* one past the last */
            real denom = MUT(5) ? (real)Bs
                         : MUT(13) ? (real)(hi - i * Bs)              /* mutant: counts P's rows */
                         : (real)(hi - lo);
            for (int h = 0; h < H; ++h) {
                for (int c = 0; c < d; ++c) {
                    real s = 0.0;
                    for (int64_t p = lo; p < hi; ++p) {
                        int64_t row = cu[b] + (p - p0);
                        s += (real)x[(row * H + h) * (int64_t)d + c] * scale[h];
                    }
                    out[((cb[b] + t) * H + h) * (int64_t)d + c] = s / denom;
                }
            }
        }
    }
    free(cb);
}

/* Per-dimension variance of the dequantised rows inside every block, around the
 * block means `mean` (from orc_block_means with the same arguments):
 * out[t, h, c] = (1/n) sum_{r in t} (x[r, h, c] * scale[h] - mean[t, h, c])^2. */
void orc_block_vars(const float* x, const real* scale, const int32_t* cu, const int64_t* pos0,
                    int B, int H, int d, int Bs, const real* mean, real* out) {
    int64_t* cb = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    block_offsets(cu, pos0, B, Bs, cb);
    for (int b = 0; b < B; ++b) {
        int64_t L = cu[b + 1] - cu[b];
        int64_t p0 = pos0 ? pos0[b] : 0;
        int64_t i0 = first_block(p0, Bs);
        int64_t nb = blocks_at(p0, L, Bs);
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < nb; ++t) {
            int64_t i = i0 + t;
            int64_t lo = i * Bs > p0 ? i * Bs : p0;
            int64_t hi = (i + 1) * Bs < p0 + L ? (i + 1) * Bs : p0 + L;
            for (int h = 0; h < H; ++h) {
                for (int c = 0; c < d; ++c) {
                    int64_t at = ((cb[b] + t) * H + h) * (int64_t)d + c;
                    real s = 0.0;
                    for (int64_t p = lo; p < hi; ++p) {
                        int64_t row = cu[b] + (p - p0);
                        real e = (real)x[(row * H + h) * (int64_t)d + c] * scale[h] - mean[at];
                        s += e * e;
                    }
                    out[at] = s / (real)(hi - lo);
                }
            }
        }
    }
    free(cb);
}

/* D1 score of one (head, q-block, k-block) pair. */
static real block_score(const real* qbar, const real* kbar, int64_t qb, int64_t kb, int h,
                          int g, int Hq, int Hkv, int d, real tau) {
    real dot = 0.0;
    for (int c = 0; c < d; ++c)
        dot += qbar[(qb * Hq + h) * (int64_t)d + c] * kbar[(kb * Hkv + g) * (int64_t)d + c];
    return MUT(7) ? dot : tau * dot;
}

/* D1 + D2: kept-block lists.
 *   qbar [total q-blocks, Hq, d] (rows at positions P_b + t, see D0), kbar
 *   [total k-blocks, Hkv, d]; request b has cu_q[b+1] - cu_q[b] query rows
 *   and cu_k[b+1] - cu_k[b] keys (cu_q == cu_k: plain prefill).
 *   kept_cnt [total q-blocks, Hkv], kept_idx [total q-blocks, Hkv, nb_max]:
 *            the request's key blocks j <= i kept by q-block i, ascending;
 *   s_out    [total q-blocks, Hq, nb_max] raw scores s (NULL to skip), entries j > i untouched;
 *   m_out    [total q-blocks, Hq] row maxima (NULL to skip).
 * Returns 0, -1 when a request has more than nb_max key blocks, -3 when one
 * has more queries than keys. */
int orc_estimate(const real* qbar, const real* kbar, const int32_t* cu_q, const int32_t* cu_k,
                 int B, int Hq, int Hkv, int d, int Bs, real tau, real alpha, int nb_max,
                 int32_t* kept_cnt, int32_t* kept_idx, real* s_out, real* m_out) {
    int G = Hq / Hkv;
    real ln_alpha = alpha > 0 ? LOG(alpha) : -INFINITY;
    int64_t* P = chunk_starts(cu_q, cu_k, B);
    if (!P) return -3;
    for (int b = 0; b < B; ++b)
        if (nblocks(cu_k[b + 1] - cu_k[b], Bs) > nb_max) { free(P); return -1; }
    int64_t* cbq = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    int64_t* cbk = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    block_offsets(cu_q, P, B, Bs, cbq);
    block_offsets(cu_k, NULL, B, Bs, cbk);
    for (int b = 0; b < B; ++b) {
        int64_t i0 = first_block(P[b], Bs);
        int64_t nbq = blocks_at(P[b], cu_q[b + 1] - cu_q[b], Bs);
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t t = 0; t < nbq; ++t) {
            int64_t i = i0 + t;                       /* block index in the request */
            int64_t qb = cbq[b] + t;                  /* global q-block id */
            real* s = (real*)malloc(sizeof(real) * (i + 1));
            unsigned char* keep = (unsigned char*)malloc(i + 1);
            for (int g = 0; g < Hkv; ++g) {
                memset(keep, 0, i + 1);
                for (int hh = 0; hh < G; ++hh) {
                    int h = g * G + hh;
                    int gk = MUT(3) ? h % Hkv : g;  /* mutant: wrong head -> group map */
                    real m = -INFINITY;
                    for (int64_t j = 0; j <= i; ++j) {
                        s[j] = block_score(qbar, kbar, qb, cbk[b] + j, h, gk, Hq, Hkv, d, tau);
                        if (s[j] > m) m = s[j];
                    }
                    for (int64_t j = 0; j <= i; ++j) {
                        int k;
                        if (alpha <= 0) k = 1;
                        else if (MUT(2)) k = s[j] >= alpha * m;          /* mutant: linear fraction */
                        else if (MUT(4)) k = s[j] - m > ln_alpha;       /* mutant: strict */
                        else k = s[j] - m >= ln_alpha;
                        if (k) keep[j] = 1;
                        if (s_out) s_out[(qb * Hq + h) * (int64_t)nb_max + j] = s[j];
                    }
                    if (m_out) m_out[qb * Hq + h] = m;
                }
                if (!MUT(8)) keep[i] = 1;
                int32_t cnt = 0;
                int32_t* idx = kept_idx + (qb * Hkv + g) * (int64_t)nb_max;
                for (int64_t j = 0; j <= i; ++j)
                    if (keep[j]) idx[cnt++] = (int32_t)j;
                kept_cnt[qb * Hkv + g] = cnt;
            }
            free(s);
            free(keep);
        }
    }
    free(P);
    free(cbq);
    free(cbk);
    return 0;
}

/* Checks one kept list: strictly ascending entries in [0, i] ending with i. */
static int list_ok(const int32_t* idx, int32_t cnt, int64_t i) {
    if (cnt < 1 || cnt > i + 1) return 0;
    for (int32_t t = 0; t < cnt; ++t) {
        if (idx[t] < 0 || idx[t] > i) return 0;
        if (t > 0 && idx[t] <= idx[t - 1]) return 0;
    }
    return idx[cnt - 1] == i;
}

/* D3: attention over the kept blocks plus (correction != 0) the mean-corrected
 * pruned blocks.
 *   q [Tq, Hq, d], k/v [Tk, Hkv, d] stored values; qs/ks/vs per-head scales;
 *   cu_q / cu_k: query rows and keys of every request (D0 chunked form;
 *   cu_q == cu_k: plain prefill);
 *   correction: 0 none, 1 mean correction (D3), 2 with the variance term, 3
 *   block-pooled, 4 with the dimension-averaged variance term (D3 variants);
 *   kbar/vbar [total k-blocks, Hkv, d] block means (needed when correction != 0);
 *   kvar [total k-blocks, Hkv, d] key variances (corrections 2, 4), qbar [total
 *   q-blocks, Hq, d] query block means (correction 3);
 *   sel: global q-block ids to compute (NULL = all), nsel entries;
 *   o [Tq, Hq, d], lse [Tq, Hq], wsum [Tq, Hq] (sum of normalised weights; NULL ok).
 * Returns 0, -1 on an invalid kept list, -2 on a bad q-block id, -3 when a
 * request has more queries than keys, -4 on a bad correction mode or a missing
 * array it needs. */
int orc_attend(const float* q, const float* k, const float* v, const real* qs, const real* ks,
               const real* vs, const int32_t* cu_q, const int32_t* cu_k, int B, int Hq, int Hkv,
               int d, int Bs, real tau, const int32_t* kept_cnt, const int32_t* kept_idx,
               int nb_max, int correction, const real* kbar, const real* vbar,
               const real* kvar, const real* qbar, const int64_t* sel, int64_t nsel,
               real* o, real* lse, real* wsum) {
    int G = Hq / Hkv;
    int64_t* P = chunk_starts(cu_q, cu_k, B);
    if (!P) return -3;
    int64_t* cbq = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    int64_t* cbk = (int64_t*)malloc(sizeof(int64_t) * (B + 1));
    block_offsets(cu_q, P, B, Bs, cbq);
    block_offsets(cu_k, NULL, B, Bs, cbk);
    int64_t total = cbq[B];
    int64_t nwork = sel ? nsel : total;
    /* request of every q-block */
    int32_t* req = (int32_t*)malloc(sizeof(int32_t) * (total > 0 ? total : 1));
    for (int b = 0; b < B; ++b)
        for (int64_t t = cbq[b]; t < cbq[b + 1]; ++t) req[t] = b;
    int status = 0;
    for (int64_t w = 0; w < nwork; ++w) {
        int64_t qb = sel ? sel[w] : w;
        if (qb < 0 || qb >= total) { status = -2; break; }
        int b = req[qb];
        int64_t i = first_block(P[b], Bs) + (qb - cbq[b]);
        for (int g = 0; g < Hkv; ++g)
            if (!list_ok(kept_idx + (qb * Hkv + g) * (int64_t)nb_max, kept_cnt[qb * Hkv + g], i))
                status = -1;
    }
    if (((correction == 2 || correction == 4) && !kvar) || (correction == 3 && !qbar) || correction < 0 ||
        correction > 4)
        status = -4;
    if (status != 0) { free(P); free(cbq); free(cbk); free(req); return status; }

#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int64_t w = 0; w < nwork; ++w) {
        for (int h = 0; h < Hq; ++h) {
            int64_t qb = sel ? sel[w] : w;
            int b = req[qb];
            int64_t p0 = P[b];                         /* position of the first query row */
            int64_t i0 = first_block(p0, Bs);
            int64_t i = i0 + (qb - cbq[b]);            /* block index in the request */
            int64_t L = cu_k[b + 1] - cu_k[b];         /* keys of the request */
            int g = MUT(3) ? h % Hkv : h / G;
            const int32_t* idx = kept_idx + (qb * Hkv + g) * (int64_t)nb_max;
            int32_t cnt = kept_cnt[qb * Hkv + g];
            /* pruned set P = {j < i not kept} */
            unsigned char* kept = (unsigned char*)calloc(i + 1, 1);
            for (int32_t t = 0; t < cnt; ++t) kept[idx[t]] = 1;
            int64_t nmax = (int64_t)cnt * Bs + i + 1;
            real* lg = (real*)malloc(sizeof(real) * nmax);     /* logits */
            const real** vrow = (const real**)malloc(sizeof(real*) * nmax);
            real* vbuf = (real*)malloc(sizeof(real) * (size_t)cnt * Bs * d);
            real* qd = (real*)malloc(sizeof(real) * d);
            real* acc = (real*)malloc(sizeof(real) * d);
            int64_t lo = i * Bs > p0 ? i * Bs : p0;                   /* positions of the block's rows */
            int64_t hi = (i + 1) * Bs < L ? (i + 1) * Bs : L;
            for (int64_t p = lo; p < hi; ++p) {
                int64_t grow = cu_q[b] + (p - p0);
                for (int c = 0; c < d; ++c) qd[c] = (real)q[(grow * Hq + h) * (int64_t)d + c] * qs[h];
                int64_t n = 0;
                int64_t nv = 0;
                for (int32_t t = 0; t < cnt; ++t) {
                    int64_t j = idx[t];
                    for (int64_t cc = 0; cc < Bs; ++cc) {
                        int64_t kp = j * Bs + cc;
                        int visible = MUT(6) ? (kp < p)
                                    : MUT(12) ? (kp <= p - p0)         /* mutant: chunk-relative mask */
                                    : (kp <= p);
                        if (kp >= L || !visible) continue;
                        int64_t krow = cu_k[b] + kp;
                        real dot = 0.0;
                        for (int c = 0; c < d; ++c)
                            dot += qd[c] * ((real)k[(krow * Hkv + g) * (int64_t)d + c] * ks[g]);
                        lg[n] = tau * dot;
                        real* vr = vbuf + nv * d;
                        real vsc = MUT(10) ? 1.0 : vs[g];
                        for (int c = 0; c < d; ++c) vr[c] = (real)v[(krow * Hkv + g) * (int64_t)d + c] * vsc;
                        vrow[n] = vr;
                        ++n;
                        ++nv;
                    }
                }
                if (correction) {
                    /* mutant 14: the cached prefix's pruned blocks left out */
                    for (int64_t j = MUT(14) ? i0 : 0; j < i; ++j) {
                        if (kept[j]) continue;
                        int64_t kb = cbk[b] + j;
                        int64_t nj = (L - j * Bs) < Bs ? (L - j * Bs) : Bs;
                        const real* kj = kbar + (kb * Hkv + g) * (int64_t)d;
                        real dot = 0.0;
                        if (correction == 3) {        /* block-pooled: qbar of q-block i */
                            const real* qi = qbar + (qb * Hq + h) * (int64_t)d;
                            for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
                        } else {
                            for (int c = 0; c < d; ++c) dot += qd[c] * kj[c];
                        }
                        lg[n] = tau * dot + (MUT(1) ? 0.0 : LOG((real)nj));
                        if (correction == 2 || correction == 4) {   /* second-order (variance) term */
                            const real* vj = kvar + (kb * Hkv + g) * (int64_t)d;
                            real q2v = 0.0;
                            if (correction == 2) {
                                for (int c = 0; c < d; ++c) q2v += qd[c] * qd[c] * vj[c];
                            } else {                  /* |q|^2 times the mean variance */
                                real q2 = 0.0, vm = 0.0;
                                for (int c = 0; c < d; ++c) { q2 += qd[c] * qd[c]; vm += vj[c]; }
                                q2v = q2 * (MUT(16) ? vm : vm / d);
                            }
                            lg[n] += (MUT(15) ? 1.0 : 0.5) * tau * tau * q2v;
                        }
                        vrow[n] = (MUT(9) ? kbar : vbar) + (kb * Hkv + g) * (int64_t)d;
                        ++n;
                    }
                }
                real m = -INFINITY;
                for (int64_t t = 0; t < n; ++t) if (lg[t] > m) m = lg[t];
                real den = 0.0;
                for (int c = 0; c < d; ++c) acc[c] = 0.0;
                for (int64_t t = 0; t < n; ++t) {
                    real e = EXP(lg[t] - m);
                    den += e;
                    for (int c = 0; c < d; ++c) acc[c] += e * vrow[t][c];
                }
                for (int c = 0; c < d; ++c) o[(grow * Hq + h) * (int64_t)d + c] = acc[c] / den;
                lse[grow * Hq + h] = MUT(11) ? LOG(den) : m + LOG(den);
                if (wsum) {
                    real ws = 0.0;
                    for (int64_t t = 0; t < n; ++t) ws += EXP(lg[t] - m) / den;
                    wsum[grow * Hq + h] = ws;
                }
            }
            free(kept); free(lg); free(vrow); free(vbuf); free(qd); free(acc);
        }
    }
    free(P);
    free(cbq);
    free(cbk);
    free(req);
    return 0;
}

int orc_mutant_id(void) { return ORC_MUTANT; }

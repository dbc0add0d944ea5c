/*
 * oracle.c -- plain, slow, fp64 CPU oracle of training-free block-sparse
 * self-attention for video DiTs.  TEST INFRASTRUCTURE ONLY: the tests, the
 * smoke check and the bench's CPU-baseline leg call it; the product path never
 * does.  It shares no code, header or table with the CUDA library.
 *
 * What it computes follows the SubBlock router description on the page
 * "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), section "How SubBlock
 * sparse attention works": queries and keys are cut into 64-token blocks, a
 * light pooling step scores every key block for every query block and head, the
 * top-scoring key blocks are kept and their indices handed to an exact
 * block-sparse attention; `sparsity` is the fraction of key blocks dropped.
 * The scoring is taken in its one-sub-block form: the score of key block J for
 * query block I is mean(q over I) . mean(k over J) / sqrt(D).  The kept count
 * is ceil((1 - s) * nKV) with ties broken towards the lower block index.
 *
 * Every function is the definition written out with plain loops, in fp64,
 * in token order.  Inputs are bf16 bit patterns, widened exactly.
 *
 * Layouts: q, k, v are [B, H, Npad, D] row-major bf16; valid_len[b] is the
 * number of real tokens of sample b (rows >= valid_len[b] are padding).
 * Blocks: nB_b = ceil(valid_len[b] / block); block I holds tokens
 * [I*block, min((I+1)*block, valid_len[b])).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int n_blocks_of(int len, int block) { return (len + block - 1) / block; }

/* Kept-count rule: clamp(ceil((1 - s) * n - 1e-9), 1, n), evaluated in fp64.
 * The 1e-9 absorbs representation error such as (1 - 0.7) * 10 = 3.0000000000000004. */
int32_t oracle_keep_count(int32_t n, double sparsity) {
    if (n <= 0) return 0;
    double x = ceil((1.0 - sparsity) * (double)n - 1e-9);
    if (x < 1.0) x = 1.0;
    if (x > (double)n) x = (double)n;
    return (int32_t)x;
}

/* Mean of each block over its valid tokens.  out: [B, H, nBmax, D] with
 * nBmax = Npad / block; blocks at or past nB_b are written as 0. */
void oracle_pool(const uint16_t* x, int B, int H, int Npad, int D,
                 const int32_t* valid_len, int block, double* out) {
    int nBmax = Npad / block;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const uint16_t* xs = x + ((size_t)b * H + h) * (size_t)Npad * D;
            int L = valid_len[b];
            for (int I = 0; I < nBmax; ++I) {
                double* o = out + (((size_t)b * H + h) * nBmax + I) * D;
                int n0 = I * block, n1 = n0 + block < L ? n0 + block : L;
                for (int d = 0; d < D; ++d) {
                    double s = 0.0;
                    for (int n = n0; n < n1; ++n) s += bf16_to_f64(xs[(size_t)n * D + d]);
                    o[d] = (n1 > n0) ? s / (double)(n1 - n0) : 0.0;
                }
            }
        }
}

/* Block scores S[b,h,I,J] = sum_d qbar[I,d] * kbar[J,d] * (1/sqrt(D)) for
 * I, J < nB_b; entries outside that square are NAN.  S: [B, H, nBmax, nBmax]. */
void oracle_scores(const double* qbar, const double* kbar, int B, int H, int nBmax, int D,
                   const int32_t* valid_len, int block, double* S) {
    double inv = 1.0 / sqrt((double)D);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            int nB = n_blocks_of(valid_len[b], block);
            const double* qb = qbar + ((size_t)b * H + h) * nBmax * D;
            const double* kb = kbar + ((size_t)b * H + h) * nBmax * D;
            double* Sb = S + ((size_t)b * H + h) * nBmax * nBmax;
            for (int I = 0; I < nBmax; ++I)
                for (int J = 0; J < nBmax; ++J) {
                    if (I >= nB || J >= nB) { Sb[(size_t)I * nBmax + J] = NAN; continue; }
                    double s = 0.0;
                    for (int d = 0; d < D; ++d) s += qb[(size_t)I * D + d] * kb[(size_t)J * D + d];
                    Sb[(size_t)I * nBmax + J] = s * inv;
                }
        }
    }
}

typedef struct { double score; int32_t index; } scored_block;

/* Order: higher score first; equal scores -> lower block index first.  This is a
 * total order, so the sort result does not depend on the sort's stability. */
static int by_score_desc_index_asc(const void* pa, const void* pb) {
    const scored_block* a = (const scored_block*)pa;
    const scored_block* b = (const scored_block*)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->index > b->index) - (a->index < b->index);
}

static int int_asc(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* Top-k routing over precomputed scores S ([B,H,nBmax,nBmax], see oracle_scores).
 * For each (b, h) and query block I < nB_b keep the k_b = keep(nB_b, s) best key
 * blocks, written ascending to kv_idx[b,h,I,0..k_b) ([B,H,nBmax,kmax], unused
 * tail entries = -1) with kv_cnt[b,h,I] = k_b; query blocks past nB_b get 0.
 * Returns 0, or -1 when some k_b exceeds kmax. */
int oracle_topk(const double* S, int B, int H, int nBmax, const int32_t* valid_len,
                int block, double sparsity, int kmax, int32_t* kv_idx, int32_t* kv_cnt) {
    int status = 0;
    for (int b = 0; b < B; ++b)
        if (oracle_keep_count(n_blocks_of(valid_len[b], block), sparsity) > kmax) status = -1;
#pragma omp parallel
    {
        scored_block* row = (scored_block*)malloc(sizeof(scored_block) * (size_t)(nBmax > 0 ? nBmax : 1));
#pragma omp for collapse(2) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h) {
                int nB = n_blocks_of(valid_len[b], block);
                int k = oracle_keep_count(nB, sparsity);
                if (k > kmax) k = kmax;
                for (int I = 0; I < nBmax; ++I) {
                    size_t r = ((size_t)b * H + h) * nBmax + I;
                    int32_t* idx = kv_idx + r * kmax;
                    for (int t = 0; t < kmax; ++t) idx[t] = -1;
                    if (I >= nB) { kv_cnt[r] = 0; continue; }
                    for (int J = 0; J < nB; ++J) {
                        row[J].score = S[r * nBmax + J];
                        row[J].index = J;
                    }
                    qsort(row, (size_t)nB, sizeof(scored_block), by_score_desc_index_asc);
                    for (int t = 0; t < k; ++t) idx[t] = row[t].index;
                    qsort(idx, (size_t)k, sizeof(int32_t), int_asc);
                    kv_cnt[r] = k;
                }
            }
        free(row);
    }
    return status;
}

/* Whole selection: pool Q and K, score, route.  pooled_q / pooled_k / scores may
 * be NULL; when given they receive the intermediate fp64 values. */
int oracle_select(const uint16_t* q, const uint16_t* k, int B, int H, int Npad, int D,
                  const int32_t* valid_len, int block, double sparsity, int kmax,
                  int32_t* kv_idx, int32_t* kv_cnt,
                  double* pooled_q, double* pooled_k, double* scores) {
    int nBmax = Npad / block;
    size_t np_ = (size_t)B * H * nBmax * D, ns = (size_t)B * H * nBmax * nBmax;
    double* pq = pooled_q ? pooled_q : (double*)malloc(sizeof(double) * np_);
    double* pk = pooled_k ? pooled_k : (double*)malloc(sizeof(double) * np_);
    double* S = scores ? scores : (double*)malloc(sizeof(double) * ns);
    oracle_pool(q, B, H, Npad, D, valid_len, block, pq);
    oracle_pool(k, B, H, Npad, D, valid_len, block, pk);
    oracle_scores(pq, pk, B, H, nBmax, D, valid_len, block, S);
    int st = oracle_topk(S, B, H, nBmax, valid_len, block, sparsity, kmax, kv_idx, kv_cnt);
    if (!pooled_q) free(pq);
    if (!pooled_k) free(pk);
    if (!scores) free(S);
    return st;
}

/* Softmax attention of one query row over an explicit token list.
 * logits_j = scale * sum_d q_d k_jd;  m = max_j logits_j;  p_j = exp(logits_j - m);
 * Z = sum_j p_j;  o = sum_j p_j v_j / Z;  lse = m + log(Z).  An empty list gives
 * o = 0 and lse = -inf.  buf holds the logits (n_tok entries). */
static void attend_row(const uint16_t* qrow, const uint16_t* ks, const uint16_t* vs, int D,
                       const int32_t* tok, int n_tok, double scale, double* buf,
                       double* orow, double* lse, double* probs_out) {
    for (int d = 0; d < D; ++d) orow[d] = 0.0;
    if (n_tok == 0) { *lse = -INFINITY; return; }
    double m = -INFINITY;
    for (int t = 0; t < n_tok; ++t) {
        const uint16_t* kr = ks + (size_t)tok[t] * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += bf16_to_f64(qrow[d]) * bf16_to_f64(kr[d]);
        buf[t] = scale * s;
        if (buf[t] > m) m = buf[t];
    }
    double Z = 0.0;
    for (int t = 0; t < n_tok; ++t) { buf[t] = exp(buf[t] - m); Z += buf[t]; }
    for (int t = 0; t < n_tok; ++t) {
        const uint16_t* vr = vs + (size_t)tok[t] * D;
        double w = buf[t] / Z;
        if (probs_out) probs_out[tok[t]] = w;
        for (int d = 0; d < D; ++d) orow[d] += w * bf16_to_f64(vr[d]);
    }
    *lse = m + log(Z);
}

/* Valid tokens of the kept blocks of one routing row, ascending.  Returns the
 * count, or -1 if a block index is outside [0, nB_b). */
static int kept_tokens(const int32_t* idx, int cnt, int nB, int L, int block, int32_t* tok) {
    int n = 0;
    for (int t = 0; t < cnt; ++t) {
        int J = idx[t];
        if (J < 0 || J >= nB) return -1;
        for (int j = J * block; j < (J + 1) * block && j < L; ++j) tok[n++] = j;
    }
    return n;
}

/* Block-sparse attention with an external routing (kv_idx [B,H,nBmax,kmax],
 * kv_cnt [B,H,nBmax]); nBmax = Npad / block.  For every valid query row i of
 * query block I the row attends to the valid tokens of the blocks kv_idx[b,h,I,
 * 0..kv_cnt).  Rows past valid_len[b] get o = 0 and lse = -inf.
 * qblocks (NULL = all) restricts the work to the listed query blocks of every
 * (b, h); rows outside them are left untouched.  scale <= 0 means 1/sqrt(D).
 * o: [B,H,Npad,D] fp64, lse: [B,H,Npad] fp64.  Returns 0, or -1 on a routing
 * entry outside the sample's blocks. */
int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int B, int H, int Npad, int D, const int32_t* valid_len, int block,
                     const int32_t* kv_idx, const int32_t* kv_cnt, int kmax, double scale,
                     const int32_t* qblocks, int n_qblocks, double* o, double* lse) {
    int nBmax = Npad / block;
    int nq = qblocks ? n_qblocks : nBmax;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
    int status = 0;
#pragma omp parallel
    {
        int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)Npad);
        double* buf = (double*)malloc(sizeof(double) * (size_t)Npad);
#pragma omp for collapse(3) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h)
                for (int qi = 0; qi < nq; ++qi) {
                    int I = qblocks ? qblocks[qi] : qi;
                    int L = valid_len[b], nB = n_blocks_of(L, block);
                    size_t bh = (size_t)b * H + h;
                    const uint16_t* ks = k + bh * (size_t)Npad * D;
                    const uint16_t* vs = v + bh * (size_t)Npad * D;
                    size_t r = bh * nBmax + I;
                    int n = kept_tokens(kv_idx + r * kmax, kv_cnt[r], nB, L, block, tok);
                    if (n < 0) {
#pragma omp atomic write
                        status = -1;
                        n = 0;
                    }
                    for (int i = I * block; i < (I + 1) * block; ++i) {
                        double* orow = o + (bh * Npad + i) * D;
                        double* l = lse + bh * Npad + i;
                        if (i >= L) {
                            for (int d = 0; d < D; ++d) orow[d] = 0.0;
                            *l = -INFINITY;
                            continue;
                        }
                        attend_row(q + (bh * Npad + i) * D, ks, vs, D, tok, n, scale, buf,
                                   orow, l, NULL);
                    }
                }
        free(tok);
        free(buf);
    }
    return status;
}

/* Dense softmax attention over all valid tokens of the sample (no routing). */
void oracle_dense(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                  int B, int H, int Npad, int D, const int32_t* valid_len, double scale,
                  double* o, double* lse) {
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
#pragma omp parallel
    {
        int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)Npad);
        double* buf = (double*)malloc(sizeof(double) * (size_t)Npad);
#pragma omp for collapse(3) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h)
                for (int i = 0; i < Npad; ++i) {
                    int L = valid_len[b];
                    size_t bh = (size_t)b * H + h;
                    double* orow = o + (bh * Npad + i) * D;
                    double* l = lse + bh * Npad + i;
                    if (i >= L) {
                        for (int d = 0; d < D; ++d) orow[d] = 0.0;
                        *l = -INFINITY;
                        continue;
                    }
                    for (int j = 0; j < L; ++j) tok[j] = j;
                    attend_row(q + (bh * Npad + i) * D, k + bh * (size_t)Npad * D,
                               v + bh * (size_t)Npad * D, D, tok, L, scale, buf, orow, l, NULL);
                }
        free(tok);
        free(buf);
    }
}

/* Probability row of query row i of (b, h) under a routing: probs[j] for
 * j in [0, Npad), zero outside the kept valid tokens.  Returns 0 or -1. */
int oracle_probs(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 int B, int H, int Npad, int D, const int32_t* valid_len, int block,
                 const int32_t* kv_idx, const int32_t* kv_cnt, int kmax, double scale,
                 int b, int h, int i, double* probs) {
    (void)B;
    int nBmax = Npad / block, L = valid_len[b], nB = n_blocks_of(L, block);
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
    for (int j = 0; j < Npad; ++j) probs[j] = 0.0;
    if (i >= L) return 0;
    size_t bh = (size_t)b * H + h, r = bh * nBmax + i / block;
    int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)Npad);
    double* buf = (double*)malloc(sizeof(double) * (size_t)Npad);
    double* orow = (double*)malloc(sizeof(double) * (size_t)D);
    double lse;
    int n = kept_tokens(kv_idx + r * kmax, kv_cnt[r], nB, L, block, tok);
    int st = 0;
    if (n < 0) st = -1;
    else attend_row(q + (bh * Npad + i) * D, k + bh * (size_t)Npad * D, v + bh * (size_t)Npad * D,
                    D, tok, n, scale, buf, orow, &lse, probs);
    free(tok); free(buf); free(orow);
    return st;
}

/* ---------------------------------------------------------------------------
 * Sub-block log-sum-exp router (the SubBlock router with n_q = n_k = nsub).
 * Same page and section as above: each 64-token block is split into nsub
 * sub-blocks of block/nsub tokens; pooling and a log-sum-exp estimate the
 * unnormalised softmax mass of each key block for each query block and head:
 *   score(I, J) = log sum_{a,b} c_{I,a} c_{J,b} exp(qbar_{I,a} . kbar_{J,b} / sqrt(D))
 * where qbar_{I,a} is the mean of the valid q rows of sub-block a of block I and
 * c_{I,a} their count (empty sub-blocks contribute nothing).  The kept count is
 * keep(nB, s), optionally rounded up to a multiple of `budget` (at most nB).
 * The log-sum-exp is evaluated as m + log(sum exp(x - m)), m = max x.
 * ------------------------------------------------------------------------- */
int oracle_select_lse(const uint16_t* q, const uint16_t* k, int B, int H, int Npad, int D,
                      const int32_t* valid_len, int block, int nsub, double sparsity, int budget,
                      int kmax, int32_t* kv_idx, int32_t* kv_cnt, double* scores) {
    if (nsub < 1 || nsub > 16 || block % nsub != 0) return -2;
    const int sub = block / nsub;
    const int nBmax = Npad / block;
    const int nS = Npad / sub;
    const double inv = 1.0 / sqrt((double)D);
    size_t np_ = (size_t)B * H * nS * D, ns = (size_t)B * H * nBmax * nBmax;
    double* pq = (double*)malloc(sizeof(double) * np_);
    double* pk = (double*)malloc(sizeof(double) * np_);
    double* S = scores ? scores : (double*)malloc(sizeof(double) * ns);
    oracle_pool(q, B, H, Npad, D, valid_len, sub, pq);   /* sub-block means */
    oracle_pool(k, B, H, Npad, D, valid_len, sub, pk);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const int L = valid_len[b], nB = n_blocks_of(L, block);
            const double* qb = pq + ((size_t)b * H + h) * nS * D;
            const double* kb = pk + ((size_t)b * H + h) * nS * D;
            double* Sb = S + ((size_t)b * H + h) * nBmax * nBmax;
            double x[256];
            for (int I = 0; I < nBmax; ++I)
                for (int J = 0; J < nBmax; ++J) {
                    if (I >= nB || J >= nB) { Sb[(size_t)I * nBmax + J] = NAN; continue; }
                    int nx = 0;
                    for (int a = 0; a < nsub; ++a) {
                        const int sa = I * nsub + a, n0a = sa * sub;
                        const int ca = (L - n0a) < 0 ? 0 : ((L - n0a) > sub ? sub : (L - n0a));
                        if (ca == 0) continue;
                        for (int c = 0; c < nsub; ++c) {
                            const int sc_ = J * nsub + c, n0c = sc_ * sub;
                            const int cc = (L - n0c) < 0 ? 0 : ((L - n0c) > sub ? sub : (L - n0c));
                            if (cc == 0) continue;
                            double s = 0.0;
                            for (int d = 0; d < D; ++d) s += qb[(size_t)sa * D + d] * kb[(size_t)sc_ * D + d];
                            x[nx++] = s * inv + log((double)ca) + log((double)cc);
                        }
                    }
                    double m = -INFINITY;
                    for (int t = 0; t < nx; ++t) if (x[t] > m) m = x[t];
                    double z = 0.0;
                    for (int t = 0; t < nx; ++t) z += exp(x[t] - m);
                    Sb[(size_t)I * nBmax + J] = m + log(z);
                }
        }
    /* kept count with the optional budget rounding, then the same top-k as above */
    int status = 0;
    int32_t* vl_k = (int32_t*)malloc(sizeof(int32_t) * (size_t)B);
    for (int b = 0; b < B; ++b) vl_k[b] = valid_len[b];
#pragma omp parallel
    {
        scored_block* row = (scored_block*)malloc(sizeof(scored_block) * (size_t)(nBmax > 0 ? nBmax : 1));
#pragma omp for collapse(2) schedule(dynamic)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h) {
                const int nB = n_blocks_of(vl_k[b], block);
                int kk = oracle_keep_count(nB, sparsity);
                if (budget > 1) {
                    kk = ((kk + budget - 1) / budget) * budget;
                    if (kk > nB) kk = nB;
                }
                if (kk > kmax) {
#pragma omp atomic write
                    status = -1;
                    kk = kmax;
                }
                for (int I = 0; I < nBmax; ++I) {
                    size_t r = ((size_t)b * H + h) * nBmax + I;
                    int32_t* idx = kv_idx + r * kmax;
                    for (int t = 0; t < kmax; ++t) idx[t] = -1;
                    if (I >= nB) { kv_cnt[r] = 0; continue; }
                    for (int J = 0; J < nB; ++J) {
                        row[J].score = S[r * nBmax + J];
                        row[J].index = J;
                    }
                    qsort(row, (size_t)nB, sizeof(scored_block), by_score_desc_index_asc);
                    for (int t = 0; t < kk; ++t) idx[t] = row[t].index;
                    qsort(idx, (size_t)kk, sizeof(int32_t), int_asc);
                    kv_cnt[r] = kk;
                }
            }
        free(row);
    }
    free(vl_k);
    free(pq);
    free(pk);
    if (!scores) free(S);
    return status;
}

/* ---------------------------------------------------------------------------
 * The producer step before the router: QK RMSNorm with 3D RoPE, then block
 * pooling.  The page "MiniMax-H3 on 8xH200 benchmark", section on the kernel
 * layer, fuses the QK RMSNorm and the 3D RoPE of the attention inputs into one
 * kernel, with head dimension 128 and RoPE dimension 96, on the rounding path
 * that rounds the normalised value before the rotation.  Per (b, h, token n):
 *   y_d = bf16( x_d / sqrt(mean_e(x_e^2) + eps) * w_d )        (RMSNorm over D)
 *   channels [0, rope_dim) form three axes of da = rope_dim/3 channels, for the
 *   token's (t, y, x) position; channel pair (2i, 2i+1) of axis a turns by
 *   theta = pos_a * base^(-2i/da):
 *       o_2i   = bf16( y_2i cos(theta) - y_2i+1 sin(theta) )
 *       o_2i+1 = bf16( y_2i sin(theta) + y_2i+1 cos(theta) )
 *   channels [rope_dim, D) pass through: o_d = y_d.
 * bf16() rounds an fp64 value to the nearest bf16 value, ties to even.
 * ------------------------------------------------------------------------- */

/* Nearest bf16 value (8 significant bits, exponent range of fp32, ties to even)
 * of a finite double, as bits.  Rounds once, directly from the double. */
static uint16_t bf16_rne(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    double a = fabs(v), r;
    if (a < ldexp(1.0, -126)) {
        r = rint(a / ldexp(1.0, -133)) * ldexp(1.0, -133);   /* subnormal grid */
    } else {
        int e;
        double m = frexp(a, &e);          /* a = m 2^e, m in [0.5, 1) */
        r = ldexp(rint(ldexp(m, 8)), e - 8);  /* 8 significant bits, ties to even */
    }
    float f = (float)(signbit(v) ? -r : r);  /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* x: bf16 [B,H,Npad,D]; w: bf16 [D]; pos: int32 [B][Npad][3] (t, y, x).
 * out: bf16 [B,H,Npad,D], every row computed; out64 (optional, may be NULL):
 * fp64 [B,H,Npad,D], the rotated values before their final rounding (for pins).
 * Returns -2 if rope_dim is not a multiple of 6 in [0, D]. */
int oracle_qk_norm_rope(const uint16_t* x, const uint16_t* w, const int32_t* pos, int B, int H,
                        int Npad, int D, int rope_dim, double base, double eps, uint16_t* out,
                        double* out64) {
    if (rope_dim < 0 || rope_dim > D || rope_dim % 6 != 0) return -2;
    const int da = rope_dim / 3;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double* y = (double*)malloc(sizeof(double) * (size_t)D);
            for (int n = 0; n < Npad; ++n) {
                const size_t row = (((size_t)b * H + h) * Npad + n) * (size_t)D;
                double ss = 0.0;
                for (int d = 0; d < D; ++d) {
                    const double v = bf16_to_f64(x[row + d]);
                    ss += v * v;
                }
                const double inv = 1.0 / sqrt(ss / D + eps);
                for (int d = 0; d < D; ++d)
                    y[d] = bf16_to_f64(bf16_rne(bf16_to_f64(x[row + d]) * inv * bf16_to_f64(w[d])));
                const int32_t* p = pos + ((size_t)b * Npad + n) * 3;
                for (int d = 0; d < D; d += 2) {
                    double o0 = y[d], o1 = y[d + 1];
                    if (d < rope_dim) {
                        const int a = d / da, i = (d % da) / 2;
                        const double theta = (double)p[a] * pow(base, -2.0 * i / da);
                        const double c = cos(theta), s = sin(theta);
                        o0 = y[d] * c - y[d + 1] * s;
                        o1 = y[d] * s + y[d + 1] * c;
                    }
                    if (out64) {
                        out64[row + d] = o0;
                        out64[row + d + 1] = o1;
                    }
                    out[row + d] = bf16_rne(o0);
                    out[row + d + 1] = bf16_rne(o1);
                }
            }
            free(y);
        }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Block-sparse attention with compensation of the dropped blocks.  PISA, as the
 * page "Sol Video Inference Engine" (sjmshsh.github.io) names it in section 4.2.2
 * (Sparse Attention), computes the critical blocks exactly and compensates the
 * other blocks by a first-order Taylor approximation.  Reading taken here: for a
 * dropped block J, each token's exponential is expanded to first order about the
 * block's mean key kbar_J,
 *     exp(s q.k_j) ~ exp(s q.kbar_J) * (1 + s q.(k_j - kbar_J)).
 * Summed over the c_J valid tokens j of J, the linear term vanishes from the
 * normaliser (the deviations sum to zero about the mean) and leaves in the
 * numerator the D x D moment
 *     M_J[d][e] = sum_j (k_j[d] - kbar_J[d]) * v_j[e]:
 *   Z_i = sum_{j kept} e^{x_ij} + sum_{J dropped} c_J e^{xbar_iJ}
 *   N_i = sum_{j kept} e^{x_ij} v_j
 *       + sum_{J dropped} e^{xbar_iJ} (c_J vbar_J + s * sum_d q_i[d] M_J[d][.])
 *   o_i = N_i / Z_i,   lse_i = log Z_i
 * with x_ij = s q_i.k_j, xbar_iJ = s q_i.kbar_J, kbar_J and vbar_J the means of the
 * valid tokens of J in fp64 (token order), and "dropped" the sample's blocks
 * J < nB_b missing from the row's kept list.  The exponentials are shifted by
 * m = the largest of the kept x_ij and the dropped xbar_iJ.  The result is exact
 * when keys are constant within every dropped block, and its error shrinks with
 * the square of the keys' spread about their block means.
 *
 * order = 0 leaves the moment term out: each dropped block is then one softmax
 * entry of logit xbar_iJ + log c_J carrying vbar_J (the mean-key form, whose error
 * shrinks only linearly with the spread).
 *
 * Same arguments and outputs as oracle_attention, plus `order` (0 or 1).  Works
 * one (b, h) at a time: the block means and moments of that head, then its rows. */
int oracle_attention_compensated(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H,
                                 int Npad, int D, const int32_t* valid_len, int block, const int32_t* kv_idx,
                                 const int32_t* kv_cnt, int kmax, double scale, int order, const int32_t* qblocks,
                                 int n_qblocks, double* o, double* lse) {
    const int nBmax = Npad / block;
    const int nq = qblocks ? n_qblocks : nBmax;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
    if (order != 0 && order != 1) return -2;
    double* km = (double*)malloc(sizeof(double) * (size_t)nBmax * D);
    double* vm = (double*)malloc(sizeof(double) * (size_t)nBmax * D);
    double* M = order ? (double*)malloc(sizeof(double) * (size_t)nBmax * D * D) : NULL;
    int status = 0;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const int L = valid_len[b], nB = n_blocks_of(L, block);
            const size_t bh = (size_t)b * H + h;
            const uint16_t* ks = k + bh * (size_t)Npad * D;
            const uint16_t* vs = v + bh * (size_t)Npad * D;
            /* block means of K and V over the valid tokens, and the moments */
#pragma omp parallel for schedule(dynamic)
            for (int J = 0; J < nB; ++J) {
                const int j0 = J * block, j1 = (J + 1) * block < L ? (J + 1) * block : L;
                const double c = (double)(j1 - j0);
                for (int d = 0; d < D; ++d) {
                    double sk = 0.0, sv = 0.0;
                    for (int j = j0; j < j1; ++j) {
                        sk += bf16_to_f64(ks[(size_t)j * D + d]);
                        sv += bf16_to_f64(vs[(size_t)j * D + d]);
                    }
                    km[(size_t)J * D + d] = sk / c;
                    vm[(size_t)J * D + d] = sv / c;
                }
                if (order) {
                    double* MJ = M + (size_t)J * D * D;
                    for (int d = 0; d < D; ++d)
                        for (int e = 0; e < D; ++e) {
                            double s = 0.0;
                            for (int j = j0; j < j1; ++j)
                                s += (bf16_to_f64(ks[(size_t)j * D + d]) - km[(size_t)J * D + d]) *
                                     bf16_to_f64(vs[(size_t)j * D + e]);
                            MJ[(size_t)d * D + e] = s;
                        }
                }
            }
#pragma omp parallel
            {
                int32_t* tok = (int32_t*)malloc(sizeof(int32_t) * (size_t)Npad);
                double* lg = (double*)malloc(sizeof(double) * (size_t)(Npad + nBmax));
                double* qm = (double*)malloc(sizeof(double) * (size_t)D);
                char* kept = (char*)malloc((size_t)(nBmax > 0 ? nBmax : 1));
#pragma omp for schedule(dynamic)
                for (int qi = 0; qi < nq; ++qi) {
                    const int I = qblocks ? qblocks[qi] : qi;
                    const size_t r = bh * nBmax + I;
                    int n = kept_tokens(kv_idx + r * kmax, kv_cnt[r], nB, L, block, tok);
                    if (n < 0) {
#pragma omp atomic write
                        status = -1;
                        n = 0;
                    }
                    for (int J = 0; J < nBmax; ++J) kept[J] = 0;
                    if (n > 0)
                        for (int t = 0; t < kv_cnt[r]; ++t) kept[kv_idx[r * kmax + t]] = 1;
                    for (int i = I * block; i < (I + 1) * block; ++i) {
                        double* orow = o + (bh * Npad + i) * D;
                        double* l = lse + bh * Npad + i;
                        for (int d = 0; d < D; ++d) orow[d] = 0.0;
                        if (i >= L || I >= nB) {
                            *l = -INFINITY;
                            continue;
                        }
                        const uint16_t* qr = q + (bh * Npad + i) * D;
                        /* exponents: the kept tokens, then one per dropped block */
                        double m = -INFINITY;
                        int ne = 0;
                        for (int t = 0; t < n; ++t) {
                            const uint16_t* kr = ks + (size_t)tok[t] * D;
                            double s = 0.0;
                            for (int d = 0; d < D; ++d) s += bf16_to_f64(qr[d]) * bf16_to_f64(kr[d]);
                            lg[ne] = scale * s;
                            if (lg[ne] > m) m = lg[ne];
                            ++ne;
                        }
                        for (int J = 0; J < nB; ++J) {
                            if (kept[J]) continue;
                            double s = 0.0;
                            for (int d = 0; d < D; ++d) s += bf16_to_f64(qr[d]) * km[(size_t)J * D + d];
                            lg[ne] = scale * s;
                            if (lg[ne] > m) m = lg[ne];
                            ++ne;
                        }
                        if (ne == 0) {
                            *l = -INFINITY;
                            continue;
                        }
                        double Z = 0.0;
                        int e = 0;
                        for (int t = 0; t < n; ++t, ++e) {
                            const double w = exp(lg[e] - m);
                            const uint16_t* vr = vs + (size_t)tok[t] * D;
                            Z += w;
                            for (int d = 0; d < D; ++d) orow[d] += w * bf16_to_f64(vr[d]);
                        }
                        for (int J = 0; J < nB; ++J) {
                            if (kept[J]) continue;
                            const int c = (L - J * block) < block ? (L - J * block) : block;
                            const double w = exp(lg[e++] - m);
                            Z += (double)c * w;
                            for (int d = 0; d < D; ++d) orow[d] += w * (double)c * vm[(size_t)J * D + d];
                            if (order) {
                                /* s * q^T M_J, weighted like the block */
                                const double* MJ = M + (size_t)J * D * D;
                                for (int d = 0; d < D; ++d) qm[d] = 0.0;
                                for (int dd = 0; dd < D; ++dd) {
                                    const double qd = bf16_to_f64(qr[dd]);
                                    for (int d = 0; d < D; ++d) qm[d] += qd * MJ[(size_t)dd * D + d];
                                }
                                for (int d = 0; d < D; ++d) orow[d] += w * scale * qm[d];
                            }
                        }
                        for (int d = 0; d < D; ++d) orow[d] /= Z;
                        *l = m + log(Z);
                    }
                }
                free(tok);
                free(lg);
                free(qm);
                free(kept);
            }
        }
    free(km);
    free(vm);
    free(M);
    return status;
}

/* ---------------------------------------------------------------------------
 * Token pruning by feature-norm saliency.  The page "Sol Video Inference Engine"
 * (sjmshsh.github.io), LTX-2.3 appendix, stage 2, keeps 50% of the video tokens by
 * feat_norm saliency before the refinement transformer's first two calls.  Reading
 * taken here: the saliency of token n of sample b is the Euclidean norm of its
 * feature vector x[b][n][0..C); the kept tokens are the keep_tokens(L_b, ratio)
 * most salient of the sample's L_b valid tokens, equal norms going to the lower
 * token index, and they keep their original (raster) order, compacted to the front.
 * The norm is ranked through its square, sum_c x_c^2 summed in channel order in
 * fp64 (every square of a bf16 value is exact in fp64).
 *
 * keep_tokens(L, r) = clamp(ceil(r * L - 1e-9), 1, L) in fp64; 0 when L <= 0. */
int32_t oracle_keep_tokens(int32_t n, double ratio) {
    if (n <= 0) return 0;
    double x = ceil(ratio * (double)n - 1e-9);
    if (x < 1.0) x = 1.0;
    if (x > (double)n) x = (double)n;
    return (int32_t)x;
}

/* x: bf16 [B, N, C]; valid_len[b] <= N.  Writes norm2 [B, N] (0 past L_b),
 * idx [B, Npad_out] (kept token indices ascending, then -1) and valid_out [B].
 * Returns 0, or -1 when a kept count exceeds Npad_out. */
int oracle_token_prune(const uint16_t* x, int B, int N, int C, const int32_t* valid_len, double ratio,
                       int Npad_out, double* norm2, int32_t* idx, int32_t* valid_out) {
    int status = 0;
    for (int b = 0; b < B; ++b) {
        const int L = valid_len[b];
        double* nb = norm2 + (size_t)b * N;
#pragma omp parallel for schedule(static)
        for (int n = 0; n < N; ++n) {
            double s = 0.0;
            if (n < L) {
                const uint16_t* row = x + ((size_t)b * N + n) * C;
                for (int c = 0; c < C; ++c) {
                    const double v = bf16_to_f64(row[c]);
                    s += v * v;
                }
            }
            nb[n] = s;
        }
        const int k = oracle_keep_tokens(L, ratio);
        int32_t* ib = idx + (size_t)b * Npad_out;
        for (int p = 0; p < Npad_out; ++p) ib[p] = -1;
        valid_out[b] = k;
        if (k > Npad_out) {
            status = -1;
            continue;
        }
        scored_block* row = (scored_block*)malloc(sizeof(scored_block) * (size_t)(L > 0 ? L : 1));
        for (int n = 0; n < L; ++n) {
            row[n].score = nb[n];
            row[n].index = n;
        }
        qsort(row, (size_t)L, sizeof(scored_block), by_score_desc_index_asc);
        for (int t = 0; t < k; ++t) ib[t] = row[t].index;
        qsort(ib, (size_t)k, sizeof(int32_t), int_asc);
        free(row);
    }
    return status;
}

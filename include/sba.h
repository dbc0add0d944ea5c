/*
 * sba.h -- C ABI of the B200 (sm_100a) block-sparse self-attention library.
 *
 * The operation is training-free block-sparse self-attention over the token
 * sequence of a video diffusion transformer, as the SubBlock router is described
 * on the page "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), section
 * "How SubBlock sparse attention works": the sequence is cut into 64-token query
 * and key blocks, a light pooling step scores each key block for each query
 * block and head, the best key blocks are kept and their indices passed to an
 * exact block-sparse attention kernel that never forms the full attention
 * matrix; `sparsity` is the fraction of key blocks dropped (0.75 keeps about a
 * quarter).  This library takes the one-sub-block form of that score:
 *
 *   qbar[I] = mean of q over the valid tokens of block I (same for kbar)
 *   score[I][J] = qbar[I] . kbar[J] / sqrt(D)
 *   kept(I) = the keep(nB, s) = clamp(ceil((1 - s) * nB - 1e-9), 1, nB) key
 *             blocks of highest score, equal scores going to the lower index
 *   o_i = sum_{j in kept tokens} softmax_j(scale * q_i . k_j) v_j   (non-causal)
 *
 * Conventions shared by every call:
 *   - q, k, v, o: bf16, [B, H, Npad, D] contiguous row-major, device memory,
 *     base addresses 16-byte aligned.  D is 64 or 128.  Npad % block == 0.
 *   - valid_len: device int32 [B] with 1 <= valid_len[b] <= Npad, or NULL
 *     (every sample is Npad long).  Rows n >= valid_len[b] are padding: as keys
 *     and values they get zero weight (their contents must be finite), and their
 *     outputs are written as 0 (o) and -inf (lse).  nB_b = ceil(valid_len[b] / block).
 *   - block must be 64.
 *   - Routing: kv_idx int32 [B, H, Npad/block, kmax] and kv_cnt int32
 *     [B, H, Npad/block]; row (b, h, I) lists kv_cnt key-block indices in
 *     ascending order in its first kv_cnt entries (later entries unspecified);
 *     query blocks I >= nB_b have kv_cnt = 0.
 *   - stream: a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on that stream; the library never synchronises except in
 *     sba_get_device_status.
 *   - Inputs must be finite.
 *   - Ownership: the caller allocates and frees every buffer passed in.  The
 *     library's only device state is one error word per device.
 *   - Errors: argument checks run on the host before any launch and return an
 *     sba_status without touching device memory.  A failed launch returns
 *     SBA_ERR_CUDA.  Faults detected inside a kernel (a wait that gave up, a
 *     routing entry outside [0, nB_b)) set a device-side error word that
 *     sba_get_device_status reports.
 */
#ifndef SBA_H_
#define SBA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SBA_OK = 0,
    SBA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, sparsity outside [0,1), kmax too small */
    SBA_ERR_UNSUPPORTED = 2,   /* D not 64/128, block not 64, Npad beyond SBA_MAX_NPAD */
    SBA_ERR_ALIGNMENT = 3,     /* a device pointer not 16-byte aligned */
    SBA_ERR_CUDA = 4,          /* a CUDA runtime or driver call failed */
    SBA_ERR_TIMEOUT = 5,       /* a kernel wait gave up (reported by sba_get_device_status) */
    SBA_ERR_DEVICE_FLAG = 6,   /* a kernel found a bad routing entry (sba_get_device_status) */
    SBA_ERR_SCRATCH_TOO_SMALL = 7  /* problem too large for sba_pool_select_noalloc's fixed scratch */
} sba_status;

/* Largest padded sequence length a call accepts (4096 blocks of 64 tokens). */
#define SBA_MAX_NPAD 262144

/* Kept key blocks per query block for n_blocks candidate blocks at sparsity s
 * (same page and section: `sparsity` is the fraction of key blocks dropped):
 * clamp(ceil((1 - s) * n_blocks - 1e-9), 1, n_blocks), evaluated in fp64; 0 when
 * n_blocks <= 0.  Pure host function. */
int32_t sba_keep_count(int32_t n_blocks, double sparsity);

/* The kept count of the sub-block router with its block budget (same page and
 * section, which rounds the kept count to an 8-block budget without giving the rule):
 * sba_keep_count(n_blocks, sparsity) rounded up to a multiple of `budget`, at most
 * n_blocks.  budget = 1 gives sba_keep_count; budget < 1 returns 0.  Pure host
 * function. */
int32_t sba_keep_count_budget(int32_t n_blocks, double sparsity, int32_t budget);

/* Bytes of device workspace sba_pool_select needs for this shape (0 on bad
 * arguments).  The workspace holds the pooled Q and K block means, one record per
 * routing row for the selection (its window around the k-th score and its keep mask),
 * and room for the screened scores of rows the selection hands to its slower exact
 * routine (none on typical inputs). */
size_t sba_pool_select_workspace_size(int B, int H, int Npad, int D, int block);

/* Routing step: pool Q and K per block, score every key block for every query
 * block, keep the best keep(nB_b, sparsity) blocks per (b, h, I).  The page
 * "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), section "How SubBlock
 * sparse attention works": the pooling and scoring step that picks the key blocks
 * and hands their indices to the attention kernel, here with one sub-block per
 * block (the mean-pooled score in the file comment).
 *   q, k        bf16 [B, H, Npad, D] (read only)
 *   valid_len   int32 [B] device, or NULL
 *   sparsity    in [0, 1)
 *   kmax        row capacity of kv_idx; must be >= sba_keep_count(Npad/block, s)
 *   kv_idx      int32 [B, H, Npad/block, kmax] (written)
 *   kv_cnt      int32 [B, H, Npad/block] (written)
 *   workspace   device buffer of at least sba_pool_select_workspace_size bytes,
 *               16-byte aligned; contents on entry are ignored
 * The kept set equals the exact (real-number) top-k of the scores except where
 * two scores differ by less than the fp64 rounding of their evaluation. */
sba_status sba_pool_select(const void* q, const void* k, int B, int H, int Npad, int D,
                           const int32_t* valid_len, int block, double sparsity, int kmax,
                           int32_t* kv_idx, int32_t* kv_cnt,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace sba_pool_select_lse needs (0 on bad arguments or an
 * unsupported nsub).  It holds the pooled sub-block means (nsub per block). */
size_t sba_pool_select_lse_workspace_size(int B, int H, int Npad, int D, int block, int nsub);

/* Routing step with the sub-block log-sum-exp score, the SubBlock router's own
 * form (same page and section: every 64-token block split into n_q = n_k = 4
 * sub-blocks of 16 tokens; pooling and a log-sum-exp estimate each key block's
 * unnormalised softmax mass for each query block and head; the kept count is
 * subject to rounding to an 8-block budget):
 *   qbar[I,a] = mean of q over the valid tokens of sub-block a of block I,
 *               n[I,a] = their count (kbar, n[J,c] likewise)
 *   score[I][J] = log sum over non-empty (a, c) of
 *                 n[I,a] n[J,c] exp(qbar[I,a] . kbar[J,c] / sqrt(D))
 *   kept(I) = the keep(nB_b, s) blocks of highest score, keep rounded up to a
 *             multiple of `budget` and capped at nB_b; equal scores go to the
 *             lower index.
 * For tokens constant within each sub-block the score is exactly the log of
 * sum_{i in I, j in J} exp(q_i . k_j / sqrt(D)).
 *   nsub     sub-blocks per block; 4 is the one supported value (else UNSUPPORTED)
 *   budget   >= 1; 1 = no rounding
 *   kmax     must be >= the budget-rounded keep(Npad/block, s)
 *   other arguments as sba_pool_select; workspace of at least
 *   sba_pool_select_lse_workspace_size bytes.
 * The kept set equals the top-k of the fp64 evaluation of the score in the
 * stated order (dot products summed over d in order, then the max-shifted
 * log-sum-exp in (a, c) order); scores within a few fp64 rounding steps of each
 * other may be ordered either way. */
sba_status sba_pool_select_lse(const void* q, const void* k, int B, int H, int Npad, int D,
                               const int32_t* valid_len, int block, int nsub, double sparsity,
                               int budget, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                               void* workspace, size_t workspace_bytes, void* stream);

/* The producer step before the router, fused with its pooling: QK RMSNorm then 3D
 * RoPE, as the page "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), the
 * kernel layer, fuses them (head dimension 128, RoPE dimension 96, the normalised
 * value rounded to bf16 before the rotation).  Per (b, h, token n):
 *   y_d = bf16( x_d / sqrt(mean_e(x_e^2) + eps) * weight_d )
 *   channels [0, rope_dim) are three axes of da = rope_dim/3 channels for the
 *   token's position (t, y, x) = pos[b][n]; pair (2i, 2i+1) of axis a turns by
 *   theta = pos_a * rope_base^(-2i/da):
 *     out_2i = bf16(y_2i cos theta - y_2i+1 sin theta),
 *     out_2i+1 = bf16(y_2i sin theta + y_2i+1 cos theta);
 *   channels [rope_dim, D) pass through (out_d = y_d).
 * Arithmetic in fp32 (the sines and cosines of fp32 angles), rounded to bf16 at
 * the two points above, so results can differ from an exact evaluation by one bf16
 * unit in the last place.  Call once for Q and once for K.
 *   x         bf16 [B, H, Npad, D] (read); may equal `out` (in place)
 *   weight    bf16 [D], shared by all heads; 16-byte aligned
 *   pos       int32 [B, Npad, 3] device, (t, y, x) per token, each in [0, 65536)
 *             (outside that range the rotation angles are wrong, never a fault);
 *             every row read
 *   rope_dim  a multiple of 6 in [0, D] (0 = no rotation)
 *   rope_base > 0; eps >= 0 (1e-6 is usual)
 *   out       bf16 [B, H, Npad, D] (written, every row)
 *   means     fp64 [B, H, Npad/block, D] (written) or NULL: the block means of `out`
 *             over each sample's valid tokens, bit for bit what sba_block_means
 *             returns for `out`, ready for sba_pool_select_means.
 * Errors as the other calls; a bad rope_dim, base or eps is SBA_ERR_INVALID_ARG.
 * The page defines nothing beyond the fused norm + RoPE; pooling in the same pass
 * is this library's. */
sba_status sba_qk_norm_rope_pool(const void* x, const void* weight, const int32_t* pos, int B, int H,
                                 int Npad, int D, const int32_t* valid_len, int block, int rope_dim,
                                 double rope_base, float eps, void* out, double* means, void* stream);

/* sba_pool_select with the block means given (as written by sba_qk_norm_rope_pool
 * or sba_block_means) instead of pooled from Q and K: the same routing, without
 * the pass over Q and K.  qmean, kmean: fp64 [B, H, Npad/block, D] device, read
 * while the call runs, blocks past nB_b holding 0.  Other arguments as
 * sba_pool_select (same workspace size). */
sba_status sba_pool_select_means(const double* qmean, const double* kmean, int B, int H, int Npad,
                                 int D, const int32_t* valid_len, int block, double sparsity,
                                 int kmax, int32_t* kv_idx, int32_t* kv_cnt, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Block-sparse attention with compensation of the dropped blocks.  PISA, as the page
 * "Sol Video Inference Engine" (sjmshsh.github.io), section 4.2.2 (Sparse Attention),
 * describes it, computes the critical blocks exactly and compensates the others by a
 * first-order Taylor approximation.  Each dropped block J's exponentials are expanded
 * to first order about its mean key:
 *   e^{s q.k_j} ~ e^{s q.kbar_J} (1 + s q.(k_j - kbar_J))   for the valid tokens j of J
 * so that, with x_j = s q.k_j and xbar_J = s q.kbar_J,
 *   o_i = [sum_{j kept} e^{x_j} v_j
 *          + sum_{J dropped} e^{xbar_J} (c_J vbar_J + s q_i^T sum_{j in J} (k_j - kbar_J) v_j^T)]
 *         / [sum_{j kept} e^{x_j} + sum_{J dropped} c_J e^{xbar_J}]
 *   lse_i = log of the denominator
 * where "dropped" are the sample's blocks J < nB_b missing from the row's kept list,
 * kbar_J / vbar_J the means of the valid tokens of J and c_J their count.  Exact when
 * keys are constant within each dropped block; the error shrinks as the square of the
 * keys' spread about their block means.
 * The kernel evaluates the expansion token by token (the weight of token j of a
 * dropped block is e^{xbar_J} (1 + x_j - xbar_J), xbar_J being the mean of the block's
 * logits), so it walks every block of the sample: the cost is that of dense attention,
 * with one exponential per dropped block instead of one per token.
 * Arguments as sba_attention_paired (pair_order may be NULL for adjacent tiles); no
 * workspace. */
sba_status sba_attention_compensated(const void* q, const void* k, const void* v, void* o, float* lse,
                                     int B, int H, int Npad, int D, const int32_t* valid_len, int block,
                                     const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                     const int32_t* pair_order, float softmax_scale, void* stream);

/* Bytes of device workspace sba_attention_mean_compensated needs (0 on bad
 * arguments): the bf16 block means of K and V. */
size_t sba_mean_compensation_workspace_size(int B, int H, int Npad, int D, int block);

/* The cheaper, zeroth-order compensation: the expansion above without its moment
 * term, so each dropped block enters the softmax as one entry of logit
 * s q.kbar_J + log(c_J) carrying vbar_J:
 *   o_i = [sum_{j kept} e^{x_j} v_j + sum_{J dropped} c_J e^{xbar_J} vbar_J]
 *         / [sum_{j kept} e^{x_j} + sum_{J dropped} c_J e^{xbar_J}]
 * Its error shrinks only linearly with the keys' spread.  The means are formed in
 * fp64 and stored in bf16 (2^-9 relative), which moves each dropped block's logit by
 * at most s sum_d |q_d kbar_d| 2^-9.  Arguments as sba_attention_compensated, plus a
 * workspace of at least sba_mean_compensation_workspace_size bytes (16-byte aligned;
 * contents on entry ignored).  Cost: the kept blocks plus ceil(nB/64) further
 * 64-column steps per tile. */
sba_status sba_attention_mean_compensated(const void* q, const void* k, const void* v, void* o, float* lse,
                                          int B, int H, int Npad, int D, const int32_t* valid_len, int block,
                                          const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                          const int32_t* pair_order, float softmax_scale, void* workspace,
                                          size_t workspace_bytes, void* stream);

/* Block means of x as fp64 values [B, H, Npad/block, D] (inspection helper;
 * blocks past nB_b are written as 0).  `out` is device memory. */
sba_status sba_block_means(const void* x, int B, int H, int Npad, int D,
                           const int32_t* valid_len, int block, double* out, void* stream);

/* Exact attention over the routed key blocks: the block-sparse attention kernel of
 * the page "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), section "How
 * SubBlock sparse attention works", which takes the kept block indices and never
 * forms the full attention matrix; it computes the softmax over the kept tokens
 * exactly (the critical blocks of PISA, page "Sol Video Inference Engine",
 * sjmshsh.github.io, section 4.2.2, without its approximation of the rest).
 *   o      bf16 [B, H, Npad, D] (written; padding rows written as 0)
 *   lse    fp32 [B, H, Npad] natural-log log-sum-exp of the scaled logits, or
 *          NULL; padding rows and rows with no kept token get -inf
 *   softmax_scale  multiplier of q.k; <= 0 selects 1/sqrt(D)
 * A query row whose routing row is empty gets o = 0, lse = -inf. */
sba_status sba_attention(const void* q, const void* k, const void* v, void* o, float* lse,
                         int B, int H, int Npad, int D, const int32_t* valid_len, int block,
                         const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                         float softmax_scale, void* stream);

/* Pairing of query blocks into attention tiles (a performance choice only).
 * The attention kernel processes two 64-row query blocks per 128-row tile over
 * the union of their kept key blocks, so a key block kept by only one of the two
 * is masked work for the other.  This pass picks, per (b, h), pairs whose kept
 * lists overlap most: bitmaps of the kept sets, four rounds of mutual-best
 * matching among query blocks at most 64 positions apart, the rest paired in
 * order.  It never changes a result of sba_attention_paired, only its speed.
 *   kv_idx, kv_cnt, kmax, valid_len  a routing as produced by sba_pool_select
 *   pair_order  int32 [B, H, 2 * ceil(Npad/block / 2)] (written): tile t holds
 *               query blocks pair_order[b,h,2t] and [2t+1]; every query block of
 *               [0, Npad/block) appears once; a final unused slot is -1
 *   workspace   device buffer of sba_pair_workspace_size() bytes, 16-byte aligned */
size_t sba_pair_workspace_size(int B, int H, int Npad, int block);
sba_status sba_pair_query_blocks(const int32_t* kv_idx, const int32_t* kv_cnt, int B, int H,
                                 int Npad, int kmax, const int32_t* valid_len, int block,
                                 int32_t* pair_order, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* sba_attention with the tiles given by pair_order (see sba_pair_query_blocks);
 * results equal sba_attention's up to the order of floating-point accumulation.
 * pair_order must not be NULL; every query block must appear in it once. */
sba_status sba_attention_paired(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int Npad, int D, const int32_t* valid_len, int block,
                                const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                const int32_t* pair_order, float softmax_scale, void* stream);

/* sba_attention_paired with the output stored straight into sequence shards: the
 * exchange back from head sharding to sequence sharding of the page "MiniMax-H3 on
 * 8xH200 benchmark", which runs attention under SP/Ulysses.  The caller holds, for its
 * H heads h_first .. h_first + H - 1 of h_total, the whole sequence (q, k, v as in
 * sba_attention); the sequence is split into n_shards equal ranges of
 * shard_len = Npad / n_shards tokens, range s owned by shard s.
 *   o_shards:   host array of n_shards device pointers, bf16 [B][h_total][shard_len][D];
 *               token n of head h_first + h goes to shard n / shard_len, row n % shard_len.
 *               Other GPUs' memory (peer pointers, e.g. symmetric memory) is allowed: the
 *               stores cross NVLink once per element, in place of an all-to-all.
 *   lse_shards: NULL, or a host array of n_shards device pointers, fp32 [B][h_total][shard_len].
 * Only the caller's heads are written; rows past a sample's valid length get 0 / -inf.
 * pair_order may be NULL (adjacent pairs).  1 <= n_shards <= 8 and Npad % n_shards == 0,
 * else SBA_ERR_INVALID_ARG; a shard pointer not 16-byte (o) or 4-byte (lse) aligned gives
 * SBA_ERR_ALIGNMENT.  Stream-ordered; the shards' owners must synchronise with this
 * stream before reading. */
sba_status sba_attention_to_shards(const void* q, const void* k, const void* v, void* const* o_shards,
                                   float* const* lse_shards, int n_shards, int h_total, int h_first, int B,
                                   int H, int Npad, int D, const int32_t* valid_len, int block,
                                   const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                   const int32_t* pair_order, float softmax_scale, void* stream);

/* Token pruning by feature-norm saliency, the producer of a ragged, pruned sequence.
 * The page "Sol Video Inference Engine" (sjmshsh.github.io), LTX-2.3 appendix, stage
 * 2, keeps 50% of the video tokens by feat_norm saliency.  Per sample b, with L_b
 * valid tokens:
 *   saliency(n) = |x[b][n]|^2 = sum_c x[b][n][c]^2, summed in channel order in fp64
 *                 (every square of a bf16 value is exact)
 *   kept = the keep_tokens(L_b, keep_ratio) tokens of largest saliency, equal values
 *          going to the lower index, listed in their original (raster) order
 *   keep_tokens(L, r) = clamp(ceil(r * L - 1e-9), 1, L), fp64 (sba_keep_token_count).
 *   x            bf16 [B, N, C] token features, C a multiple of 8 (else UNSUPPORTED),
 *                16-byte aligned
 *   valid_len    int32 [B] device (1 <= valid_len[b] <= N), or NULL (all N valid)
 *   keep_ratio   in [0, 1]
 *   Npad_out     row length of idx; must be >= keep_tokens(N, keep_ratio)
 *   idx          int32 [B, Npad_out] (written): the kept token indices ascending,
 *                then -1
 *   valid_len_out int32 [B] (written): the kept counts (a valid_len for the pruned
 *                sequence)
 *   workspace    device buffer of sba_token_prune_workspace_size bytes, 16-byte
 *                aligned; on return its first B * N fp64 values are the saliencies
 *                (0 for padding tokens)
 * HBM-bound: x is read once. */
int32_t sba_keep_token_count(int32_t n_tokens, double keep_ratio);
size_t sba_token_prune_workspace_size(int B, int N);
sba_status sba_token_prune_select(const void* x, int B, int N, int C, const int32_t* valid_len,
                                  double keep_ratio, int Npad_out, int32_t* idx, int32_t* valid_len_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* The pruned sequence's rows: dst[b][h][p] = src[b][h][idx[b][p]] for
 * p < valid_len_out[b], zero rows for the rest of [0, Npad_out).  Companion of
 * sba_token_prune_select for the per-token tensors that follow the pruning (Q, K, V
 * [B, H, N, D], positions [B, N, 3] with H = 1, ...).
 *   src          [B, H, N] rows of row_bytes bytes (row_bytes a multiple of 4, else
 *                UNSUPPORTED); 16-byte aligned when row_bytes is a multiple of 16,
 *                else 4-byte aligned (dst likewise)
 *   idx, valid_len_out, Npad_out  as written by sba_token_prune_select (an index
 *                outside [0, N) raises SBA_ERR_DEVICE_FLAG and copies row 0)
 *   dst          [B, H, Npad_out] rows (written, every row)
 * HBM-bound row copy. */
sba_status sba_gather_tokens(const void* src, int B, int H, int N, int row_bytes, const int32_t* idx,
                             const int32_t* valid_len_out, int Npad_out, void* dst, void* stream);

/* Dense attention over all valid tokens of each sample (the sparsity = 0 case
 * without a routing), same layouts as sba_attention.  On the page "MiniMax-H3 on
 * 8xH200 benchmark", section "How SubBlock sparse attention works", sparsity is the
 * fraction of key blocks dropped, so sparsity 0 keeps every block: full attention,
 * which this call computes directly. */
sba_status sba_dense_attention(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int Npad, int D, const int32_t* valid_len,
                               float softmax_scale, void* stream);

/* Synchronises `stream`, returns and clears the device-side error word of the
 * current device: SBA_OK, SBA_ERR_TIMEOUT or SBA_ERR_DEVICE_FLAG (or
 * SBA_ERR_CUDA if the synchronisation itself failed). */
sba_status sba_get_device_status(void* stream);

/* Limit, in GPU clock cycles, of every wait inside the attention kernel
 * (default about 2^32 cycles, i.e. seconds).  A wait that reaches it gives up,
 * sets SBA_ERR_TIMEOUT and lets the kernel exit cleanly.  0 restores the
 * default.  Meant for tests of the timeout path. */
void sba_set_wait_limit(uint64_t cycles);

/* Which attention kernel sba_attention, sba_attention_paired and sba_dense_attention
 * run for D = 128 (the compensated path and D = 64 always use the first):
 *   SBA_ATTN_KERNEL_QUERY_PAIRS  one SM per tile of two query blocks, walking the union
 *                                of their kept lists (64 keys per step);
 *   SBA_ATTN_KERNEL_CTA_PAIR     a 2-SM cluster per tile of four adjacent query blocks
 *                                (tcgen05 MMAs of M = 256 across the pair, 128 keys per
 *                                step), walking the union of their four lists;
 *                                pair_order is not used;
 *   SBA_ATTN_KERNEL_AUTO         (default) the query pairs, the faster of the two on
 *                                every workload measured on B200.
 * Outputs agree up to floating-point accumulation order.  Process-wide; returns
 * SBA_ERR_INVALID_ARG for another value. */
#define SBA_ATTN_KERNEL_AUTO 0
#define SBA_ATTN_KERNEL_QUERY_PAIRS 1
#define SBA_ATTN_KERNEL_CTA_PAIR 2
sba_status sba_set_attention_kernel(int which);

/* Routing for callers that cannot allocate device memory.
 *
 * No counterpart on the pages: this is a library convenience.  Some callers may
 * not call cudaMalloc at all -- for instance code that runs inside a host
 * framework which owns every byte of device memory and hands the kernel no
 * workspace, or a latency-critical path where an allocation (which can
 * synchronise the device) is not allowed.  For them this entry point does what
 * sba_pool_select does, with the same arguments apart from the workspace, using
 * scratch that lives in a fixed array inside the library instead.
 *
 *   - The array holds sba_noalloc_scratch_bytes() bytes (16 MiB).  Every GPU that
 *     loads the library keeps that much device memory for it until the process
 *     exits.  A problem whose sba_pool_select_workspace_size() exceeds it is
 *     rejected with SBA_ERR_SCRATCH_TOO_SMALL before anything is launched.
 *   - Nothing is allocated or freed: the call makes no cudaMalloc/cudaFree and
 *     calls no allocating library routine.
 *   - The first call on a device looks up the array's device address (once per
 *     device, under a lock) with cudaGetSymbolAddress; make that first call
 *     before any stream capture.  The address is kept for the life of the process,
 *     so do not call this entry point on a device after cudaDeviceReset there.
 *   - All calls on a device share the one array and it keeps whatever the last
 *     call left in it.  That is harmless here, since every value a call reads
 *     from it was written earlier in the same call, so nothing has to start at
 *     zero.  But two calls whose kernels overlap on the GPU (different streams,
 *     no ordering between them) race on the array and may return wrong
 *     routings: serialise them. */
sba_status sba_pool_select_noalloc(const void* q, const void* k, int B, int H, int Npad, int D,
                                   const int32_t* valid_len, int block, double sparsity, int kmax,
                                   int32_t* kv_idx, int32_t* kv_cnt, void* stream);

/* Size in bytes of the fixed scratch array sba_pool_select_noalloc uses. */
size_t sba_noalloc_scratch_bytes(void);

/* Static description of a status code. */
const char* sba_strerror(sba_status status);

#ifdef __cplusplus
}
#endif

#endif /* SBA_H_ */

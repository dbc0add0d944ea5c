// attention.cuh -- exact softmax attention over routed 64-token key blocks, sm_100a.
//
// The computation is the block-sparse stage of the SubBlock router on the page
// "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), section "How SubBlock
// sparse attention works": each query block attends, exactly, to the tokens of
// its kept key blocks only, and the full attention matrix is never formed.
//
// Tiling.  A CTA owns two 64-row query blocks of one (b, h) -- by default the
// adjacent I0 = 2p, I1 = 2p + 1, or the pair a routing-side pass chose for overlap
// of their kept lists -- as a 128-row Q tile, the full-rate M of a single-CTA
// tcgen05.mma.
// It walks the ascending union of the two kept lists; a key block kept by only
// one of the two is masked to -inf for the other half's rows.
//
// Warp roles (192 threads; two CTAs share an SM, so one CTA's MMAs run while the
// other's softmax warps work):
//   warps 0-3  softmax + epilogue; thread t owns query row t = TMEM lane t.  Warps
//              0-1 serve query block I0, warps 2-3 query block I1, so "this key
//              block is kept" is uniform over a warp and unkept blocks cost no
//              exponentials (the warp writes P = 0)
//   warp 4     builds the union list, then issues TMA loads: Q once, then K and V
//              per key block in two rings; K(j) is freed when S(j) is done and V(j)
//              when PV(j) is, and K is issued one block ahead of V
//   warp 5     allocates TMEM (256 columns) and issues the MMAs (one elected lane)
// Per key block j:  S_j = Q K_j^T  (M=128, N=64, K=D) into TMEM buffer j%2;
//                   softmax reads S_j and writes P_j (bf16) back over it;
//                   O += P_j V_j (M=128, N=D, K=64), P read from TMEM.
// The MMA warp issues S_{j+1} before PV_j so the tensor core works on the next
// scores while the softmax warps exponentiate.  The running max is only moved
// when it grows by more than 8 (log2 units); O is then rescaled in TMEM.
//
// Every wait is bounded: on expiry the CTA records SBA_ERR_TIMEOUT, unwinds all
// roles, drains its own TMA loads and MMAs and frees its TMEM.
//
// MODE selects what the dropped key blocks contribute (the compensation of the
// dropped blocks; page "Sol Video Inference Engine", section 4.2.2: PISA computes the
// critical blocks exactly and compensates the others by a first-order Taylor
// approximation):
//   kPlain      nothing: the kept blocks only.
//   kMeanComp   each dropped block as one softmax entry: after the union walk, the
//               tile walks the rows of kbar / vbar (the bf16 block means,
//               [BH][nBpad][D]) as further 64-column steps, column c of step b
//               standing for block J = 64 b + c with logit s q.kbar_J + log(c_J); a
//               column is masked for a half whose query block keeps J, and past the
//               sample's blocks.  The online softmax merges the two parts exactly as
//               it merges key blocks.
//   kFirstOrder the first-order expansion of every dropped block's exponentials about
//               its mean key: the tile walks all blocks of the sample; a block the
//               half keeps gets weights e^{x_j}, a dropped one the tangent line
//               e^{xbar} (1 + x_j - xbar), where x_j = s q.k_j and xbar = s q.kbar_J is
//               the mean of the block's logits over its valid tokens, and adds
//               c_J e^{xbar} to the normaliser.  Summed over the block this is
//               e^{xbar} (c_J vbar_J + s q^T sum_j (k_j - kbar_J) v_j^T): the
//               zeroth- and first-order terms, with no D x D moment ever formed.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace sba {

enum AttnMode : int { kPlain = 0, kMeanComp = 1, kFirstOrder = 2 };

constexpr int kMaxBlocks = 4096;  // SBA_MAX_NPAD / 64
constexpr int kMaxShards = 8;

struct AttnParams {
    __nv_bfloat16* o;
    float* lse;
    const int32_t* valid_len;
    const int32_t* kv_idx;
    const int32_t* kv_cnt;
    const int32_t* pair_order;  // [B*H][2*ceil(nQ/2)] query blocks per tile, -1 = none; NULL = adjacent
    int H;
    int Npad;
    int kmax;
    int dense;
    float scale_log2;  // softmax scale * log2(e)
    unsigned long long wait_limit;
    // Output to sequence shards: the Ulysses exchange back to sequence sharding, done by
    // the epilogue's stores.  With n_shards > 0, token n of this call's head h goes to
    // shard s = n / shard_len, row (b * h_total + h_first + h) * shard_len + n - s * shard_len
    // of o_shard[s] / lse_shard[s] ([B][h_total][shard_len][D] and [.][.][shard_len]);
    // the shards may be other GPUs' memory (peer pointers), so each output element
    // crosses NVLink once, in place of an all-to-all and its copy.
    int n_shards = 0;
    int shard_len = 0;
    int h_total = 0;
    int h_first = 0;
    __nv_bfloat16* o_shard[kMaxShards] = {};
    float* lse_shard[kMaxShards] = {};
};

template <int D, int NS>
struct AttnSmem {
    static constexpr int kQBytes = 128 * D * 2;
    static constexpr int kKVBytes = 64 * D * 2;
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQBytes;
    static constexpr int kV = kK + NS * kKVBytes;
    static constexpr int kBars = kV + NS * kKVBytes;
    // barriers: q_full, k_full[NS], v_full[NS], k_empty[NS], v_empty[NS], s_full[2],
    //           p_full[2], pv_done[2], drain
    static constexpr int kNumBars = 1 + 4 * NS + 7;
    static constexpr int kCtl = kBars + kNumBars * 8;      // tmem base, abort, n_union, pad
    static constexpr int kBitmap = kCtl + 16;              // uint32 [2][kMaxBlocks/32]
    static constexpr int kList = kBitmap + 2 * (kMaxBlocks / 32) * 4;  // uint16 [kMaxBlocks]
    static constexpr int kTotal = kList + kMaxBlocks * 2;
    static constexpr int kAlloc = kTotal + 1024;            // slack for 1024-byte alignment
};

// Drains after an abort wait for work that always completes on its own (this CTA's
// TMA copies and MMAs), so their limit is fixed and generous, independent of the
// wait limit the caller set.
constexpr uint64_t kDrainLimit = 1ull << 32;

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t limit = kDrainLimit) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if ((uint64_t)(clock64() - t0) > limit) return false;
    }
    return true;
}

// The body of both kernels below; the tensor maps are the kernels' own __grid_constant__
// parameters, passed by address (the plain kernel keeps its three-map signature).
template <int D, int NS, int MODE>
__device__ __forceinline__ void attn_body(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                          const CUtensorMap& tmKb, const CUtensorMap& tmVb, const AttnParams& p) {
    using SM = AttnSmem<D, NS>;
    constexpr int NCH = D / 64;                 // 128-byte column chunks per row
    constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
    constexpr uint32_t kTmemCols = 256;         // S[2] at 0 / 64, O at 128

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sQ = smem_u32(sm + SM::kQ);
    const uint32_t sK = smem_u32(sm + SM::kK);
    const uint32_t sV = smem_u32(sm + SM::kV);
    const uint32_t bars = smem_u32(sm + SM::kBars);
    const uint32_t bar_q = bars;
    auto bar_kf = [&](int s) { return bars + 8u * (1 + s); };
    auto bar_vf = [&](int s) { return bars + 8u * (1 + NS + s); };
    auto bar_ke = [&](int s) { return bars + 8u * (1 + 2 * NS + s); };
    auto bar_ve = [&](int s) { return bars + 8u * (1 + 3 * NS + s); };
    auto bar_sf = [&](int s) { return bars + 8u * (1 + 4 * NS + s); };
    auto bar_pf = [&](int s) { return bars + 8u * (3 + 4 * NS + s); };
    auto bar_pv = [&](int s) { return bars + 8u * (5 + 4 * NS + s); };
    const uint32_t bar_drain = bars + 8u * (7 + 4 * NS);
    uint32_t* ctl = reinterpret_cast<uint32_t*>(sm + SM::kCtl);
    volatile uint32_t* abort_flag = ctl + 1;
    uint32_t* bm = reinterpret_cast<uint32_t*>(sm + SM::kBitmap);
    uint16_t* ulist = reinterpret_cast<uint16_t*>(sm + SM::kList);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int nQ = p.Npad / 64;
    // the tile's two query blocks; a slot outside [0, nQ) is empty
    int qb[2] = {2 * (int)blockIdx.x, 2 * (int)blockIdx.x + 1};
    if (p.pair_order) {
        const int32_t* po = p.pair_order + (size_t)bh * (2 * gridDim.x) + 2 * blockIdx.x;
        qb[0] = po[0];
        qb[1] = po[1];
    }
    const int L = p.valid_len ? p.valid_len[b] : p.Npad;
    const int nB = (L + 63) / 64;
    const int W = (nB + 31) / 32;

    if (tid == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar_kf(s), 1);
            mbar_init(bar_vf(s), 1);
            mbar_init(bar_ke(s), 1);
            mbar_init(bar_ve(s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_sf(s), 1);
            mbar_init(bar_pf(s), 128);
            mbar_init(bar_pv(s), 1);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(smem_u32(ctl), kTmemCols);
    if (warp == 4) {
        // union of the two kept lists as a bitmap per half, then an ascending list
        for (int w = lane; w < W; w += 32) {
            uint32_t full = 0;
            if (p.dense) full = (w * 32 + 32 <= nB) ? 0xffffffffu : ((1u << (nB - w * 32)) - 1u);
            bm[w] = (p.dense && qb[0] >= 0 && qb[0] < nB) ? full : 0u;
            bm[kMaxBlocks / 32 + w] = (p.dense && qb[1] >= 0 && qb[1] < nB) ? full : 0u;
        }
        __syncwarp();
        if (!p.dense) {
            for (int half = 0; half < 2; ++half) {
                const int I = qb[half];
                if (I < 0 || I >= nQ) continue;
                const size_t row = (size_t)bh * nQ + I;
                int cnt = p.kv_cnt[row];
                if (cnt < 0 || cnt > p.kmax) {
                    raise_device_error(kErrBadRouting);
                    cnt = cnt < 0 ? 0 : p.kmax;
                }
                const int32_t* lst = p.kv_idx + row * p.kmax;
                for (int t = lane; t < cnt; t += 32) {
                    const int J = lst[t];
                    if (J >= 0 && J < nB)
                        atomicOr(&bm[half * (kMaxBlocks / 32) + (J >> 5)], 1u << (J & 31));
                    else
                        raise_device_error(kErrBadRouting);
                }
            }
        }
        __syncwarp();
        int base = 0;
        for (int w0 = 0; w0 < W; w0 += 32) {
            const int w = w0 + lane;
            uint32_t u = w < W ? (bm[w] | bm[kMaxBlocks / 32 + w]) : 0u;
            if (MODE == kFirstOrder) {
                // every block of the sample: kept ones exactly, dropped ones by the expansion
                const bool any = (qb[0] >= 0 && qb[0] < nB) || (qb[1] >= 0 && qb[1] < nB);
                u = (w < W && any) ? ((w * 32 + 32 <= nB) ? 0xffffffffu : ((1u << (nB - w * 32)) - 1u)) : 0u;
            }
            const int c = __popc(u);
            int incl = c;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            int pos = base + incl - c;
            uint32_t bits = u;
            while (bits) {
                const int bit = __ffs(bits) - 1;
                bits &= bits - 1;
                ulist[pos++] = static_cast<uint16_t>(w * 32 + bit);
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) ctl[2] = static_cast<uint32_t>(base);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl[0];
    const int n = static_cast<int>(ctl[2]);
    // with compensation, the block-mean steps follow the union (none for a tile whose
    // two slots both lie past the sample)
    const bool any_slot = (qb[0] >= 0 && qb[0] < nB) || (qb[1] >= 0 && qb[1] < nB);
    const int n_all = MODE == kMeanComp && any_slot ? n + (nB + 63) / 64 : n;
    const uint64_t lim = p.wait_limit;
    int issued_k = 0, issued_v = 0;  // K / V blocks whose loads the producer has issued

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n_all > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            // Q: one 64-row box per query block of the tile (an empty slot's rows stay
            // unloaded; its rows keep nothing, so they only ever multiply P = 0)
            const bool q1 = qb[1] >= 0 && qb[1] < nQ;
            mbar_arrive_expect_tx(bar_q, (q1 ? 2 : 1) * (64 * D * 2));
            for (int h2 = 0; h2 < (q1 ? 2 : 1); ++h2)
                for (int c = 0; c < NCH; ++c)
                    tma_load_3d(sQ + c * (128 * 128) + h2 * (64 * 128), &tmQ, bar_q, c * 64, qb[h2] * 64, bh);
            // K runs one block ahead of V: K(j) is released as soon as S(j) is done,
            // V(j) only after PV(j).  Issue order K0, K1, V0, K2, V1, ...
            for (int j = 0; j <= n_all; ++j) {
                if (j < n_all) {
                    const int st = j % NS;
                    if (j >= NS && !wait_bounded(bar_ke(st), ((j / NS) - 1) & 1, abort_flag, lim)) break;
                    const bool mean_step = MODE == kMeanComp && j >= n;
                    const int row = mean_step ? (j - n) * 64 : ulist[j] * 64;
                    mbar_arrive_expect_tx(bar_kf(st), SM::kKVBytes);
                    for (int c = 0; c < NCH; ++c)
                        tma_load_3d(sK + st * SM::kKVBytes + c * (64 * 128), mean_step ? &tmKb : &tmK, bar_kf(st),
                                    c * 64, row, bh);
                    issued_k = j + 1;
                }
                if (j >= 1) {
                    const int jv = j - 1, st = jv % NS;
                    if (jv >= NS && !wait_bounded(bar_ve(st), ((jv / NS) - 1) & 1, abort_flag, lim)) break;
                    const bool mean_step = MODE == kMeanComp && jv >= n;
                    const int row = mean_step ? (jv - n) * 64 : ulist[jv] * 64;
                    mbar_arrive_expect_tx(bar_vf(st), SM::kKVBytes);
                    for (int c = 0; c < NCH; ++c)
                        tma_load_3d(sV + st * SM::kKVBytes + c * (64 * 128), mean_step ? &tmVb : &tmV, bar_vf(st),
                                    c * 64, row, bh);
                    issued_v = jv + 1;
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        // The tensor pipe queues only a few MMAs, so this thread issues without stalls:
        // descriptors are precomputed (a shared-memory descriptor steps by adding
        // (byte offset >> 4) to its start-address field), the barriers of the next
        // group are tested (non-blocking) before the current group issues and read
        // after it, and a pending one is waited for by polling.
        if (lane == 0 && n_all > 0) {
            bool ok = poll_bounded(bar_q, 0, abort_flag, lim);
            tc_fence_after();
            uint64_t dq[D / 16], dk[D / 16], dv[4];
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                dq[kk] = smem_desc_sw128(sQ + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
                dk[kk] = smem_desc_sw128(sK + (kk / 4) * (64 * 128) + (kk % 4) * 32, 16, 1024);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) dv[kk] = smem_desc_sw128(sV + kk * (16 * 128), 64 * 128, 1024);
            constexpr uint64_t kStep = SM::kKVBytes >> 4;
            bool k_pre = false;  // K(j) seen ready during the previous PV group
            for (int j = 0; ok && j <= n_all; ++j) {
                bool p_ok = false, v_ok = false;
                const int jj = j - 1, sv = jj >= 0 ? jj % NS : 0;
                if (j < n_all) {
                    const int st = j % NS;
                    if (!k_pre && !poll_bounded(bar_kf(st), (j / NS) & 1, abort_flag, lim)) { ok = false; break; }
                    tc_fence_after();
                    if (jj >= 0) {
                        p_ok = mbar_test_wait(bar_pf(jj & 1), (jj >> 1) & 1);
                        v_ok = mbar_test_wait(bar_vf(sv), (jj / NS) & 1);
                    }
                    const uint32_t dS = tmem + (j & 1) * 64;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_bf16_ss(dS, dq[kk], dk[kk] + st * kStep, kIdescS, kk > 0 ? 1u : 0u);
                    mma_commit(bar_sf(j & 1));
                    mma_commit(bar_ke(st));
                }
                k_pre = false;
                if (jj >= 0) {
                    if (!p_ok && !poll_bounded(bar_pf(jj & 1), (jj >> 1) & 1, abort_flag, lim)) { ok = false; break; }
                    if (!v_ok && !poll_bounded(bar_vf(sv), (jj / NS) & 1, abort_flag, lim)) { ok = false; break; }
                    tc_fence_after();
                    const int jn = j + 1;
                    if (jn < n_all) k_pre = mbar_test_wait(bar_kf(jn % NS), (jn / NS) & 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tmem + 128, tmem + (jj & 1) * 64 + kk * 8, dv[kk] + sv * kStep, kIdescPV,
                                    (jj > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar_pv(jj & 1));
                    mma_commit(bar_ve(sv));
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int r = tid;                      // query row of the tile = TMEM lane
        const int half = r >> 6;
        const int tok = qb[half] * 64 + (r & 63);
        const uint32_t* bmh = bm + half * (kMaxBlocks / 32);
        const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sc = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        const bool half_ok = qb[half] >= 0 && qb[half] < nB;
        for (int j = 0; j < n_all; ++j) {
            bool kept;                 // exponential weights for this half (uniform over the warp)
            bool tangent = false;      // first-order weights of a dropped block (kFirstOrder)
            int ncol;
            uint64_t cmask = ~0ull;    // mean steps: the columns that carry weight for this half
            float off_full = 0.f, off_last = 0.f;
            int last_col = -1;
            if (MODE == kMeanComp && j >= n) {
                // columns 0..63 stand for blocks J = 64 pb + c: the half's dropped blocks
                // of the sample, each with logit offset log2(c_J) (folded in as / sc)
                const int pb = j - n;
                const uint64_t kb = (uint64_t)bmh[2 * pb] | ((uint64_t)bmh[2 * pb + 1] << 32);
                const int nv = nB - 64 * pb;
                const uint64_t inb = nv >= 64 ? ~0ull : ((1ull << nv) - 1ull);
                cmask = half_ok ? (~kb & inb) : 0ull;
                kept = cmask != 0ull;
                ncol = 64;
                off_full = 6.0f / sc;  // log2(64)
                if (nv <= 64) {
                    last_col = nv - 1;
                    off_last = log2f((float)(L - 64 * (nB - 1))) / sc;
                }
            } else {
                const int J = ulist[j];
                kept = (bmh[J >> 5] >> (J & 31)) & 1u;
                tangent = MODE == kFirstOrder && !kept && half_ok;
                ncol = (kept || tangent) ? L - J * 64 : 0;
                ncol = ncol > 64 ? 64 : ncol;
            }
            if (!warp_wait_bounded(bar_sf(j & 1), (j >> 1) & 1, abort_flag, lim)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sbuf = tl + (j & 1) * 64;
            if (!kept && !tangent) {
                // the other query block of the tile keeps this key block: P = 0 for these rows
                uint32_t z[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) z[i] = 0u;
                tmem_st32(sbuf, z);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_pf(j & 1));
                continue;
            }
            float x[64];
            {
                uint32_t a[32], c[32];
                tmem_ld32(sbuf, a);
                tmem_ld32(sbuf + 32, c);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = __uint_as_float(a[i]);
                    x[32 + i] = __uint_as_float(c[i]);
                }
            }
            float m_step;              // this step's largest exponent (log2 units)
            float xbar = 0.f;          // tangent: mean logit of the block's valid tokens (q.k units)
            if (MODE == kFirstOrder && tangent) {
                uint64_t s2 = pack2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    s2 = fadd2(s2, pack2(2 * i < ncol ? x[2 * i] : 0.f, 2 * i + 1 < ncol ? x[2 * i + 1] : 0.f));
                float s0, s1;
                unpack2(s2, s0, s1);
                xbar = (s0 + s1) / (float)ncol;
                m_step = xbar * sc;
            } else {
                if (ncol < 64) {  // ragged tail block of the sample
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] = i < ncol ? x[i] : -INFINITY;
                }
                if constexpr (MODE == kMeanComp) {
                    if (j >= n) {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            x[i] = ((cmask >> i) & 1ull) ? x[i] + (i == last_col ? off_last : off_full) : -INFINITY;
                    }
                }
                float mx0 = x[0], mx1 = x[1];
#pragma unroll
                for (int i = 2; i < 62; i += 4) {
                    mx0 = fmax3(mx0, x[i], x[i + 1]);
                    mx1 = fmax3(mx1, x[i + 2], x[i + 3]);
                }
                mx0 = fmax3(mx0, x[62], x[63]);
                m_step = fmaxf(mx0, mx1) * sc;
            }
            const float m_new = fmaxf(m, m_step);
            const bool grow = m_new > m + 8.f;
            if (j > 0 && __any_sync(0xffffffffu, grow)) {
                // O holds sum P V with the old running max: move the max, rescale O and l.
                if (!warp_wait_bounded(bar_pv((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m - m_new);
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(tl + 128 + ch * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tl + 128 + ch * 32, o);
                }
                l *= alpha;
                m = m_new;
            } else if (grow || j == 0) {
                m = m_new;
            }
            uint32_t pk[32];
            if (MODE == kFirstOrder && tangent) {
                // w_j = e^{xbar} (1 + s (q.k_j - q.kbar)), relative to the running max:
                // e = 2^(xbar sc - m), slope e ln2 sc; the normaliser gains c_J e
                const float e = ex2_approx(m_step - m);
                const float slope = e * (sc * 0.69314718055994530942f);
                const uint64_t nx2 = pack2(-xbar, -xbar), sl2 = pack2(slope, slope), e2 = pack2(e, e);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float w0, w1;
                    unpack2(ffma2(fadd2(pack2(x[2 * i], x[2 * i + 1]), nx2), sl2, e2), w0, w1);
                    w0 = 2 * i < ncol ? w0 : 0.f;
                    w1 = 2 * i + 1 < ncol ? w1 : 0.f;
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(w0, w1);
                    pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                }
                l += (float)ncol * e;
            } else {
                // p = 2^(s * scale * log2e - m), packed to bf16 pairs over the S columns just read
                const float nm = (m == -INFINITY) ? 0.f : -m;
                const uint64_t sc2 = pack2(sc, sc), nm2 = pack2(nm, nm);
                uint64_t acc0 = pack2(0.f, 0.f), acc1 = acc0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float y0, y1;
                    unpack2(ffma2(pack2(x[2 * i], x[2 * i + 1]), sc2, nm2), y0, y1);
                    const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
                    if (i & 1) acc1 = fadd2(acc1, pack2(p0, p1));
                    else acc0 = fadd2(acc0, pack2(p0, p1));
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                }
                float a0, a1, b0, b1;
                unpack2(acc0, a0, a1);
                unpack2(acc1, b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            tmem_st32(sbuf, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_pf(j & 1));
        }

        // ------------------------------------------------------------ epilogue
        if (ok && n_all > 0) ok = warp_wait_bounded(bar_pv((n_all - 1) & 1), ((n_all - 1) >> 1) & 1, abort_flag, lim);
        tc_fence_after();
        const bool in_range = qb[half] >= 0 && qb[half] < nQ;
        const bool valid = tok < L && l > 0.f;
        __nv_bfloat16* orow;
        float* lrow;
        if (p.n_shards > 0) {
            int sh = tok / p.shard_len;
            sh = sh < p.n_shards ? sh : p.n_shards - 1;  // rows outside the range are not stored
            const size_t row = (size_t)(b * p.h_total + p.h_first + h) * p.shard_len + (tok - sh * p.shard_len);
            orow = p.o_shard[sh] + row * D;
            lrow = p.lse_shard[sh] ? p.lse_shard[sh] + row : nullptr;
        } else {
            orow = p.o + ((size_t)bh * p.Npad + tok) * D;
            lrow = p.lse ? p.lse + (size_t)bh * p.Npad + tok : nullptr;
        }
        if (ok) {
            const float inv_l = valid ? 1.f / l : 0.f;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t o[32];
                if (n_all > 0) {
                    tmem_ld32(tl + 128 + ch * 32, o);
                    tmem_wait_ld();
                }
                if (in_range) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float o0 = (n_all > 0 && valid) ? __uint_as_float(o[2 * i]) * inv_l : 0.f;
                        const float o1 = (n_all > 0 && valid) ? __uint_as_float(o[2 * i + 1]) * inv_l : 0.f;
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(o0, o1);
                        pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            if (in_range && lrow) *lrow = valid ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // An aborted CTA still lets its own TMA copies land and its MMAs finish
        // before it frees TMEM and exits.
        if (warp == 4 && lane == 0 && n_all > 0) {
            wait_drain(bar_q, 0);
            for (int j = issued_k > NS ? issued_k - NS : 0; j < issued_k; ++j)
                wait_drain(bar_kf(j % NS), (j / NS) & 1);
            for (int j = issued_v > NS ? issued_v - NS : 0; j < issued_v; ++j)
                wait_drain(bar_vf(j % NS), (j / NS) & 1);
        }
        if (warp == 5 && lane == 0) {
            mma_commit(bar_drain);
            wait_drain(bar_drain, 0);
        }
        __syncthreads();
    }
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D, int NS>
__global__ void __launch_bounds__(192, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    attn_body<D, NS, kPlain>(tmQ, tmK, tmV, tmK, tmV, p);
}

// Mean-key compensation of the dropped blocks: kbar / vbar maps over [BH][nBpad][D].
template <int D, int NS>
__global__ void __launch_bounds__(192, 2)
    attn_comp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                     const __grid_constant__ CUtensorMap tmVb, const AttnParams p) {
    attn_body<D, NS, kMeanComp>(tmQ, tmK, tmV, tmKb, tmVb, p);
}

// First-order compensation of the dropped blocks: every block of the sample is walked.
template <int D, int NS>
__global__ void __launch_bounds__(192, 2)
    attn_first_order_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    attn_body<D, NS, kFirstOrder>(tmQ, tmK, tmV, tmK, tmV, p);
}

}  // namespace sba

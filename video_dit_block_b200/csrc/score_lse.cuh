// score_lse.cuh -- screened block scores of the sub-block log-sum-exp router, as one
// persistent, pipelined kernel on the tensor cores.
//
// Per (b, h) the sub-block logits x[r][s] = qbar_r . kbar_s / sqrt(D) (r, s index
// 16-token sub-blocks, 4 per 64-token block) form an nP x nP matrix, nP = 4 nB.  The
// block score of query block I and key block J is
//     log sum_{a,c} n_{4I+a} n_{4J+c} exp(x[4I+a][4J+c])
// over the non-empty sub-blocks (n = valid tokens).  Each fp64 sub-block mean is
// split into bf16 hi + lo, and qh.kl + ql.kh + qh.kh (cross terms first, so that
// their small partial sums add little error) is accumulated in fp32 by tcgen05.mma;
// the top-k kernel states the error bound and re-scores its band in fp64.
//
// Work item = (bh, 128-row tile of query sub-blocks = 32 query blocks); the CTA keeps
// that tile's qh/ql in shared memory and walks every 128-row tile of key sub-blocks
// (32 key blocks) through a 2-stage ring.  Each key tile gives a 128 x 128 fp32
// accumulator in one of 4 TMEM buffers (all 512 columns), so the MMAs of later tiles
// run while the epilogue folds earlier ones into block scores.
//
// Warps: 0 = TMA producer (lane 0), 1 = TMEM allocation and MMA issue (lane 0),
// 2..9 = epilogue (warp w reads TMEM lanes 32 (w % 4) .., half of each tile's
// columns; lane = sub-row, the 4 lanes of one query block combine through
// shuffles).  Where a tile has only full key sub-blocks and its logits stay within
// +-100 in log2 units, the sum needs no max shift: z = w * sum 2^y directly, and a
// transposing reduction leaves each lane two block sums to take the log of.  Every
// wait is bounded; an aborted CTA lets its own copies land and MMAs finish before
// it frees TMEM.
#pragma once
#include <cstdint>
#include <cuda.h>

#include "common.cuh"

namespace sba {

template <int D>
struct LseSmem {
    static constexpr int kTile = 128 * D * 2;        // one 128-row bf16 operand tile
    static constexpr int kStages = 2;
    static constexpr int kQh = 0;
    static constexpr int kQl = kTile;
    static constexpr int kK = 2 * kTile;              // stage s: hi at kK + 2 s kTile, lo after it
    static constexpr int kBars = kK + kStages * 2 * kTile;
    // a_full, a_empty, b_full[2], b_empty[2], acc_full[4], acc_empty[4], drain
    static constexpr int kNumBars = 15;
    static constexpr int kCtl = kBars + kNumBars * 8;  // tmem base, abort flag
    static constexpr int kTotal = kCtl + 16;
    // at least 116 KB so that two CTAs never share an SM (each holds all of TMEM)
    static constexpr int kAlloc = kTotal + 1024 > 116 * 1024 ? kTotal + 1024 : 116 * 1024;
};

constexpr int kLseAccBufs = 4;

// maps: bf16 [BH][nP][D] as 3-D (D, nP, BH), box 64 columns x 128 rows.
// scores: fp32 [BH][nB][ld] (nB = nP / 4 rows); columns past the sample's blocks hold
// unused values.
template <int D>
__global__ void __launch_bounds__(320, 1)
    score_lse_kernel(const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQl,
                     const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
                     float* __restrict__ scores, int nB, int ld, const int32_t* __restrict__ valid_len, int H,
                     int Npad, int BH, unsigned long long wait_limit) {
    using SM = LseSmem<D>;
    constexpr int NCH = D / 64;
    constexpr int SUB = 16;                 // tokens per sub-block
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, 0, 0);
    constexpr float kInv = D == 128 ? 0.0883883476483184405f : 0.125f;  // fp32(1 / sqrt(D))
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kScale = kInv * kLog2e;  // logits in log2 units
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sQh = smem_u32(sm + SM::kQh), sQl = smem_u32(sm + SM::kQl);
    const uint32_t sK = smem_u32(sm + SM::kK);
    const uint32_t bars = smem_u32(sm + SM::kBars);
    const uint32_t bar_a_full = bars, bar_a_empty = bars + 8;
    auto bar_b_full = [&](int s) { return bars + 16u + 8u * s; };
    auto bar_b_empty = [&](int s) { return bars + 32u + 8u * s; };
    auto bar_acc_full = [&](int t) { return bars + 48u + 8u * t; };
    auto bar_acc_empty = [&](int t) { return bars + 80u + 8u * t; };
    const uint32_t bar_drain = bars + 112u;
    uint32_t* ctl = reinterpret_cast<uint32_t*>(sm + SM::kCtl);
    volatile uint32_t* abort_flag = ctl + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nP = nB * 4;
    const int MT = (nP + 127) / 128;        // 128-row tiles per (b, h), both operands
    const long long items = (long long)BH * MT;
    const uint64_t lim = wait_limit;

    if (tid == 0) {
        mbar_init(bar_a_full, 1);
        mbar_init(bar_a_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_b_full(s), 1);
            mbar_init(bar_b_empty(s), 1);
        }
        for (int t = 0; t < kLseAccBufs; ++t) {
            mbar_init(bar_acc_full(t), 1);
            mbar_init(bar_acc_empty(t), 8);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(ctl), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl[0];

    int a_issued = 0, b_issued = 0;  // producer: A tiles and B tiles whose loads were issued
    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        bool ok = true;
        for (long long it = blockIdx.x; it < items && ok; it += gridDim.x) {
            const int bh = (int)(it / MT), m0 = (int)(it % MT) * 128;
            if (a_issued > 0 && !wait_bounded(bar_a_empty, (a_issued - 1) & 1, abort_flag, lim)) break;
            mbar_arrive_expect_tx(bar_a_full, 2 * SM::kTile);
            for (int c = 0; c < NCH; ++c) {
                tma_load_3d(sQh + c * (128 * 128), &tmQh, bar_a_full, c * 64, m0, bh);
                tma_load_3d(sQl + c * (128 * 128), &tmQl, bar_a_full, c * 64, m0, bh);
            }
            ++a_issued;
            for (int nt = 0; nt < MT; ++nt) {
                const int s = b_issued & 1, u = b_issued >> 1;
                if (u > 0 && !wait_bounded(bar_b_empty(s), (u - 1) & 1, abort_flag, lim)) {
                    ok = false;
                    break;
                }
                const uint32_t kh = sK + s * 2 * SM::kTile, kl = kh + SM::kTile;
                mbar_arrive_expect_tx(bar_b_full(s), 2 * SM::kTile);
                for (int c = 0; c < NCH; ++c) {
                    tma_load_3d(kh + c * (128 * 128), &tmKh, bar_b_full(s), c * 64, nt * 128, bh);
                    tma_load_3d(kl + c * (128 * 128), &tmKl, bar_b_full(s), c * 64, nt * 128, bh);
                }
                ++b_issued;
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issue
        int a_used = 0, b_used = 0, tiles = 0;
        bool ok = true;
        for (long long it = blockIdx.x; it < items && ok; it += gridDim.x) {
            if (!wait_bounded(bar_a_full, a_used & 1, abort_flag, lim)) break;
            ++a_used;
            tc_fence_after();
            for (int nt = 0; nt < MT; ++nt) {
                const int s = b_used & 1, t = tiles % kLseAccBufs, v = tiles / kLseAccBufs;
                if (!wait_bounded(bar_b_full(s), (b_used >> 1) & 1, abort_flag, lim) ||
                    (v > 0 && !wait_bounded(bar_acc_empty(t), (v - 1) & 1, abort_flag, lim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t kh = sK + s * 2 * SM::kTile, kl = kh + SM::kTile;
                const uint32_t acc = tmem + (uint32_t)(t * 128);
                // qh.kl, ql.kh, then qh.kh
                const uint32_t As[3] = {sQh, sQl, sQh};
                const uint32_t Bs[3] = {kl, kh, kh};
#pragma unroll
                for (int term = 0; term < 3; ++term) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * (128 * 128) + (kk % 4) * 32;
                        mma_bf16_ss(acc, smem_desc_sw128(As[term] + off, 16, 1024),
                                    smem_desc_sw128(Bs[term] + off, 16, 1024), kIdesc,
                                    (term > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bar_b_empty(s));
                mma_commit(bar_acc_full(t));
                ++b_used;
                ++tiles;
            }
            mma_commit(bar_a_empty);  // the A tile is free once these MMAs complete
        }
        // the last commit has landed (so no arrive is still in flight at exit)
        if (ok && !*abort_flag && a_used > 0) wait_bounded(bar_a_empty, (a_used - 1) & 1, abort_flag, lim);
    } else if (warp >= 2) {
        // ------------------------------------------------------------ epilogue
        // two warps per TMEM lane quarter: warps 2..5 take chunks 0-1 (columns
        // 0..63 of a tile), warps 6..9 chunks 2-3
        const int quarter = warp & 3;           // TMEM lanes 32 * quarter ..
        const int half = (warp - 2) >> 2;
        const int rl = 32 * quarter + lane;     // row of the tile
        const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
        const int g = lane & 3;                 // sub-row of the query block in this lane
        // after the transposing reduction lane g holds blocks base, base + 1 of a chunk
        const int base = 4 * (g & 1) + 2 * (g >> 1);
        int tiles = 0;
        bool ok = true;
        for (long long it = blockIdx.x; it < items && ok; it += gridDim.x) {
            const int bh = (int)(it / MT), m0 = (int)(it % MT) * 128;
            const int L = valid_len ? valid_len[bh / H] : Npad;
            const int r = m0 + rl;              // query sub-block
            const int I = r >> 2;               // lanes 4i..4i+3 hold the sub-blocks of one block
            int na = L - r * SUB;
            na = na < 0 ? 0 : (na > SUB ? SUB : na);
            const float wa = (float)na;
            float* dst = scores + ((size_t)bh * nB + I) * ld;
            for (int nt = 0; nt < MT; ++nt) {
                const int t = tiles % kLseAccBufs, v = tiles / kLseAccBufs;
                if (!warp_wait_bounded(bar_acc_full(t), v & 1, abort_flag, lim)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // every key sub-block of this tile full: all weights are wa * 16
                const bool full_cols = (nt * 128 + 128) * SUB <= L;
#pragma unroll 1
                for (int ch = 2 * half; ch < 2 * half + 2; ++ch) {
                    uint32_t x[32];
                    tmem_ld32(tmem + (uint32_t)(t * 128 + ch * 32) + lane_off, x);
                    tmem_wait_ld();
                    if (ch == 2 * half + 1) {  // the buffer is free for the MMAs of a later tile
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_acc_empty(t));
                    }
                    float y[32];
                    float ymax = 0.f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        y[i] = __uint_as_float(x[i]) * kScale;
                        ymax = fmaxf(ymax, fabsf(y[i]));
                    }
                    float* drow = dst + nt * 32 + ch * 8;
                    if (__all_sync(0xffffffffu, full_cols && ymax <= 100.f)) {
                        // no shift needed: 2^y stays normal and the sum finite
                        const float w = wa * 16.0f;
                        float pz[8];
#pragma unroll
                        for (int jb = 0; jb < 8; ++jb)
                            pz[jb] = w * ((ex2_approx(y[4 * jb]) + ex2_approx(y[4 * jb + 1])) +
                                          (ex2_approx(y[4 * jb + 2]) + ex2_approx(y[4 * jb + 3])));
                        // transposing reduction over the 4 lanes of the block: after it,
                        // lane g holds the sums of blocks base, base + 1
                        float h4[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float send = (g & 1) ? pz[i] : pz[4 + i];
                            h4[i] = ((g & 1) ? pz[4 + i] : pz[i]) + __shfl_xor_sync(0xffffffffu, send, 1);
                        }
                        float h2[2];
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const float send = (g & 2) ? h4[i] : h4[2 + i];
                            h2[i] = ((g & 2) ? h4[2 + i] : h4[i]) + __shfl_xor_sync(0xffffffffu, send, 2);
                        }
                        if (I < nB)
                            *reinterpret_cast<float2*>(drow + base) =
                                make_float2(__log2f(h2[0]) * 0.69314718055994530942f,
                                            __log2f(h2[1]) * 0.69314718055994530942f);
                    } else {
                        // general form: per-column weights (partial key blocks), max-shifted
                        float blk[8];
#pragma unroll
                        for (int jb = 0; jb < 8; ++jb) {
                            float w[4];
                            float m = -INFINITY;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                int nc = L - (nt * 128 + ch * 32 + 4 * jb + c) * SUB;
                                nc = nc < 0 ? 0 : (nc > SUB ? SUB : nc);
                                w[c] = wa * (float)nc;  // exact: at most 256
                                if (w[c] > 0.f) m = fmaxf(m, y[4 * jb + c]);
                            }
                            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
                            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
                            float z = 0.f;
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                if (w[c] > 0.f) z = fmaf(w[c], ex2_approx(y[4 * jb + c] - m), z);
                            z += __shfl_xor_sync(0xffffffffu, z, 1);
                            z += __shfl_xor_sync(0xffffffffu, z, 2);
                            blk[jb] = m == -INFINITY ? -INFINITY : (m + __log2f(z)) * 0.69314718055994530942f;
                        }
                        if (g == 0 && I < nB) {
                            float4* d4 = reinterpret_cast<float4*>(drow);
                            d4[0] = make_float4(blk[0], blk[1], blk[2], blk[3]);
                            d4[1] = make_float4(blk[4], blk[5], blk[6], blk[7]);
                        }
                    }
                }
                ++tiles;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        if (warp == 0 && lane == 0) {
            if (a_issued > 0) {
                const long long t0 = clock64();
                while (!mbar_try_wait(bar_a_full, (a_issued - 1) & 1) && (uint64_t)(clock64() - t0) < (1ull << 32)) {}
            }
            for (int j = b_issued > 2 ? b_issued - 2 : 0; j < b_issued; ++j) {
                const long long t0 = clock64();
                while (!mbar_try_wait(bar_b_full(j & 1), (j >> 1) & 1) && (uint64_t)(clock64() - t0) < (1ull << 32)) {}
            }
        }
        if (warp == 1 && lane == 0) {
            mma_commit(bar_drain);
            const long long t0 = clock64();
            while (!mbar_try_wait(bar_drain, 0) && (uint64_t)(clock64() - t0) < (1ull << 32)) {}
        }
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace sba

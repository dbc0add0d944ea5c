// score_mma.cuh -- block scores of one (b, h) on the tensor cores, for screening.
//
// The screen needs the dot products qbar[I] . kbar[J] (fp64 block means) to about
// 1e-4 relative accuracy, far more than one bf16 product gives.  Each mean is split
// into bf16 parts, x = hi + lo + r with |r| <= 2^-16 |x| (roughly), and
//     S = qhi . khi + (qhi . klo + qlo . khi)
// is formed by tcgen05.mma (M=128 query rows x N=256 key rows) in two fp32 TMEM
// accumulators, one per bracket, added once in the epilogue: the long sum of the
// large terms is D products, not 3D.  The dropped lo.lo and remainder terms and the
// fp32 accumulation bound the error (see the top-k kernel, which turns that bound
// into a band that is re-scored exactly in fp64).
//
// CTA: 128 threads, one per SM (both accumulators fill the 512 TMEM columns); warp 0
// allocates TMEM, lane 0 issues the TMA loads of the four operand tiles (one stage,
// 192 KB for D = 128) and the MMAs; all four warps read the 128 x 256 fp32 tile out
// of TMEM (thread r = row r = TMEM lane r) and store it.
// Every wait is bounded (SBA_ERR_TIMEOUT, then the CTA drains and exits).

#pragma once
#include <cstdint>
#include <cuda.h>

#include "common.cuh"

namespace sba {

template <int D>
struct ScoreSmem {
    static constexpr int kATile = 128 * D * 2;  // 128 query-block rows
    static constexpr int kBTile = 256 * D * 2;  // 256 key-block rows
    static constexpr int kQh = 0;
    static constexpr int kQl = kQh + kATile;
    static constexpr int kKh = kQl + kATile;
    static constexpr int kKl = kKh + kBTile;
    static constexpr int kBars = kKl + kBTile;  // load_full, mma_done
    static constexpr int kCtl = kBars + 16;     // tmem base, abort flag
    static constexpr int kTotal = kCtl + 16;
    // at least 116 KB so that two CTAs never share an SM (each holds all of TMEM)
    static constexpr int kAlloc = kTotal + 1024 > 116 * 1024 ? kTotal + 1024 : 116 * 1024;
};

// maps: bf16 [BH][nB][D] viewed as 3-D (D, nB, BH); A maps box 64 x 128 rows, B maps
// box 64 x 256 rows.  scores: fp32 [BH][nB][ld], columns >= nB not written.
template <int D>
__global__ void __launch_bounds__(128, 1)
    score_mma_kernel(const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQl,
                     const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
                     float* __restrict__ scores, int nB, int ld, unsigned long long wait_limit) {
    using SM = ScoreSmem<D>;
    constexpr int NCH = D / 64;
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, 256, 0, 0);
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sQh = smem_u32(sm + SM::kQh), sQl = smem_u32(sm + SM::kQl);
    const uint32_t sKh = smem_u32(sm + SM::kKh), sKl = smem_u32(sm + SM::kKl);
    const uint32_t bar_load = smem_u32(sm + SM::kBars), bar_mma = bar_load + 8;
    uint32_t* ctl = reinterpret_cast<uint32_t*>(sm + SM::kCtl);
    volatile uint32_t* abort_flag = ctl + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * 128, n0 = blockIdx.y * 256, bh = blockIdx.z;

    if (tid == 0) {
        mbar_init(bar_load, 1);
        mbar_init(bar_mma, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(smem_u32(ctl), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl[0];

    bool loads_issued = false;
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_load, 2 * SM::kATile + 2 * SM::kBTile);
        for (int c = 0; c < NCH; ++c) {
            tma_load_3d(sQh + c * (128 * 128), &tmQh, bar_load, c * 64, m0, bh);
            tma_load_3d(sQl + c * (128 * 128), &tmQl, bar_load, c * 64, m0, bh);
            tma_load_3d(sKh + c * (256 * 128), &tmKh, bar_load, c * 64, n0, bh);
            tma_load_3d(sKl + c * (256 * 128), &tmKl, bar_load, c * 64, n0, bh);
        }
        loads_issued = true;
        if (wait_bounded(bar_load, 0, abort_flag, wait_limit)) {
            tc_fence_after();
            // three passes: (hi, hi) into columns [0, 256), (hi, lo) and (lo, hi) into [256, 512)
            const uint32_t As[3] = {sQh, sQh, sQl};
            const uint32_t Bs[3] = {sKh, sKl, sKh};
            for (int term = 0; term < 3; ++term) {
                const uint32_t acc = term == 0 ? tmem : tmem + 256;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = smem_desc_sw128(As[term] + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
                    const uint64_t b = smem_desc_sw128(Bs[term] + (kk / 4) * (256 * 128) + (kk % 4) * 32, 16, 1024);
                    mma_bf16_ss(acc, a, b, kIdesc, (term == 2 || kk > 0) ? 1u : 0u);
                }
            }
        }
        mma_commit(bar_mma);   // also covers "no MMA issued" (arrives at once)
    }
    // epilogue: row r of the tile = TMEM lane r
    const bool ok = warp_wait_bounded(bar_mma, 0, abort_flag, wait_limit);
    tc_fence_after();
    const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const bool go = __all_sync(0xffffffffu, ok && !*abort_flag);
    if (go) {
        // Each 32 x 32 chunk of the warp's rows goes through shared memory (the operand
        // tiles are free once the MMAs are done), so that the global stores are whole
        // 128-byte row segments: thread t writes row t of the chunk as eight 16-byte
        // stores, then eight lanes write each row (row stride 36 words: both phases are
        // free of bank conflicts).
        float* stage = reinterpret_cast<float*>(sm) + warp * (32 * 36);
        const int rbase = m0 + warp * 32;
#pragma unroll 1
        for (int c0 = 0; c0 < 256; c0 += 32) {
            uint32_t v[32], v2[32];
            tmem_ld32(tl + c0, v);
            tmem_ld32(tl + 256 + c0, v2);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i)
                *reinterpret_cast<float4*>(stage + lane * 36 + 4 * i) =
                    make_float4(__uint_as_float(v[4 * i]) + __uint_as_float(v2[4 * i]),
                                __uint_as_float(v[4 * i + 1]) + __uint_as_float(v2[4 * i + 1]),
                                __uint_as_float(v[4 * i + 2]) + __uint_as_float(v2[4 * i + 2]),
                                __uint_as_float(v[4 * i + 3]) + __uint_as_float(v2[4 * i + 3]));
            __syncwarp();
            if (n0 + c0 < ld) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {   // four rows per pass, eight lanes per row
                    const int r = 4 * k + lane / 8;
                    const float4 val = *reinterpret_cast<const float4*>(stage + r * 36 + 4 * (lane % 8));
                    if (rbase + r < nB)
                        *reinterpret_cast<float4*>(scores + ((size_t)bh * nB + rbase + r) * ld + n0 + c0 +
                                                   4 * (lane % 8)) = val;
                }
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && tid == 0) {
        // let this CTA's own copies land and MMAs finish before TMEM is freed
        if (loads_issued) {
            const long long t0 = clock64();
            while (!mbar_try_wait(bar_load, 0) && (uint64_t)(clock64() - t0) < (1ull << 32)) {}
        }
        const long long t1 = clock64();
        while (!mbar_try_wait(bar_mma, 0) && (uint64_t)(clock64() - t1) < (1ull << 32)) {}
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace sba

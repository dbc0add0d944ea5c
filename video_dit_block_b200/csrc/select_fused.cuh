// select_fused.cuh -- the one-sub-block router's screen and top-k without a score matrix.
//
// Same selection as the block-mean routing of the page "MiniMax-H3 on 8xH200
// benchmark", section "How SubBlock sparse attention works" (keep the best-scoring
// keep(n, s) key blocks per query block, ties to the lower index), reached the same
// exact way as topk_kernel (fp32 screen with a proven error bound delta, fp64
// re-scoring of the band around the k-th value), but the screened scores live only in
// TMEM and registers.
//
// select_fused_kernel.  A CTA owns 128 query blocks I = m0 + t of one (b, h): row t is
// TMEM lane t, served by four threads (see the warp roles).  The tensor cores score the
// row against 128
// key blocks at a time (a "chunk": M128 N128, S = qhi.khi + qlo.khi + qhi.klo in one
// fp32 TMEM buffer of 128 columns, two buffers), in this order:
//   sample   one hi.hi product against 128 key blocks spread evenly over the head
//            gives the row a value range [lo, hi];
//   pass A   every chunk: a 256-bucket histogram of the screened scores over that
//            range (the edge buckets open), which locates the bucket [A, Bv) holding
//            the k-th largest screened value, and its rank kk inside;
//   pass B   every chunk again (the tensor cores give the same bits): scores at or
//            above hiT = Bv + 2 delta are kept outright (a bitmask), scores in
//            [A - 2 delta, hiT) -- the window -- go to a list of at most kFusedList
//            (value, J) entries.
// Each row then writes a record (header, window, mask) for select_finish_kernel.  A row
// whose window overflows, or whose bound is not finite, gets a pass C instead: its
// screened scores go to ws.scores and its index to ws.ovf_rows, and topk_rest_kernel
// finishes it with topk_kernel's routine.
//
// Warp roles (576 threads, one CTA per SM: 224 KB of shared memory for D = 128):
//   warps 0-15 rows: warp w reads TMEM lanes 32 (w mod 4) .. + 31 and columns 32 (w / 4)
//              .. + 31 of each chunk, so four threads share a row (its histogram by
//              shared-memory atomics, its window by an atomic slot counter)
//   warp 16    TMA: Q hi/lo once, then K hi / K lo tiles through a 3-slot ring
//   warp 17    TMEM allocation (256 columns) and the MMAs (one lane)
// Every wait is bounded (SBA_ERR_TIMEOUT; the CTA then drains its own copies and
// MMAs before freeing TMEM).
//
// select_finish_kernel, one warp per row: tau = the k-th largest screened value,
// found among the window's entries of [A, Bv); entries above tau + 2 delta kept, below
// tau - 2 delta dropped, the rest (the band) ordered by an fp64 dot product in any
// order, and only the members that its error cannot separate at the cut decided on
// exact_score (fixed sequential order), ties to the lower J; the kept blocks written in
// ascending order from the mask.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "select.cuh"

namespace sba {

constexpr int kFusedRowWarps = 16;  // four per 32-lane group of TMEM, 32 columns each
constexpr int kFusedThreads = 32 * kFusedRowWarps + 64;
constexpr int kProducerWarp = kFusedRowWarps, kMmaWarp = kFusedRowWarps + 1;

template <int D>
struct FusedSmem {
    static constexpr int kTile = 128 * D * 2;          // 128 rows of bf16 means
    static constexpr int kSlots = 3;
    static constexpr int kQh = 0;
    static constexpr int kQl = kQh + kTile;
    static constexpr int kK = kQl + kTile;
    // histograms [128 words][128 rows] during pass A; then the window lists
    // [kFusedList][128], the rows' FusedRowInfo and their list counters
    static constexpr int kList = kK + kSlots * kTile;
    static constexpr int kListBytes = kFusedList * 128 * 8;
    static constexpr int kRegionBytes = 128 * 128 * 4;
    // q_full, k_full[3], k_free[3], acc_full[2], acc_empty[2], drain
    static constexpr int kBars = kList + kRegionBytes;
    static constexpr int kCtl = kBars + 12 * 8;  // tmem base, abort flag
    static constexpr int kTotal = kCtl + 16;
    static constexpr int kAlloc = kTotal + 1024;
    static_assert(kListBytes + 128 * 32 + 128 * 4 <= kRegionBytes, "lists, row info and counters share the region");
};

// Header of a row's record in ws.finish (32 bytes); the window entries follow, then
// the keep mask.
struct FusedRowHead {
    float A, Bv;   // bucket of the k-th largest screened value: [A, Bv)
    double delta;  // screen error bound of the row
    int32_t cnt;   // window entries; -1: the row was handed to topk_rest_kernel
    int32_t kk;    // rank of the k-th value inside its bucket (1-based)
    int32_t pad[2];
};

// What the row's thread of part 0 publishes for the row's other three threads.
struct FusedRowInfo {
    float A, Bv, hiT, loT;
    double delta;
    int32_t kk;
    int32_t flags;  // 1: collect the window; 2: hand the row to topk_rest_kernel
};

// Bucket of a screened value: floor(f * bscale + boff) clamped to [0, 255] (one fused
// multiply-add, rounded to nearest, then a floor conversion to an unsigned byte, which
// clamps to [0, 255] by itself and sends NaN to 0), so the map is non-decreasing in f.
// boff = -lo * bscale puts the row's smallest sampled value lo at the bottom of bucket 0,
// up to rounding.
__device__ __forceinline__ int fused_bucket(float f, float bscale, float boff) {
    unsigned short b;
    asm("cvt.rmi.u8.f32 %0, %1;" : "=h"(b) : "f"(__fmaf_rn(f, bscale, boff)));
    return (int)b;
}

// Smallest float x (over all non-NaN floats, in order) with fused_bucket(x) >= b, for
// 1 <= b <= 255 and a finite bscale > 0 (then bucket(-inf) = 0 and bucket(+inf) = 255).
// Starts from (b - boff) / bscale, within a few units in the last place of the edge for
// ranges that fp32 resolves, and steps float by float; a bisection over the whole
// float order decides when that has not settled within 64 steps.
__device__ float fused_bucket_edge(int b, float bscale, float boff) {
    uint32_t g = f32_key(__fdiv_rn(__fsub_rn((float)b, boff), bscale));
    const uint32_t kmin = f32_key(-INFINITY), kmax = f32_key(INFINITY);
    if (g > kmin && g <= kmax) {
        if (fused_bucket(key_to_f32(g), bscale, boff) >= b) {
            for (int step = 0; step < 64; ++step) {  // down while the float below is still in
                if (g == kmin || fused_bucket(key_to_f32(g - 1u), bscale, boff) < b) return key_to_f32(g);
                --g;
            }
        } else {
            for (int step = 0; step < 64; ++step) {  // up until in
                ++g;
                if (g > kmax) break;
                if (fused_bucket(key_to_f32(g), bscale, boff) >= b) return key_to_f32(g);
            }
        }
    }
    uint32_t lo = kmin, hi = kmax;
    while (hi - lo > 1u) {
        const uint32_t mid = lo + (hi - lo) / 2u;
        if (fused_bucket(key_to_f32(mid), bscale, boff) >= b)
            hi = mid;
        else
            lo = mid;
    }
    return key_to_f32(hi);
}

// maps: bf16 [BH][nB][D] as 3-D (D, nB, BH), box 64 x 128 rows; tmKs views khi with
// row stride `stride` blocks (the sample).  Grid (ceil(nB / 128), BH).
template <int D>
__global__ void __launch_bounds__(kFusedThreads, 1)
    select_fused_kernel(const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmQl,
                        const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmKl,
                        const __grid_constant__ CUtensorMap tmKs, SelectWorkspace ws,
                        const int32_t* __restrict__ valid_len, int H, int Npad, int stride, double sparsity,
                        int budget, int kmax, int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
                        unsigned long long wait_limit) {
    using SM = FusedSmem<D>;
    constexpr int NCH = D / 64;
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, 0, 0);
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nBmax = Npad / kBlock;
    const int m0 = blockIdx.x * 128, bh = blockIdx.y;
    const int L = sample_len(valid_len, bh / H, Npad);
    const int nBb = (L + kBlock - 1) / kBlock;
    const int k = keep_count_budget(nBb, sparsity, budget);

    // ---- nothing dropped: every block, ascending; no tensor work.  (Rows I >= nBb
    // of other tiles are left to select_finish_kernel.)
    if (k >= nBb || m0 >= nBb) {
        if (k >= nBb) {
            for (int r = warp; r < 128 && m0 + r < nBmax; r += kFusedThreads / 32) {
                const size_t rid = (size_t)bh * nBmax + m0 + r;
                const int n = m0 + r < nBb ? nBb : 0;
                for (int j = lane; j < n; j += 32) kv_idx[rid * kmax + j] = j;
                if (lane == 0) kv_cnt[rid] = n;
            }
        }
        return;
    }

    const uint32_t sQh = smem_u32(sm + SM::kQh), sQl = smem_u32(sm + SM::kQl), sK = smem_u32(sm + SM::kK);
    const uint32_t bars = smem_u32(sm + SM::kBars);
    const uint32_t q_full = bars, k_full = bars + 8, k_free = bars + 32, acc_full = bars + 56,
                   acc_empty = bars + 72, drain_bar = bars + 88;
    uint32_t* ctl = reinterpret_cast<uint32_t*>(sm + SM::kCtl);
    volatile uint32_t* abort_flag = ctl + 1;
    const int nC = (nBb + 127) / 128;  // chunks of this sample's key blocks

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 3; ++i) {
            mbar_init(k_full + 8 * i, 1);
            mbar_init(k_free + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(acc_full + 8 * i, 1);
            mbar_init(acc_empty + 8 * i, kFusedRowWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(smem_u32(ctl), 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl[0];

    bool any_fallback = false;
    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        int g = 0;  // K tiles issued
        auto load_k = [&](const CUtensorMap* map, int row) -> bool {
            const int slot = g % 3;
            if (g >= 3 && !wait_bounded(k_free + 8 * slot, ((g / 3) - 1) & 1, abort_flag, wait_limit)) return false;
            mbar_arrive_expect_tx(k_full + 8 * slot, SM::kTile);
            for (int c = 0; c < NCH; ++c)
                tma_load_3d(sK + slot * SM::kTile + c * (128 * 128), map, k_full + 8 * slot, c * 64, row, bh);
            ++g;
            return true;
        };
        auto load_passes = [&](int npass) {
            for (int p = 0; p < npass; ++p)
                for (int ch = 0; ch < nC; ++ch)
                    if (!load_k(&tmKh, ch * 128) || !load_k(&tmKl, ch * 128)) return;
        };
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, 2 * SM::kTile);
            for (int c = 0; c < NCH; ++c) {
                tma_load_3d(sQh + c * (128 * 128), &tmQh, q_full, c * 64, m0, bh);
                tma_load_3d(sQl + c * (128 * 128), &tmQl, q_full, c * 64, m0, bh);
            }
            if (load_k(&tmKs, 0)) load_passes(2);
        }
        __syncwarp();
        any_fallback = __syncthreads_or(0);
        if (any_fallback && lane == 0 && !*abort_flag) load_passes(1);
        __syncwarp();
        if (*abort_flag && lane == 0) {
            // let the copies this CTA issued land before the CTA exits
            const long long t0 = clock64();
            while (!mbar_try_wait(q_full, 0) && (uint64_t)(clock64() - t0) < (1ull << 32)) {}
            for (int i = g - 3 < 0 ? 0 : g - 3; i < g; ++i) {
                const long long t1 = clock64();
                while (!mbar_try_wait(k_full + 8 * (i % 3), (i / 3) & 1) && (uint64_t)(clock64() - t1) < (1ull << 32)) {}
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        int g = 0, a = 0;  // K tiles consumed, accumulator uses
        auto acquire = [&](uint32_t& d) -> bool {
            const int buf = a & 1;
            if (a >= 2 && !poll_bounded(acc_empty + 8 * buf, ((a >> 1) - 1) & 1, abort_flag, wait_limit)) return false;
            d = tmem + 128u * buf;
            return true;
        };
        auto product = [&](uint32_t d, uint32_t A, uint32_t B, bool first) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t ad = smem_desc_sw128(A + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(B + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
                mma_bf16_ss(d, ad, bd, kIdesc, (first && kk == 0) ? 0u : 1u);
            }
        };
        auto chunk = [&]() -> bool {
            uint32_t d;
            if (!acquire(d)) return false;
            const int hs = g % 3, ls = (g + 1) % 3;
            if (!poll_bounded(k_full + 8 * hs, (g / 3) & 1, abort_flag, wait_limit)) return false;
            tc_fence_after();
            product(d, sQh, sK + hs * SM::kTile, true);   // hi.hi
            product(d, sQl, sK + hs * SM::kTile, false);  // lo.hi
            mma_commit(k_free + 8 * hs);
            if (!poll_bounded(k_full + 8 * ls, ((g + 1) / 3) & 1, abort_flag, wait_limit)) return false;
            tc_fence_after();
            product(d, sQh, sK + ls * SM::kTile, false);  // hi.lo
            mma_commit(k_free + 8 * ls);
            mma_commit(acc_full + 8 * (a & 1));
            g += 2;
            ++a;
            return true;
        };
        auto passes = [&](int npass) {
            for (int p = 0; p < npass; ++p)
                for (int ch = 0; ch < nC; ++ch)
                    if (!chunk()) return;
        };
        if (lane == 0 && wait_bounded(q_full, 0, abort_flag, wait_limit)) {
            uint32_t d;
            if (acquire(d) && poll_bounded(k_full, 0, abort_flag, wait_limit)) {
                tc_fence_after();
                product(d, sQh, sK, true);  // the sample: hi.hi only
                mma_commit(k_free);
                mma_commit(acc_full);
                g = 1;
                a = 1;
                passes(2);
            }
        }
        __syncwarp();
        any_fallback = __syncthreads_or(0);
        if (any_fallback && lane == 0 && !*abort_flag) passes(1);
        __syncwarp();
        if (*abort_flag && lane == 0) {
            mma_commit(drain_bar);  // arrives once every MMA issued above is done
            const long long t0 = clock64();
            while (!mbar_try_wait(drain_bar, 0) && (uint64_t)(clock64() - t0) < (1ull << 32)) {}
        }
    } else {
        // ------------------------------------------------------------ rows
        // Warp w serves rows 32 (w mod 4) .. + 31 (its TMEM lanes) and columns
        // 32 part .. + 31 of every chunk, part = w / 4: four threads per row.
        const int part = warp >> 2;
        const int t = 32 * (warp & 3) + lane;  // row of the tile = TMEM lane
        const int I = m0 + t;
        const bool active = I < nBb;
        const long long rid = (long long)bh * nBmax + I;
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        unsigned char* region = sm + SM::kList;
        uint32_t* hist = reinterpret_cast<uint32_t*>(region);  // [128 words][128 rows], pass A
        float2* list = reinterpret_cast<float2*>(region);      // [kFusedList][128] (value, J bits), pass B
        FusedRowInfo* info = reinterpret_cast<FusedRowInfo*>(region + SM::kListBytes);
        int* rowcnt = reinterpret_cast<int*>(region + SM::kListBytes + 128 * sizeof(FusedRowInfo));
        float* part_lo = reinterpret_cast<float*>(region);  // [4][128] sample ranges, before pass A
        float* part_hi = part_lo + 4 * 128;
        unsigned char* rec = ws.finish + (size_t)rid * ws.fstride;
        auto rows_sync = [&]() { named_bar_sync(1, 32 * kFusedRowWarps); };
        int a = 0, buf = 0;
        bool ok = true;
        // this warp's 32 columns of the next accumulator use; then the buffer is released
        auto fetch = [&](uint32_t (&v)[32]) -> bool {
            buf = a & 1;
            const bool got = warp_wait_bounded(acc_full + 8 * buf, (a >> 1) & 1, abort_flag, wait_limit);
            ++a;
            if (!got) return false;
            tc_fence_after();
            tmem_ld32(tl + 128u * buf + 32u * part, v);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty + 8 * buf);
            return true;
        };

        // ---- sample: the row's value range [lo, hi], and the bucket map over it
        {
            float lo = INFINITY, hi = -INFINITY;
            uint32_t v[32];
            ok = fetch(v);
            if (ok) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const bool in = (long long)stride * (32 * part + i) < nBb;
                    lo = in ? fminf(lo, __uint_as_float(v[i])) : lo;
                    hi = in ? fmaxf(hi, __uint_as_float(v[i])) : hi;
                }
            }
            part_lo[part * 128 + t] = lo;
            part_hi[part * 128 + t] = hi;
        }
        rows_sync();
        float bscale = 0.f, boff = 0.f;
        {
            float lo = part_lo[t], hi = part_hi[t];
#pragma unroll
            for (int q = 1; q < 4; ++q) {
                lo = fminf(lo, part_lo[q * 128 + t]);
                hi = fmaxf(hi, part_hi[q * 128 + t]);
            }
            const float range = hi - lo;
            if (range > 0.f && range <= 3.0e38f) {
                const float sc = 256.0f / range;
                if (sc <= 3.0e38f && fabsf(lo) * sc <= 3.0e38f) {
                    bscale = sc;
                    boff = -lo * sc;
                }
            }
        }
        rows_sync();  // the ranges are read: clear this thread's quarter of the row's histogram
#pragma unroll 8
        for (int w = 32 * part; w < 32 * part + 32; ++w) hist[w * 128 + t] = 0u;
        rows_sync();

        // the bound's inputs, fetched before pass A so that their latency is hidden
        const double qn_row = part == 0 && active ? ws.qnorm[(size_t)rid] : 0.0;
        const double kmx_bh = part == 0 && active ? ws.kmaxn[bh] : 0.0;

        // ---- pass A: 256-bucket histogram of the row's screened scores
        for (int ch = 0; ch < nC && ok; ++ch) {
            uint32_t v[32];
            if (!(ok = fetch(v))) break;
            const int lim = active ? nBb - ch * 128 - 32 * part : 0;  // columns i < lim are blocks
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const uint32_t b = (uint32_t)fused_bucket(__uint_as_float(v[i]), bscale, boff);
                atomicAdd(&hist[(b >> 1) * 128 + t], i < lim ? 1u + (b & 1u) * 0xFFFFu : 0u);
            }
        }
        rows_sync();

        // ---- (part 0) the bucket [A, Bv) of the k-th largest value, its rank kk inside,
        // and the window around it
        FusedRowInfo ri;
        ri.A = -INFINITY;
        ri.Bv = INFINITY;
        ri.hiT = INFINITY;
        ri.loT = -INFINITY;
        ri.delta = INFINITY;
        ri.kk = 0;
        ri.flags = 0;
        if (part == 0 && active && ok) {
            int cum = 0, bstar = -1;
            // buckets from the top, 16 words (32 buckets) loaded at a time
            for (int w0 = 112; w0 >= 0 && bstar < 0; w0 -= 16) {
                uint32_t words[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) words[i] = hist[(w0 + i) * 128 + t];
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    const int c1 = (int)(words[i] >> 16), c0 = (int)(words[i] & 0xFFFFu);
                    if (bstar < 0) {
                        if (cum + c1 >= k) {
                            bstar = 2 * (w0 + i) + 1;
                        } else {
                            cum += c1;
                            if (cum + c0 >= k)
                                bstar = 2 * (w0 + i);
                            else
                                cum += c0;
                        }
                    }
                }
            }
            ri.kk = k - cum;  // 1 <= kk <= the bucket's count
            const double qn = qn_row, kmx = kmx_bh;
            ri.delta = 2.0 * (4.0 * 0x1p-16 + 3.0 * D * 0x1p-22) * qn * kmx + 3.0 * D * 0x1p-120 * (1.0 + qn + kmx);
            // a bound that is not meaningful in fp32 goes to the row routine
            if (bstar < 0 || !(qn * kmx < 1.0e30) || !(ri.delta < 1.0e30)) {
                ri.flags = 2;
            } else {
                ri.flags = 1;
                if (bscale > 0.f) {
                    if (bstar > 0) ri.A = fused_bucket_edge(bstar, bscale, boff);
                    if (bstar < 255) ri.Bv = fused_bucket_edge(bstar + 1, bscale, boff);
                }
                if (ri.Bv < INFINITY) ri.hiT = __double2float_ru((double)ri.Bv + 2.0 * ri.delta);
                if (ri.A > -INFINITY) ri.loT = __double2float_rd((double)ri.A - 2.0 * ri.delta);
            }
        }
        rows_sync();  // histograms read: the lists and row info may overwrite them
        if (part == 0) {
            info[t] = ri;
            rowcnt[t] = 0;
        }
        rows_sync();
        ri = info[t];
        const bool collect = (ri.flags & 1) != 0;

        // ---- pass B: sure keeps into the row's mask, the window into the list
        for (int ch = 0; ch < nC && ok; ++ch) {
            uint32_t v[32];
            if (!(ok = fetch(v))) break;
            const int j0 = ch * 128 + 32 * part;
            const int lim = collect ? nBb - j0 : 0;
            uint32_t word = 0u;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float f = __uint_as_float(v[i]);
                const bool in = i < lim;
                word |= (in && f >= ri.hiT) ? 1u << i : 0u;
                const bool win = in && f >= ri.loT && f < ri.hiT;
                if (__any_sync(0xffffffffu, win)) {  // rare: no shared-memory traffic otherwise
                    if (win) {
                        const int slot = atomicAdd(&rowcnt[t], 1);
                        if (slot < kFusedList) list[slot * 128 + t] = make_float2(f, __int_as_float(j0 + i));
                    }
                }
            }
            if (collect) *reinterpret_cast<uint32_t*>(rec + 32 + 8 * kFusedList + 16 * ch + 4 * part) = word;
        }
        rows_sync();
        const int cnt = rowcnt[t];
        const bool fallback = (ri.flags & 2) != 0 || (collect && cnt > kFusedList);
        any_fallback = __syncthreads_or(part == 0 && active && fallback && ok);

        // ---- pass C (only when some row of the tile fell back): its screened scores
        if (any_fallback && ok) {
            for (int ch = 0; ch < nC && ok; ++ch) {
                uint32_t v[32];
                if (!(ok = fetch(v))) break;
                if (active && fallback) {
                    const int c0 = ch * 128 + 32 * part;
                    float* dst = ws.scores + (size_t)rid * ws.ld + c0;
#pragma unroll
                    for (int i = 0; i < 32; i += 4)
                        if (c0 + i + 4 <= ws.ld)
                            *reinterpret_cast<float4*>(dst + i) =
                                make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                            __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                }
            }
            if (part == 0 && ok && active && fallback) ws.ovf_rows[atomicAdd(ws.ovf_count, 1)] = (int32_t)rid;
        }
        if (!__all_sync(0xffffffffu, ok)) ok = false;

        // ---- the record: header, then (warp by warp, coalesced) the window entries
        if (part == 0 && ok && active) {
            FusedRowHead h;
            h.A = ri.A;
            h.Bv = ri.Bv;
            h.delta = ri.delta;
            h.cnt = fallback ? -1 : cnt;
            h.kk = ri.kk;
            h.pad[0] = 0;
            h.pad[1] = 0;
            *reinterpret_cast<FusedRowHead*>(rec) = h;
        }
        if (part == 0) {
            const int n_copy = (ok && active && !fallback) ? cnt : 0;
            for (int r = 0; r < 32; ++r) {
                const int row = 32 * (warp & 3) + r;
                const int n = __shfl_sync(0xffffffffu, n_copy, r);
                float2* dst =
                    reinterpret_cast<float2*>(ws.finish + ((size_t)bh * nBmax + m0 + row) * ws.fstride + 32);
                for (int e = lane; e < n; e += 32) dst[e] = list[e * 128 + row];
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ------------------------------------------------------------------ finish
constexpr int kFinishWarps = 8;

// Shared-memory bytes per warp: the band's refined and exact scores and blocks, the
// blocks kept beyond the mask, and the row's mask words.
template <int D>
struct FinishSmem {
    static constexpr int kR = 0;                       // double [64] refined band scores
    static constexpr int kX = kR + kFusedList * 8;     // double [64] exact scores (or blocks)
    static constexpr int kJ = kX + kFusedList * 8;     // int [64] band blocks
    static constexpr int kE = kJ + kFusedList * 4;     // int [64] extra kept blocks
    static constexpr int kW = kE + kFusedList * 4;     // uint32 [128] mask words
    static constexpr int kWarp = kW + 128 * 4;
    static constexpr int kTotal = kFinishWarps * kWarp;
};

// One routing row per warp from its record (see the file comment).  Rows of samples
// that keep every block were written by select_fused_kernel; rows past the sample's
// blocks get kv_cnt = 0 here; rows handed to topk_rest_kernel are skipped.
template <int D>
__global__ void __launch_bounds__(32 * kFinishWarps) select_finish_kernel(SelectWorkspace ws,
                                                                          const int32_t* __restrict__ valid_len,
                                                                          int H, int Npad, double sparsity, int budget,
                                                                          int kmax, int32_t* __restrict__ kv_idx,
                                                                          int32_t* __restrict__ kv_cnt, long long rows) {
    using FS = FinishSmem<D>;
    extern __shared__ __align__(16) unsigned char fsm_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rid = blockIdx.x * kFinishWarps + warp;  // rows < 2^28
    if (rid >= rows) return;
    unsigned char* wsm = fsm_raw + warp * FS::kWarp;
    const int nBmax = Npad / kBlock;
    const int bh = rid / nBmax;
    const int I = rid - bh * nBmax;
    const int L = sample_len(valid_len, bh / H, Npad);
    const int nBb = (L + kBlock - 1) / kBlock;
    const int k = keep_count_budget(nBb, sparsity, budget);
    if (I >= nBb) {
        if (lane == 0) kv_cnt[rid] = 0;
        return;
    }
    if (k >= nBb) return;
    const unsigned char* rec = ws.finish + (size_t)rid * ws.fstride;
    const FusedRowHead h = *reinterpret_cast<const FusedRowHead*>(rec);
    if (h.cnt < 0) return;
    const int cnt = min(h.cnt, kFusedList);
    const float2* ent = reinterpret_cast<const float2*>(rec + 32);

    // ---- the window (lane holds entries lane and lane + 32), the row's mask (the
    // blocks kept outright) and its query mean: all loads issued together
    const int W = (nBb + 31) / 32;
    const uint32_t* mw = reinterpret_cast<const uint32_t*>(rec + 32 + 8 * kFusedList);
    uint32_t mwords[4];  // words lane + 32 i (W <= 128)
#pragma unroll
    for (int i = 0; i < 4; ++i) mwords[i] = lane + 32 * i < W ? mw[lane + 32 * i] : 0u;
    const double* qrow = ws.qmean64 + (size_t)rid * D;
    double qd[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) qd[i] = qrow[lane + 32 * i];
    float f[2];
    int jb[2];
    bool has[2], mem[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int e = lane + 32 * q;
        has[q] = e < cnt;
        const float2 x = has[q] ? ent[e] : make_float2(0.f, 0.f);
        f[q] = x.x;
        jb[q] = __float_as_int(x.y);
        mem[q] = has[q] && f[q] >= h.A && f[q] < h.Bv;
    }
    // a record not written by this call (its screen aborted) must not send us out of bounds
    if (__any_sync(0xffffffffu, (has[0] && (jb[0] < 0 || jb[0] >= nBb)) || (has[1] && (jb[1] < 0 || jb[1] >= nBb)))) {
        if (lane == 0) raise_device_error(kErrBadRouting);
        return;
    }
    // tau: the kk-th largest member of the bucket (the members' values gathered first)
    float* mf = reinterpret_cast<float*>(wsm + FS::kX);  // free until the band needs it
    const uint32_t mb0 = __ballot_sync(0xffffffffu, mem[0]), mb1 = __ballot_sync(0xffffffffu, mem[1]);
    if (mem[0]) mf[__popc(mb0 & lanemask_lt())] = f[0];
    if (mem[1]) mf[__popc(mb0) + __popc(mb1 & lanemask_lt())] = f[1];
    const int n_mem = __popc(mb0) + __popc(mb1);
    __syncwarp();
    int gt[2] = {0, 0}, ge[2] = {0, 0};
    for (int u = 0; u < n_mem; ++u) {
        const float fu = mf[u];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            gt[q] += fu > f[q] ? 1 : 0;
            ge[q] += fu >= f[q] ? 1 : 0;
        }
    }
    __syncwarp();
    const bool hit0 = mem[0] && gt[0] < h.kk && h.kk <= ge[0];
    const bool hit1 = mem[1] && gt[1] < h.kk && h.kk <= ge[1];
    const uint32_t hb0 = __ballot_sync(0xffffffffu, hit0), hb1 = __ballot_sync(0xffffffffu, hit1);
    if (!hb0 && !hb1) {  // cannot happen when both passes saw the same scores
        if (lane == 0) raise_device_error(kErrBadRouting);
        return;
    }
    const float tau =
        hb0 ? __shfl_sync(0xffffffffu, f[0], __ffs(hb0) - 1) : __shfl_sync(0xffffffffu, f[1], __ffs(hb1) - 1);
    const float hi2 = __double2float_ru((double)tau + 2.0 * h.delta);
    const float lo2 = __double2float_rd((double)tau - 2.0 * h.delta);
    bool keep[2], band[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        keep[q] = has[q] && f[q] > hi2;
        band[q] = has[q] && !keep[q] && f[q] >= lo2;
    }
    const uint32_t kb0 = __ballot_sync(0xffffffffu, keep[0]), kb1 = __ballot_sync(0xffffffffu, keep[1]);
    const uint32_t bb0 = __ballot_sync(0xffffffffu, band[0]), bb1 = __ballot_sync(0xffffffffu, band[1]);
    // the row's mask into shared memory, and its count
    uint32_t* words = reinterpret_cast<uint32_t*>(wsm + FS::kW);
    int n_sure = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (lane + 32 * i < W) words[lane + 32 * i] = mwords[i];
        n_sure += __popc(mwords[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n_sure += __shfl_xor_sync(0xffffffffu, n_sure, off);
    const int n_in = n_sure + __popc(kb0) + __popc(kb1);
    const int n_band = __popc(bb0) + __popc(bb1);
    const int need = k - n_in;  // 1 <= need <= n_band

    int* xj = reinterpret_cast<int*>(wsm + FS::kE);  // blocks kept beyond the mask
    int n_extra = 0;
#pragma unroll
    for (int q = 0; q < 2; ++q) {  // window entries above the band
        const uint32_t kb = q ? kb1 : kb0;
        if (keep[q]) xj[n_extra + __popc(kb & lanemask_lt())] = jb[q];
        n_extra += __popc(kb);
    }
    if (need >= n_band) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint32_t bb = q ? bb1 : bb0;
            if (band[q]) xj[n_extra + __popc(bb & lanemask_lt())] = jb[q];
            n_extra += __popc(bb);
        }
    } else {
        // The band in fp64.  First every member's dot product q.k_J in any order (lanes
        // over channels, fused multiply-adds, a butterfly): r_m.  It and exact_score
        // (the fixed sequential order) are each within (D + 2) 2^-53 sum_d |q_d k_d|
        // <= (D + 2) 2^-53 |q| max|k| of the true product, so members whose r differ by
        // more than 2 eps are ordered by r; only those within 2 eps of the cut are
        // decided on exact_score, ties to the lower J.
        double* rx = reinterpret_cast<double*>(wsm + FS::kR);
        double* ex = reinterpret_cast<double*>(wsm + FS::kX);
        int* bj = reinterpret_cast<int*>(wsm + FS::kJ);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint32_t bb = q ? bb1 : bb0;
            const int base = q ? __popc(bb0) : 0;
            if (band[q]) bj[base + __popc(bb & lanemask_lt())] = jb[q];
        }
        __syncwarp();
        const double* kbase = ws.kmean64 + (size_t)bh * nBmax * D;
        const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)D));
        for (int m = 0; m < n_band; m += 4) {  // four members per step: their loads in flight together
            double p[4];
            double kv[4][D / 32];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const double* kr = kbase + (size_t)bj[m + u < n_band ? m + u : m] * D;
#pragma unroll
                for (int i = 0; i < D / 32; ++i) kv[u][i] = kr[lane + 32 * i];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                p[u] = 0.0;
#pragma unroll
                for (int i = 0; i < D / 32; ++i) p[u] = fma(qd[i], kv[u][i], p[u]);
            }
            // a transposing butterfly: at distance 16 each lane keeps two of the four
            // sums (members 0, 1 below lane 16, members 2, 3 from it) and sends the
            // other two, at distance 8 one of those, then three plain steps; lanes
            // 8u .. 8u + 7 end with member u's sum over all 32 lanes
            const bool up16 = (lane & 16) != 0, up8 = (lane & 8) != 0;
            double h0 = up16 ? p[2] : p[0], h1 = up16 ? p[3] : p[1];
            h0 += __shfl_xor_sync(0xffffffffu, up16 ? p[0] : p[2], 16);
            h1 += __shfl_xor_sync(0xffffffffu, up16 ? p[1] : p[3], 16);
            double r = up8 ? h1 : h0;
            r += __shfl_xor_sync(0xffffffffu, up8 ? h0 : h1, 8);
#pragma unroll
            for (int off = 4; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
            if ((lane & 7) == 0 && m + (lane >> 3) < n_band) rx[m + (lane >> 3)] = r * inv;
        }
        __syncwarp();
        const double qn = ws.qnorm[(size_t)rid], kmx = ws.kmaxn[bh];
        const double eps = 2.0 * (D + 4.0) * 0x1p-53 * qn * kmx * inv + 0x1p-1000;
        // r_cut: the need-th largest r
        double r_cut = 0.0;
        bool got = false;
        for (int r0 = 0; r0 < n_band; r0 += 32) {
            const int m = r0 + lane;
            bool hit = false;
            double rm = 0.0;
            if (m < n_band) {
                rm = rx[m];
                int gt = 0, ge = 0;
                for (int u = 0; u < n_band; ++u) {
                    gt += rx[u] > rm ? 1 : 0;
                    ge += rx[u] >= rm ? 1 : 0;
                }
                hit = gt < need && need <= ge;
            }
            const uint32_t hb = __ballot_sync(0xffffffffu, hit);
            if (hb && !got) {
                r_cut = __shfl_sync(0xffffffffu, rm, __ffs(hb) - 1);
                got = true;
            }
        }
        const double hiC = r_cut + 2.0 * eps, loC = r_cut - 2.0 * eps;
        // above the cut: kept; at the cut: to decide exactly
        int n_top = 0, n_tie = 0;
        for (int r0 = 0; r0 < n_band; r0 += 32) {
            const int m = r0 + lane;
            const double rm = m < n_band ? rx[m] : -INFINITY;
            const bool top = m < n_band && rm > hiC;
            const bool tie = m < n_band && !top && rm >= loC;
            const uint32_t tb = __ballot_sync(0xffffffffu, top);
            if (top) xj[n_extra + __popc(tb & lanemask_lt())] = bj[m];
            n_extra += __popc(tb);
            n_top += __popc(tb);
            const uint32_t eb = __ballot_sync(0xffffffffu, tie);
            if (tie) ex[n_tie + __popc(eb & lanemask_lt())] = __longlong_as_double((long long)bj[m]);
            n_tie += __popc(eb);
        }
        __syncwarp();
        const int slots = need - n_top;  // 1 <= slots <= n_tie
        if (slots >= n_tie) {
            for (int e = lane; e < n_tie; e += 32) xj[n_extra + e] = (int)__double_as_longlong(ex[e]);
            n_extra += n_tie;
        } else {
            // exact_score for the members at the cut (rare: near-equal scores)
            int* tj = bj;  // reuse: the band's blocks are no longer needed
            for (int e = lane; e < n_tie; e += 32) tj[e] = (int)__double_as_longlong(ex[e]);
            __syncwarp();
            for (int e = lane; e < n_tie; e += 32) ex[e] = exact_score(qrow, kbase + (size_t)tj[e] * D, D, inv);
            __syncwarp();
            for (int r0 = 0; r0 < n_tie; r0 += 32) {
                const int m = r0 + lane;
                bool kept = false;
                if (m < n_tie) {
                    const double xm = ex[m];
                    const int jm = tj[m];
                    int rank = 0;
                    for (int u = 0; u < n_tie; ++u)
                        rank += (ex[u] > xm || (ex[u] == xm && tj[u] < jm)) ? 1 : 0;
                    kept = rank < slots;
                }
                const uint32_t kbm = __ballot_sync(0xffffffffu, kept);
                if (kept) xj[n_extra + __popc(kbm & lanemask_lt())] = tj[m];
                n_extra += __popc(kbm);
            }
        }
    }
    __syncwarp();

    // ---- the mask plus the extra blocks, written in ascending order
    for (int e = lane; e < n_extra; e += 32) atomicOr(&words[xj[e] >> 5], 1u << (xj[e] & 31));
    __syncwarp();
    int32_t* out = kv_idx + (size_t)rid * kmax;
    int pos = 0;
    for (int w0 = 0; w0 < W; w0 += 32) {
        uint32_t word = w0 + lane < W ? words[w0 + lane] : 0u;
        const int c = __popc(word);
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        int p = pos + incl - c;
        while (word) {
            const int bit = __ffs(word) - 1;
            word &= word - 1;
            if (p < kmax) out[p] = 32 * (w0 + lane) + bit;
            ++p;
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        kv_cnt[rid] = pos;
        if (pos != k) raise_device_error(kErrBadRouting);
    }
}

}  // namespace sba

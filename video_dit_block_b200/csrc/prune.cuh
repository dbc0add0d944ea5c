// prune.cuh -- token pruning by feature-norm saliency, and the gather of the kept rows.
//
// The page "Sol Video Inference Engine" (sjmshsh.github.io), LTX-2.3 appendix,
// stage 2, prunes the video tokens before the refinement transformer: 50% of them
// are kept by feat_norm saliency.  Here the saliency of token n of sample b is the
// Euclidean norm of its feature vector x[b][n][0..C), ranked through its square;
// each sample keeps keep_tokens(L_b, r) = clamp(ceil(r L_b - 1e-9), 1, L_b) of its
// L_b valid tokens, equal norms going to the lower index, listed in their original
// order (the pruned sequence keeps the raster order of the latent lattice).
//
// Exactness.  Every square of a bf16 value is exact in fp64, and each token's sum
// runs over its channels in order, one fp64 fused multiply-add per channel, so the
// squared norms are bit for bit the sequential fp64 sums; the selection on them is
// then exact (a radix select on the order-preserving bits, ties to the lower index).
//
//   token_norm_kernel    HBM-bound: 128 tokens per CTA, their rows streamed through a
//                        4-stage ring of TMA tiles (128 tokens x 64 channels, 128-byte
//                        swizzle, so the threads reading one 16-byte chunk each of
//                        eight consecutive rows hit distinct banks); thread t sums
//                        token t's channels in order.
//   prune_select_kernel  one CTA per sample: a bucket histogram over the sample's range
//                        locates the k-th largest squared norm, a radix select among
//                        that bucket's members finds it, an in-order compaction by
//                        block scans lists the kept tokens.
//   gather_rows_kernel   HBM-bound row copy dst[bh][p] = src[bh][idx[b][p]] (zero rows
//                        past the kept count), 16-byte units.
#pragma once
#include <cstdint>
#include <type_traits>
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace sba {

constexpr int kNormRows = 128;      // tokens per CTA
constexpr int kNormBoxCols = 64;    // channels per TMA box (128 bytes)
constexpr int kNormBoxes = 1;       // boxes per stage
constexpr int kNormStages = 4;
constexpr int kNormStageBytes = kNormBoxes * kNormRows * kNormBoxCols * 2;   // 16 KB
constexpr int kNormSmem = kNormStages * kNormStageBytes + 1024 + 2 * kNormStages * 8 + 16;

// keep_tokens(n, r) with the same fp64 operations as the host rule.
__host__ __device__ inline int keep_tokens(int n, double r) {
    if (n <= 0) return 0;
#ifdef __CUDA_ARCH__
    double x = ceil(__dadd_rn(__dmul_rn(r, (double)n), -1e-9));
#else
    volatile double t = r * (double)n;  // volatile: no fused multiply-add
    double x = ceil(t - 1e-9);
#endif
    if (x < 1.0) x = 1.0;
    if (x > (double)n) x = (double)n;
    return (int)x;
}

// x viewed as rows [B*N][C] (tensor map tmX: box 64 channels x 128 rows, 128-byte
// swizzle).  norm2[row] = sum_c x[row][c]^2 in channel order (0 for padding tokens).
// 160 threads: warps 0-3 sum (thread t = token t of the tile), warp 4 lane 0 loads.
__global__ void __launch_bounds__(160) token_norm_kernel(const __grid_constant__ CUtensorMap tmX,
                                                        const int32_t* __restrict__ valid_len, int N, int C,
                                                        long long rows, double* __restrict__ norm2,
                                                        unsigned long long wait_limit) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t base = smem_u32(sm);
    const uint32_t bars = base + kNormStages * kNormStageBytes;
    auto bar_full = [&](int s) { return bars + 8u * s; };
    auto bar_empty = [&](int s) { return bars + 8u * (kNormStages + s); };
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sm + kNormStages * kNormStageBytes +
                                                                         2 * kNormStages * 8);
    const int tid = threadIdx.x, warp = tid >> 5;
    const long long r0 = (long long)blockIdx.x * kNormRows;
    const int n_steps = (C + kNormBoxes * kNormBoxCols - 1) / (kNormBoxes * kNormBoxCols);
    if (tid == 0) {
        for (int s = 0; s < kNormStages; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), kNormRows);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    int issued = 0;
    if (warp == 4) {
        if ((tid & 31) == 0) {
            tma_prefetch_desc(&tmX);
            for (int st = 0; st < n_steps; ++st) {
                const int s = st % kNormStages;
                if (st >= kNormStages &&
                    !wait_bounded(bar_empty(s), ((st / kNormStages) - 1) & 1, abort_flag, wait_limit))
                    break;
                mbar_arrive_expect_tx(bar_full(s), kNormStageBytes);
                for (int bx = 0; bx < kNormBoxes; ++bx)
                    tma_load_2d(base + s * kNormStageBytes + bx * (kNormRows * 128), &tmX, bar_full(s),
                                (st * kNormBoxes + bx) * kNormBoxCols, (int)r0);
                issued = st + 1;
            }
        }
    } else {
        const int r = tid;  // row of the tile
        const long long row = r0 + r;
        double s = 0.0;
        bool ok = true;
        for (int st = 0; st < n_steps; ++st) {
            const int sidx = st % kNormStages;
            if (!wait_bounded(bar_full(sidx), (st / kNormStages) & 1, abort_flag, wait_limit)) {
                ok = false;
                break;
            }
            const unsigned char* tile = sm + sidx * kNormStageBytes;
#pragma unroll
            for (int bx = 0; bx < kNormBoxes; ++bx) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 v = *reinterpret_cast<const uint4*>(tile + bx * (kNormRows * 128) + r * 128 +
                                                                    ((j ^ (r & 7)) << 4));
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const double lo = (double)__uint_as_float(w[e] << 16);
                        const double hi = (double)__uint_as_float(w[e] & 0xFFFF0000u);
                        s = __fma_rn(lo, lo, s);
                        s = __fma_rn(hi, hi, s);
                    }
                }
            }
            mbar_arrive(bar_empty(sidx));
        }
        if (ok && row < rows) {
            const int b = (int)(row / N), n = (int)(row % N);
            const int L = valid_len ? valid_len[b] : N;
            norm2[row] = n < L ? s : 0.0;
        }
    }
    __syncthreads();
    if (*abort_flag && warp == 4 && (tid & 31) == 0) {
        // let this CTA's own copies land before it exits
        for (int st = issued > kNormStages ? issued - kNormStages : 0; st < issued; ++st) {
            const long long t0 = clock64();
            while (!mbar_try_wait(bar_full(st % kNormStages), (st / kNormStages) & 1) &&
                   (uint64_t)(clock64() - t0) < (1ull << 32)) {
            }
        }
    }
}

// Block-wide exclusive scan of one int per thread (blockDim.x = 1024).  Returns the
// exclusive prefix; *total receives the block sum.  scratch: 33 ints of shared memory.
__device__ __forceinline__ int block_scan_1024(int v, int* scratch, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += u;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int t = scratch[lane];
        int ti = t;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, ti, off);
            if (lane >= off) ti += u;
        }
        scratch[lane] = ti - t;            // exclusive prefix of warp totals
        if (lane == 31) scratch[32] = ti;  // block total
    }
    __syncthreads();
    const int excl = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return excl;
}

// One CTA of 1024 threads per sample b: keep the k = keep_tokens(L_b, ratio) tokens of
// largest norm2 (ties to the lower index), idx[b][0..k) ascending, then -1 up to
// Npad_out; valid_out[b] = k.
//   1. the sample's smallest and largest squared norm;
//   2. a kSelBuckets-bucket histogram between them; bucketing is monotone, so the k-th
//      largest value tau lies in the bucket b* where the count from the top reaches k;
//   3. tau exactly: a radix select (8-bit digits of the fp64 bits, which order
//      non-negative values) over the members of b* only, gathered into shared memory;
//      when b* holds more than kSelGather tokens (many equal norms), over the whole
//      sample instead;
//   4. an in-order compaction by block scans: every value above tau, and the first
//      values equal to it, as many as the selection needs.
constexpr int kSelBuckets = 2048;
constexpr int kSelGather = 1024;

// Block-wide (1024 threads) k-th largest of the 64-bit keys key_of(i), i < n, among
// those with pred(i); returns tau and, in *remaining, how many keys equal to tau the
// k largest include.  hist: 256 words of shared memory.
template <typename KeyOf>
__device__ uint64_t block_radix_select(int n, uint32_t k, uint32_t* hist, uint32_t* sel, KeyOf key_of,
                                       uint32_t* remaining_out) {
    const int tid = threadIdx.x, lane = tid & 31;
    uint64_t prefix = 0, mask = 0;
    uint32_t remaining = k;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += 1024) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += 1024) {
            const uint64_t x = key_of(i);
            if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // lane l holds bins 255 - 8l - e (e = 0..7), highest first
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                c[e] = hist[255 - (8 * lane + e)];
                tot += c[e];
            }
            uint32_t incl = tot;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t u = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += u;
            }
            const uint32_t excl = incl - tot;
            const uint32_t ball = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
            const int src = ball ? __ffs(ball) - 1 : 31;
            if (lane == src) {
                uint32_t acc = excl;
                for (int e = 0; e < 8; ++e) {
                    if (acc + c[e] >= remaining) {
                        sel[0] = 255u - (8u * lane + e);
                        sel[1] = acc;
                        break;
                    }
                    acc += c[e];
                }
            }
        }
        __syncthreads();
        prefix |= (uint64_t)sel[0] << shift;
        mask |= 0xFFull << shift;
        remaining -= sel[1];
        __syncthreads();
    }
    *remaining_out = remaining;
    return prefix;
}

__global__ void __launch_bounds__(1024) prune_select_kernel(const double* __restrict__ norm2,
                                                            const int32_t* __restrict__ valid_len, int N,
                                                            double ratio, int Npad_out, int32_t* __restrict__ idx,
                                                            int32_t* __restrict__ valid_out) {
    __shared__ uint32_t bhist[kSelBuckets];
    __shared__ uint64_t gkey[kSelGather];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t sel[4];
    __shared__ double red[64];
    __shared__ int scan_scratch[33];
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    int L = valid_len ? valid_len[b] : N;
    if (L < 0 || L > N) {  // outside the documented range: flag it, never read past the sample
        if (tid == 0) raise_device_error(kErrBadRouting);
        L = L < 0 ? 0 : N;
    }
    const int k = keep_tokens(L, ratio);
    const double* val = norm2 + (size_t)b * N;
    const uint64_t* key = reinterpret_cast<const uint64_t*>(val);  // >= +0: bits are ordered
    int32_t* out = idx + (size_t)b * Npad_out;

    uint64_t tau = 0;
    uint32_t remaining = 0;
    if (k > 0) {
        // ---- 1. range
        double lo = INFINITY, hi = -INFINITY;
        for (int n = tid; n < L; n += 1024) {
            lo = fmin(lo, val[n]);
            hi = fmax(hi, val[n]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        if (lane == 0) {
            red[wid] = lo;
            red[32 + wid] = hi;
        }
        __syncthreads();
        if (wid == 0) {
            lo = red[lane];
            hi = red[32 + lane];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, off));
                hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, off));
            }
            if (lane == 0) {
                red[0] = lo;
                red[1] = hi;
            }
        }
        __syncthreads();
        lo = red[0];
        hi = red[1];
        const double range = hi - lo;
        const double bscale = range > 0.0 ? kSelBuckets / range : 0.0;
        bool whole = !(range > 0.0 && bscale < 1e300);   // all equal: select over the whole sample
        int bstar = 0;
        uint32_t above = 0, members = 0;
        if (!whole) {
            // ---- 2. bucket histogram and the bucket holding tau
            auto bucket = [&](double x) { return max(0, min(kSelBuckets - 1, (int)((x - lo) * bscale))); };
            for (int i = tid; i < kSelBuckets; i += 1024) bhist[i] = 0u;
            __syncthreads();
            for (int n = tid; n < L; n += 1024) atomicAdd(&bhist[bucket(val[n])], 1u);
            __syncthreads();
            if (wid == 0) {
                // lane l holds buckets 2047 - 64l - e (e = 0..63), highest first
                uint32_t tot = 0;
                for (int e = 0; e < 64; ++e) tot += bhist[kSelBuckets - 1 - (64 * lane + e)];
                uint32_t incl = tot;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const uint32_t u = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += u;
                }
                const uint32_t excl = incl - tot;
                const uint32_t ball = __ballot_sync(0xffffffffu, excl < (uint32_t)k && (uint32_t)k <= incl);
                const int src = ball ? __ffs(ball) - 1 : 31;
                if (lane == src) {
                    uint32_t acc = excl;
                    for (int e = 0; e < 64; ++e) {
                        const int bk = kSelBuckets - 1 - (64 * lane + e);
                        if (acc + bhist[bk] >= (uint32_t)k) {
                            sel[0] = (uint32_t)bk;
                            sel[1] = acc;
                            sel[2] = bhist[bk];
                            break;
                        }
                        acc += bhist[bk];
                    }
                }
            }
            __syncthreads();
            bstar = (int)sel[0];
            above = sel[1];
            members = sel[2];
            __syncthreads();
            whole = members > (uint32_t)kSelGather;
            if (!whole) {
                // ---- 3. gather bucket b*'s keys (any order) and select among them
                if (tid == 0) sel[3] = 0u;
                __syncthreads();
                for (int n = tid; n < L; n += 1024)
                    if (bucket(val[n]) == bstar) gkey[atomicAdd(&sel[3], 1u)] = key[n];
                __syncthreads();
                tau = block_radix_select((int)members, (uint32_t)k - above, hist, sel,
                                         [&](int i) { return gkey[i]; }, &remaining);
            }
        }
        if (whole)
            tau = block_radix_select(L, (uint32_t)k, hist, sel, [&](int i) { return key[i]; }, &remaining);
    }
    // ---- 4. in-order compaction: keys above tau, and the first `remaining` keys equal to it
    int pos_base = 0, eq_base = 0;
    for (int n0 = 0; n0 < L; n0 += 1024) {
        const int n = n0 + tid;
        const uint64_t x = n < L ? key[n] : 0ull;
        const bool gt = n < L && k > 0 && x > tau;
        const bool eq = n < L && k > 0 && x == tau;
        int eq_tot;
        const int eq_rank = block_scan_1024(eq ? 1 : 0, scan_scratch, &eq_tot);
        const bool sel_ = gt || (eq && (uint32_t)(eq_base + eq_rank) < remaining);
        int sel_tot;
        const int pos = block_scan_1024(sel_ ? 1 : 0, scan_scratch, &sel_tot);
        if (sel_) out[pos_base + pos] = n;
        pos_base += sel_tot;
        eq_base += eq_tot;
    }
    for (int p = k + tid; p < Npad_out; p += 1024) out[p] = -1;
    if (tid == 0) {
        valid_out[b] = k;
        if (pos_base != k) raise_device_error(kErrBadRouting);
    }
}

// dst[bh][p][:] = src[bh][idx[b][p]][:] for p < valid_out[b], zero rows up to Npad_out.
// src: [B*H][N][row_bytes], dst: [B*H][Npad_out][row_bytes]; UNIT-byte copies
// (UNIT 16 or 4, dividing row_bytes).  blockIdx.y = bh, so the sample's kept count and
// index list are fixed per CTA and the unit arithmetic stays in 32 bits; each thread has
// four loads in flight before it stores.
template <int UNIT>
__global__ void __launch_bounds__(256) gather_rows_kernel(const unsigned char* __restrict__ src,
                                                          unsigned char* __restrict__ dst,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ valid_out, int H, int N,
                                                          int row_bytes, int Npad_out) {
    using T = typename std::conditional<UNIT == 16, uint4, uint32_t>::type;
    constexpr int kIn = 4;
    const int per_row = row_bytes / UNIT;
    const int bh = blockIdx.y, b = bh / H;
    const int kept = valid_out[b];
    const int units = Npad_out * per_row;
    const T* s = reinterpret_cast<const T*>(src + (size_t)bh * N * row_bytes);
    T* d = reinterpret_cast<T*>(dst + (size_t)bh * Npad_out * row_bytes);
    const int32_t* ib = idx + (size_t)b * Npad_out;
    const int stride = gridDim.x * blockDim.x;
    for (int u0 = blockIdx.x * blockDim.x + threadIdx.x; u0 < units; u0 += kIn * stride) {
        T v[kIn];
#pragma unroll
        for (int i = 0; i < kIn; ++i) {
            const int u = u0 + i * stride;
            v[i] = T{};
            if (u < units) {
                const int p = u / per_row;
                if (p < kept) {
                    int n = ib[p];
                    if (n < 0 || n >= N) {
                        raise_device_error(kErrBadRouting);
                        n = 0;
                    }
                    v[i] = s[(size_t)n * per_row + (u - p * per_row)];
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kIn; ++i) {
            const int u = u0 + i * stride;
            if (u < units) d[u] = v[i];
        }
    }
}

}  // namespace sba

// select.cuh -- routing kernels: block pooling, block scoring and top-k selection.
//
// Routing as described on the page "MiniMax-H3 on 8xH200 benchmark"
// (news.paixiangai.cn), section "How SubBlock sparse attention works": per head,
// pool queries and keys over 64-token blocks, score every key block for every
// query block, keep the best-scoring key blocks (the `sparsity` fraction is
// dropped) and hand their indices to the attention kernel.  One-sub-block form:
//   qbar[I] = mean of the valid q rows of block I, kbar likewise,
//   score[I][J] = qbar[I] . kbar[J] / sqrt(D),
//   keep(n, s) = clamp(ceil((1 - s) n - 1e-9), 1, n) blocks, ties to the lower J.
//
// Exactness.  A block sum of 64 bf16 values is formed channel by channel in
// token order in fp64; the mean is one correctly rounded division.  Scores are
// first screened in fp32 (FFMA) with a proven bound delta on their error; only
// candidates within 2*delta of the fp32 k-th value are re-scored in fp64, with
// a fixed summation order and explicit round-to-nearest operations, and the
// selection among them is made on those fp64 values.  Everything above the
// band is kept, everything below is dropped.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace sba {

constexpr int kBlock = 64;

// Workspace layout of sba_pool_select (all offsets 256-byte aligned):
//   qmean64, kmean64 : double [BH][nB][D]
//   qmean32, kmean32 : float  [BH][nBc][D][64], nBc = ceil(nB / 64): block means
//                      rounded to fp32, transposed in chunks of 64 blocks so the
//                      scoring kernel stages them with straight copies
//   qnorm,   knorm   : double [BH][nB]    (Euclidean norm of each block mean)
struct SelectWorkspace {
    double* qmean64;
    double* kmean64;
    float* qmean32;
    float* kmean32;
    double* qnorm;
    double* knorm;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline size_t select_workspace_bytes(size_t BH, size_t nB, size_t D) {
    size_t m64 = align256(BH * nB * D * sizeof(double));
    size_t m32 = align256(BH * ((nB + 63) / 64) * 64 * D * sizeof(float));
    size_t nrm = align256(BH * nB * sizeof(double));
    return 2 * (m64 + m32 + nrm);
}

__host__ __device__ inline SelectWorkspace carve_select_workspace(void* base, size_t BH, size_t nB,
                                                                  size_t D) {
    char* p = static_cast<char*>(base);
    size_t m64 = align256(BH * nB * D * sizeof(double));
    size_t m32 = align256(BH * ((nB + 63) / 64) * 64 * D * sizeof(float));
    size_t nrm = align256(BH * nB * sizeof(double));
    SelectWorkspace w;
    w.qmean64 = reinterpret_cast<double*>(p); p += m64;
    w.kmean64 = reinterpret_cast<double*>(p); p += m64;
    w.qmean32 = reinterpret_cast<float*>(p); p += m32;
    w.kmean32 = reinterpret_cast<float*>(p); p += m32;
    w.qnorm = reinterpret_cast<double*>(p); p += nrm;
    w.knorm = reinterpret_cast<double*>(p);
    return w;
}

// keep(n, s) with the same fp64 operations, in the same order, as the host rule.
__host__ __device__ inline int keep_count(int n, double s) {
    if (n <= 0) return 0;
#ifdef __CUDA_ARCH__
    double x = ceil(__dadd_rn(__dmul_rn(__dadd_rn(1.0, -s), (double)n), -1e-9));
#else
    volatile double t = (1.0 - s) * (double)n;  // volatile: no fused multiply-add
    double x = ceil(t - 1e-9);
#endif
    if (x < 1.0) x = 1.0;
    if (x > (double)n) x = (double)n;
    return (int)x;
}

__device__ __forceinline__ int sample_len(const int32_t* valid_len, int b, int Npad) {
    return valid_len ? valid_len[b] : Npad;
}

// ------------------------------------------------------------------ pooling
// One group of D/8 lanes per (bh, block): lane g owns channels [8g, 8g+8) and
// walks the block's valid rows in token order, 16-byte loads, fp64 sums.
// Writes the fp64 mean and, when the pointers are non-null, its fp32 rounding
// (chunk-transposed layout) and the norm of the block mean.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ x,
                                                   const int32_t* __restrict__ valid_len, int H,
                                                   int Npad, double* __restrict__ mean64,
                                                   float* __restrict__ mean32,
                                                   double* __restrict__ norm, long long n_groups) {
    constexpr int LPB = D / 8;  // lanes per block group
    constexpr int UNROLL = 16;
    const int nB = Npad / kBlock;
    long long grp = (long long)blockIdx.x * (256 / LPB) + threadIdx.x / LPB;
    const int g = threadIdx.x % LPB;
    const bool active = grp < n_groups;
    if (!active) grp = n_groups - 1;  // keep the shuffles below warp-uniform
    const long long bh = grp / nB;
    const int I = (int)(grp % nB);
    const int b = (int)(bh / H);
    const int L = sample_len(valid_len, b, Npad);
    const int n0 = I * kBlock;
    int cnt = L - n0;
    cnt = cnt < 0 ? 0 : (cnt > kBlock ? kBlock : cnt);

    const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)bh * Npad + n0) * D) + g;
    double s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = 0.0;
    for (int n = 0; n < cnt; n += UNROLL) {
        uint4 buf[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
            if (n + u < cnt) buf[u] = __ldg(src + (size_t)(n + u) * LPB);
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            if (n + u < cnt) {
                const uint32_t w[4] = {buf[u].x, buf[u].y, buf[u].z, buf[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float lo = __uint_as_float(w[e] << 16);
                    float hi = __uint_as_float(w[e] & 0xFFFF0000u);
                    s[2 * e] = __dadd_rn(s[2 * e], (double)lo);
                    s[2 * e + 1] = __dadd_rn(s[2 * e + 1], (double)hi);
                }
            }
        }
    }
    double m[8];
    double sq = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        m[e] = cnt > 0 ? __ddiv_rn(s[e], (double)cnt) : 0.0;
        sq = fma(m[e], m[e], sq);
    }
#pragma unroll
    for (int off = LPB / 2; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (!active) return;
    double* dst64 = mean64 + (size_t)grp * D + 8 * g;
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        *reinterpret_cast<double2*>(dst64 + e) = make_double2(m[e], m[e + 1]);
    }
    if (mean32) {
        const int nBc = (nB + 63) / 64;
        float* dst32 = mean32 + (((size_t)bh * nBc + I / 64) * D + 8 * g) * 64 + (I % 64);
#pragma unroll
        for (int e = 0; e < 8; ++e) dst32[(size_t)e * 64] = (float)m[e];
    }
    if (norm && g == 0) norm[grp] = sqrt(sq);
}

// ------------------------------------------------------------------ scoring + top-k
__device__ __forceinline__ uint32_t f32_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_f32(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ uint64_t f64_key(double f) {
    uint64_t u = static_cast<uint64_t>(__double_as_longlong(f));
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// fp64 block score with one fixed operation order: s = 0; s += q_d * k_d for
// d = 0..D-1, each product and sum rounded to nearest; then s * (1/sqrt(D)).
// Adding +0.0 maps a -0.0 result to +0.0 so that equal values compare equal.
__device__ __forceinline__ double exact_score(const double* __restrict__ q,
                                              const double* __restrict__ k, int D, double inv) {
    double s = 0.0;
    for (int d = 0; d < D; ++d) s = __dadd_rn(s, __dmul_rn(q[d], k[d]));
    return __dadd_rn(__dmul_rn(s, inv), 0.0);
}

// Warp-cooperative radix select: the k-th largest (1-based) of the 32-bit keys
// key(j), j in [0, n), with `pred(j)` filtering the candidates.  8-bit digits,
// most significant first, 256-bin histogram in shared memory.
template <typename KeyOf>
__device__ uint32_t warp_radix_select32(int n, int k, uint32_t* hist, KeyOf key_of) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0;
    uint32_t remaining = (uint32_t)k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int j = lane; j < n; j += 32) {
            bool ok;
            uint32_t key = key_of(j, ok);
            if (ok && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            c[e] = hist[255 - (8 * lane + e)];
            tot += c[e];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const uint32_t excl = incl - tot;
        const uint32_t ball = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
        const int src = ball ? __ffs(ball) - 1 : 31;
        uint32_t digit = 0, above = 0;
        if (lane == src) {
            uint32_t acc = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (acc + c[e] >= remaining) {
                    digit = 255u - (8u * lane + e);
                    above = acc;
                    break;
                }
                acc += c[e];
            }
        }
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        prefix |= digit << shift;
        mask |= 0xFFu << shift;
        remaining -= above;
        __syncwarp();
    }
    return prefix;
}

// The same on 64-bit keys (8 passes), used only when the refinement band is wide.
template <typename KeyOf>
__device__ uint64_t warp_radix_select64(int n, int k, uint32_t* hist, KeyOf key_of) {
    const int lane = threadIdx.x & 31;
    uint64_t prefix = 0, mask = 0;
    uint32_t remaining = (uint32_t)k;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int j = lane; j < n; j += 32) {
            bool ok;
            uint64_t key = key_of(j, ok);
            if (ok && (key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            c[e] = hist[255 - (8 * lane + e)];
            tot += c[e];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const uint32_t excl = incl - tot;
        const uint32_t ball = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
        const int src = ball ? __ffs(ball) - 1 : 31;
        uint32_t digit = 0, above = 0;
        if (lane == src) {
            uint32_t acc = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (acc + c[e] >= remaining) {
                    digit = 255u - (8u * lane + e);
                    above = acc;
                    break;
                }
                acc += c[e];
            }
        }
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        prefix |= static_cast<uint64_t>(digit) << shift;
        mask |= 0xFFull << shift;
        remaining -= above;
        __syncwarp();
    }
    return prefix;
}

// Shared-memory bytes of score_select_kernel for a tile of TQ query blocks.
__host__ __device__ inline size_t score_select_smem(int D, int TQ, int nBmax) {
    const int nBpad = ((nBmax + 63) / 64) * 64;
    return (size_t)D * TQ * 4 + (size_t)D * 64 * 4 + (size_t)TQ * nBpad * 4 + 8 * 256 * 4 +
           8 * 32 * 4 + (size_t)TQ * 8 + 16;
}

// Scores and top-k routing for TQ (8, 16 or 32) consecutive query blocks of one
// (b, h) = blockIdx.y; 256 threads.  Phase 1 computes fp32 scores of all key
// blocks into shared memory (warp w owns rows 4w..4w+3, lane owns columns
// 2*lane, 2*lane+1 of each 64-block chunk).  Phase 2: one warp per row selects.
template <int D>
__global__ void __launch_bounds__(256) score_select_kernel(
    SelectWorkspace ws, const int32_t* __restrict__ valid_len, int H, int Npad, double sparsity,
    int kmax, int TQ, int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int nBmax = Npad / kBlock;
    const int nBc = (nBmax + 63) / 64;
    const int nBpad = nBc * 64;
    const int bh = blockIdx.y;
    const int b = bh / H;
    const int L = sample_len(valid_len, b, Npad);
    const int nB = (L + kBlock - 1) / kBlock;
    const int k = keep_count(nB, sparsity);
    const int I0 = blockIdx.x * TQ;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t* cnt_out = kv_cnt + (size_t)bh * nBmax;
    int32_t* idx_out = kv_idx + (size_t)bh * nBmax * kmax;

    int nrows = nBmax - I0;
    nrows = nrows > TQ ? TQ : nrows;
    int nact = nB - I0;  // rows with I < nB
    nact = nact < 0 ? 0 : (nact > nrows ? nrows : nact);
    for (int r = nact + tid; r < nrows; r += 256) cnt_out[I0 + r] = 0;
    if (nact == 0) return;
    if (k >= nB) {  // nothing dropped: every block, ascending
        for (int r = warp; r < nact; r += 8) {
            int32_t* out = idx_out + (size_t)(I0 + r) * kmax;
            for (int j = lane; j < nB; j += 32) out[j] = j;
            if (lane == 0) cnt_out[I0 + r] = nB;
        }
        return;
    }

    float* sq = reinterpret_cast<float*>(smem_raw);          // [D][TQ]
    float* sk = sq + D * TQ;                                  // [D][64]
    float* ssc = sk + D * 64;                                 // [TQ][nBpad]
    uint32_t* hist = reinterpret_cast<uint32_t*>(ssc + (size_t)TQ * nBpad);  // [8][256]
    int32_t* slots = reinterpret_cast<int32_t*>(hist + 8 * 256);             // [8][32]
    double* qn = reinterpret_cast<double*>(slots + 8 * 32);                  // [TQ]
    double* kmaxn = qn + TQ;                                                 // [1]

    // stage the fp32 query means of this tile: [D][TQ] from the [D][64] chunk layout
    const float* qsrc = ws.qmean32 + ((size_t)bh * nBc + I0 / 64) * D * 64 + (I0 % 64);
    for (int i = tid; i < D * TQ; i += 256) {
        const int d = i / TQ, r = i % TQ;
        sq[i] = qsrc[(size_t)d * 64 + r];
    }
    for (int r = tid; r < TQ; r += 256) qn[r] = r < nact ? ws.qnorm[(size_t)bh * nBmax + I0 + r] : 0.0;
    if (warp == 0) {  // largest key-block mean norm over the sample's blocks
        double m = 0.0;
        for (int j = lane; j < nB; j += 32) m = fmax(m, ws.knorm[(size_t)bh * nBmax + j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) *kmaxn = m;
    }

    // phase 1: fp32 scores, chunk by chunk of 64 key blocks
    const int nchunks = (nB + 63) / 64;
    const float* ksrc = ws.kmean32 + (size_t)bh * nBc * D * 64;
    for (int c = 0; c < nchunks; ++c) {
        __syncthreads();
        const float4* src4 = reinterpret_cast<const float4*>(ksrc + (size_t)c * D * 64);
        float4* dst4 = reinterpret_cast<float4*>(sk);
        for (int i = tid; i < D * 16; i += 256) dst4[i] = __ldg(src4 + i);
        __syncthreads();
        if (4 * warp < TQ) {
            float acc[4][2];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) {
                const float4 q4 = *reinterpret_cast<const float4*>(sq + d * TQ + 4 * warp);
                const float2 k2 = *reinterpret_cast<const float2*>(sk + d * 64 + 2 * lane);
                acc[0][0] = fmaf(q4.x, k2.x, acc[0][0]);
                acc[0][1] = fmaf(q4.x, k2.y, acc[0][1]);
                acc[1][0] = fmaf(q4.y, k2.x, acc[1][0]);
                acc[1][1] = fmaf(q4.y, k2.y, acc[1][1]);
                acc[2][0] = fmaf(q4.z, k2.x, acc[2][0]);
                acc[2][1] = fmaf(q4.z, k2.y, acc[2][1]);
                acc[3][0] = fmaf(q4.w, k2.x, acc[3][0]);
                acc[3][1] = fmaf(q4.w, k2.y, acc[3][1]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float2*>(ssc + (size_t)(4 * warp + i) * nBpad + c * 64 + 2 * lane) =
                    make_float2(acc[i][0], acc[i][1]);
        }
    }
    __syncthreads();

    // phase 2: per-row selection, one warp per row
    const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)D));
    uint32_t* whist = hist + warp * 256;
    int32_t* wslots = slots + warp * 32;
    for (int r = warp; r < nact; r += 8) {
        const int I = I0 + r;
        const float* row = ssc + (size_t)r * nBpad;
        const double* qrow64 = ws.qmean64 + ((size_t)bh * nBmax + I) * D;
        const double* kbase64 = ws.kmean64 + (size_t)bh * nBmax * D;
        int32_t* out = idx_out + (size_t)I * kmax;

        // k-th largest fp32 score
        const uint32_t tau_key = warp_radix_select32(nB, k, whist, [&](int j, bool& ok) {
            ok = true;
            return f32_key(row[j]);
        });
        const double tau = (double)key_to_f32(tau_key);
        // Error bound of an fp32 score against the fp64 one: D fused multiply-adds
        // plus the two fp32 roundings of the means give (D + 3) u sum|q_d k_d|
        // <= (D + 3) u |qbar| |kbar| (Cauchy-Schwarz), u = 2^-24; doubled for
        // margin, plus an absolute term for gradual underflow.
        const double delta = 2.0 * (D + 4) * 0x1p-24 * qn[r] * (*kmaxn) + D * 0x1p-126;
        const double hi = tau + 2.0 * delta, lo = tau - 2.0 * delta;

        int n_in = 0, n_band = 0;
        for (int j0 = 0; j0 < nB; j0 += 32) {
            const int j = j0 + lane;
            const double f = j < nB ? (double)row[j] : -INFINITY;
            const bool in_a = j < nB && f > hi;
            const bool in_b = j < nB && !in_a && f >= lo;
            n_in += __popc(__ballot_sync(0xffffffffu, in_a));
            n_band += __popc(__ballot_sync(0xffffffffu, in_b));
        }
        const int need = k - n_in;  // band members to keep, 1 <= need <= n_band

        // mode 0: keep the whole band; 1: small band ranked in registers; 2: wide band
        int mode = need >= n_band ? 0 : (n_band <= 32 ? 1 : 2);
        uint32_t chosen_mask = 0xffffffffu;
        uint64_t tau_x = 0;
        int eq_take = 0;
        if (mode == 1) {
            int base = 0;
            for (int j0 = 0; j0 < nB; j0 += 32) {
                const int j = j0 + lane;
                const double f = j < nB ? (double)row[j] : -INFINITY;
                const bool in_b = j < nB && !(f > hi) && f >= lo;
                const uint32_t bb = __ballot_sync(0xffffffffu, in_b);
                if (in_b) wslots[base + __popc(bb & lanemask_lt())] = j;
                base += __popc(bb);
            }
            __syncwarp();
            const int myj = lane < n_band ? wslots[lane] : 0;
            const double my_s = lane < n_band ? exact_score(qrow64, kbase64 + (size_t)myj * D, D, inv)
                                              : -INFINITY;
            int rank = 0;
            for (int t = 0; t < n_band; ++t) {
                const double s_t = __shfl_sync(0xffffffffu, my_s, t);
                const int j_t = __shfl_sync(0xffffffffu, myj, t);
                rank += (s_t > my_s || (s_t == my_s && j_t < myj)) ? 1 : 0;
            }
            chosen_mask = __ballot_sync(0xffffffffu, lane < n_band && rank < need);
            __syncwarp();
        } else if (mode == 2) {
            auto band_key = [&](int j, bool& ok) -> uint64_t {
                const double f = (double)row[j];
                ok = !(f > hi) && f >= lo;
                return ok ? f64_key(exact_score(qrow64, kbase64 + (size_t)j * D, D, inv)) : 0ull;
            };
            tau_x = warp_radix_select64(nB, need, whist, band_key);
            int gt = 0;
            for (int j0 = 0; j0 < nB; j0 += 32) {
                const int j = j0 + lane;
                bool ok = false;
                uint64_t x = 0;
                if (j < nB) x = band_key(j, ok);
                gt += __popc(__ballot_sync(0xffffffffu, ok && x > tau_x));
            }
            eq_take = need - gt;
        }

        // emit the kept blocks in ascending order
        int pos = 0, band_seen = 0, eq_seen = 0;
        for (int j0 = 0; j0 < nB; j0 += 32) {
            const int j = j0 + lane;
            const double f = j < nB ? (double)row[j] : -INFINITY;
            const bool in_a = j < nB && f > hi;
            const bool in_b = j < nB && !in_a && f >= lo;
            const uint32_t bb = __ballot_sync(0xffffffffu, in_b);
            bool sel = in_a;
            if (mode == 0) {
                sel = sel || in_b;
            } else if (mode == 1) {
                const int slot = band_seen + __popc(bb & lanemask_lt());
                sel = sel || (in_b && ((chosen_mask >> slot) & 1u));
            } else {
                uint64_t x = 0;
                if (in_b) x = f64_key(exact_score(qrow64, kbase64 + (size_t)j * D, D, inv));
                const bool eq = in_b && x == tau_x;
                const uint32_t eb = __ballot_sync(0xffffffffu, eq);
                const int eq_rank = eq_seen + __popc(eb & lanemask_lt());
                sel = sel || (in_b && x > tau_x) || (eq && eq_rank < eq_take);
                eq_seen += __popc(eb);
            }
            band_seen += __popc(bb);
            const uint32_t sb = __ballot_sync(0xffffffffu, sel);
            if (sel) out[pos + __popc(sb & lanemask_lt())] = j;
            pos += __popc(sb);
        }
        if (lane == 0) {
            cnt_out[I] = pos;
            if (pos != k) raise_device_error(kErrBadRouting);
        }
        __syncwarp();
    }
}

}  // namespace sba

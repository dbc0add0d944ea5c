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
// first screened on the tensor cores (select_fused_kernel: bf16 hi/lo splits of the
// means, fp32 accumulation in TMEM) with a proven bound delta on their error; only
// candidates within 2*delta of the screened k-th value are re-scored in fp64, and
// the selection among them is made on fp64 values computed with a fixed summation
// order and explicit round-to-nearest operations.  Everything above the band is
// kept, everything below is dropped.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace sba {

constexpr int kBlock = 64;

// Workspace layout of the routers (all offsets 256-byte aligned).  Means are
// pooled over 64-token blocks (nsub = 1) or over the nsub sub-blocks of each
// block (the log-sum-exp router, nsub = 4); nP = nB * nsub pooled rows:
//   qmean64, kmean64 : double [BH][nP][D]   pooled means
//   qhi, qlo, khi, klo : bf16 [BH][nP][D]   hi/lo split of the means for the screen
//   qnorm, knorm     : double [BH][nP]      Euclidean norm of each mean
//   kmaxn            : double [BH]          largest key-mean norm of the sample
//   scores           : float [BH][nB][ld]   screened block scores, ld = 64 * ceil(nB / 64)
//   ovf_count, ovf_rows : int32 [1], [BH * nB]  rows left by the fused screen
//   finish           : [BH * nB] records of fused_row_bytes(nB) bytes (fused screen)
struct SelectWorkspace {
    double* qmean64;
    double* kmean64;
    __nv_bfloat16* qhi;
    __nv_bfloat16* qlo;
    __nv_bfloat16* khi;
    __nv_bfloat16* klo;
    double* qnorm;
    double* knorm;
    double* kmaxn;
    float* scores;
    int32_t* ovf_count;     // rows the fused screen hands to topk_rest_kernel
    int32_t* ovf_rows;      // [BH * nB]
    unsigned char* finish;  // [BH * nB] records of fused_row_bytes(nB): the fused screen's
                            // per-row result for select_finish_kernel
    int ld;
    int fstride;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline size_t select_score_ld(size_t nB) { return (nB + 63) / 64 * 64; }

// The fused screen's per-row record: a 32-byte header, kFusedList window entries
// (value, block) of 8 bytes, and the keep mask, four words per 128 key blocks.
constexpr int kFusedList = 56;
__host__ __device__ inline size_t fused_row_bytes(size_t nB) { return 32 + 8 * kFusedList + 16 * ((nB + 127) / 128); }

__host__ __device__ inline size_t select_workspace_bytes(size_t BH, size_t nB, size_t D, size_t nsub = 1) {
    const size_t nP = nB * nsub;
    const size_t m64 = align256(BH * nP * D * sizeof(double));
    const size_t m16 = align256(BH * nP * D * 2);
    const size_t nrm = align256(BH * nP * sizeof(double));
    const size_t kmx = align256(BH * sizeof(double));
    const size_t sco = align256(BH * nB * select_score_ld(nB) * sizeof(float));
    const size_t ovf = 256 + align256(BH * nB * sizeof(int32_t));
    const size_t fin = align256(BH * nB * fused_row_bytes(nB));
    return 2 * m64 + 4 * m16 + 2 * nrm + kmx + sco + ovf + fin;
}

__host__ __device__ inline SelectWorkspace carve_select_workspace(void* base, size_t BH, size_t nB,
                                                                  size_t D, size_t nsub = 1) {
    char* p = static_cast<char*>(base);
    const size_t nP = nB * nsub;
    const size_t m64 = align256(BH * nP * D * sizeof(double));
    const size_t m16 = align256(BH * nP * D * 2);
    const size_t nrm = align256(BH * nP * sizeof(double));
    const size_t kmx = align256(BH * sizeof(double));
    SelectWorkspace w;
    w.qmean64 = reinterpret_cast<double*>(p); p += m64;
    w.kmean64 = reinterpret_cast<double*>(p); p += m64;
    w.qhi = reinterpret_cast<__nv_bfloat16*>(p); p += m16;
    w.qlo = reinterpret_cast<__nv_bfloat16*>(p); p += m16;
    w.khi = reinterpret_cast<__nv_bfloat16*>(p); p += m16;
    w.klo = reinterpret_cast<__nv_bfloat16*>(p); p += m16;
    w.qnorm = reinterpret_cast<double*>(p); p += nrm;
    w.knorm = reinterpret_cast<double*>(p); p += nrm;
    w.kmaxn = reinterpret_cast<double*>(p); p += kmx;
    w.scores = reinterpret_cast<float*>(p);
    w.ld = (int)select_score_ld(nB);
    p += align256(BH * nB * (size_t)w.ld * sizeof(float));
    w.ovf_count = reinterpret_cast<int32_t*>(p);
    w.ovf_rows = reinterpret_cast<int32_t*>(p + 256);
    p += 256 + align256(BH * nB * sizeof(int32_t));
    w.finish = reinterpret_cast<unsigned char*>(p);
    w.fstride = (int)fused_row_bytes(nB);
    return w;
}

// The log-sum-exp router splits each 64-token block into kNsub sub-blocks.
constexpr int kNsub = 4;
constexpr int kSubBlock = kBlock / kNsub;

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

// keep(n, s) rounded up to a multiple of `budget` blocks, at most n.
__host__ __device__ inline int keep_count_budget(int n, double s, int budget) {
    int k = keep_count(n, s);
    if (budget > 1) {
        k = (k + budget - 1) / budget * budget;
        if (k > n) k = n;
    }
    return k;
}

__device__ __forceinline__ int sample_len(const int32_t* valid_len, int b, int Npad) {
    return valid_len ? valid_len[b] : Npad;
}

// ------------------------------------------------------------------ pooling
// One group of D/8 lanes per (bh, block): lane g owns channels [8g, 8g+8) and
// walks the block's valid rows in token order, 16-byte loads, fp64 sums.
// Writes the fp64 mean and, when the pointers are non-null, its bf16 hi/lo split
// and the norm of the block mean.  BLK is the pooling granularity: 64-token
// blocks, or the 16-token sub-blocks of the log-sum-exp router.  The fp64 means of
// the kBlock / BLK sub-blocks of a block are interleaved channel by channel,
// [..][block][D][kBlock / BLK], so that the lanes re-scoring the sub-block pairs of
// a block read adjacent words; hi/lo and the norms stay one row per pooled row.
// The second tensor, pooled by CTAs blockIdx.x >= blocks0 of the same launch (the
// router's Q and K in one grid); blocks0 = gridDim.x: one tensor.
struct PoolSecond {
    const __nv_bfloat16* x;
    double* mean64;
    __nv_bfloat16* hi16;
    __nv_bfloat16* lo16;
    double* norm;
    unsigned blocks0;
};

template <int D, int BLK = kBlock>
__global__ void __launch_bounds__(256, 4) pool_kernel(const __nv_bfloat16* __restrict__ x,
                                                   const int32_t* __restrict__ valid_len, int H,
                                                   int Npad, double* __restrict__ mean64,
                                                   __nv_bfloat16* __restrict__ hi16,
                                                   __nv_bfloat16* __restrict__ lo16,
                                                   double* __restrict__ norm, long long n_groups,
                                                   PoolSecond second) {
    constexpr int LPB = D / 8;  // lanes per block group
    constexpr int UNROLL = 8;   // with four CTAs per SM: more rows in flight per SM than 16 with two
    const int nB = Npad / BLK;
    unsigned bid = blockIdx.x;
    if (bid >= second.blocks0) {
        bid -= second.blocks0;
        x = second.x;
        mean64 = second.mean64;
        hi16 = second.hi16;
        lo16 = second.lo16;
        norm = second.norm;
    }
    long long grp = (long long)bid * (256 / LPB) + threadIdx.x / LPB;
    const int g = threadIdx.x % LPB;
    const bool active = grp < n_groups;
    if (!active) grp = n_groups - 1;  // keep the shuffles below warp-uniform
    const long long bh = grp / nB;
    const int I = (int)(grp % nB);
    const int b = (int)(bh / H);
    const int L = sample_len(valid_len, b, Npad);
    const int n0 = I * BLK;
    int cnt = L - n0;
    cnt = cnt < 0 ? 0 : (cnt > BLK ? BLK : cnt);

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
    if constexpr (BLK == kBlock) {
        double* dst64 = mean64 + (size_t)grp * D + 8 * g;
#pragma unroll
        for (int e = 0; e < 8; e += 2) *reinterpret_cast<double2*>(dst64 + e) = make_double2(m[e], m[e + 1]);
    } else {
        constexpr int NS = kBlock / BLK;
        const long long blk = grp / NS;
        const int a = (int)(grp % NS);
        double* dst64 = mean64 + ((size_t)blk * D + 8 * g) * NS + a;
#pragma unroll
        for (int e = 0; e < 8; ++e) dst64[(size_t)e * NS] = m[e];
    }
    if (hi16) {
        // hi = bf16(mean), lo = bf16(mean - hi): the split the tensor-core screen uses
        uint32_t ph[4], pl[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn((float)m[e]);
            const __nv_bfloat16 h1 = __float2bfloat16_rn((float)m[e + 1]);
            const __nv_bfloat16 l0 = __float2bfloat16_rn((float)(m[e] - (double)__bfloat162float(h0)));
            const __nv_bfloat16 l1 = __float2bfloat16_rn((float)(m[e + 1] - (double)__bfloat162float(h1)));
            __nv_bfloat162 hh = __halves2bfloat162(h0, h1), ll = __halves2bfloat162(l0, l1);
            ph[e / 2] = *reinterpret_cast<uint32_t*>(&hh);
            pl[e / 2] = *reinterpret_cast<uint32_t*>(&ll);
        }
        *reinterpret_cast<uint4*>(hi16 + (size_t)grp * D + 8 * g) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
        *reinterpret_cast<uint4*>(lo16 + (size_t)grp * D + 8 * g) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
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
#pragma unroll 4
    for (int d = 0; d < D; ++d) s = __dadd_rn(s, __dmul_rn(q[d], k[d]));
    return __dadd_rn(__dmul_rn(s, inv), 0.0);
}

// fp64 log-sum-exp block score of query block I against key block J, in the same
// operation order as the definition it restates: for every pair (a, c) of
// non-empty sub-blocks, a-major,
//   x = ((qbar_a . kbar_c) * inv + log(n_a)) + log(n_c)
// with the dot product summed over d in order, each step rounded to nearest; then
// m = max x, z = sum over the pairs (same order) of exp(x - m), score = m + log z.
// q4, k4: the fp64 sub-block means of the two blocks, [D][NSUB] (sub-block innermost).
template <int NSUB>
__device__ double exact_lse(const double* __restrict__ q4, const double* __restrict__ k4, int D, int L,
                            int I, int J, double inv) {
    // Only the wide-band fallback calls this (one lane per block), so the loops stay
    // rolled: the 16 logits live in local memory rather than in registers.
    constexpr int SUB = kBlock / NSUB;
    double x[NSUB * NSUB];
    double m = -INFINITY;
#pragma unroll 1
    for (int p = 0; p < NSUB * NSUB; ++p) {
        const int a = p / NSUB, c = p % NSUB;
        int na = L - (I * NSUB + a) * SUB;
        na = na < 0 ? 0 : (na > SUB ? SUB : na);
        int nc = L - (J * NSUB + c) * SUB;
        nc = nc < 0 ? 0 : (nc > SUB ? SUB : nc);
        x[p] = -INFINITY;  // empty pair: no term
        if (na > 0 && nc > 0) {
            double s = 0.0;
#pragma unroll 4
            for (int d = 0; d < D; ++d) s = __dadd_rn(s, __dmul_rn(q4[d * NSUB + a], k4[d * NSUB + c]));
            const double xv = __dadd_rn(__dadd_rn(__dmul_rn(s, inv), log((double)na)), log((double)nc));
            x[p] = xv;
            m = xv > m ? xv : m;
        }
    }
    double z = 0.0;
#pragma unroll 1
    for (int t = 0; t < NSUB * NSUB; ++t)
        if (x[t] != -INFINITY) z = __dadd_rn(z, exp(__dadd_rn(x[t], -m)));
    return __dadd_rn(__dadd_rn(m, log(z)), 0.0);
}

// fp64 log-sum-exp scores of the n_band (<= kBandCache) key blocks listed in
// `slots` for query block I (4 sub-blocks per block), one block at a time by the
// whole warp.  For each half of the 16 sub-block pairs (query sub-blocks 2h, 2h + 1),
// lane l forms partial dot products over channels l, l + 32, .. (fp64 fused
// multiply-adds) and a transposing butterfly leaves the 4 lanes with equal bits
// 4..2 one pair's dot product; then the max, the exponentials and their sum go over
// the 16 pairs.  Same definition as exact_lse, evaluated in another order: values
// agree with it to a few fp64 roundings.  q4, k4: sub-block means [D][4].  Writes
// out[t], t < n_band.
template <int D>
__device__ void band_lse_warp(const double* __restrict__ q4, const double* __restrict__ kbase, int L, int I,
                              double inv, const int32_t* slots, int n_band, double* out) {
    constexpr int NSUB = 4, SUB = kBlock / NSUB, CPL = D / 32;  // channels per lane
    const int lane = threadIdx.x & 31;
    // pair within a half held after the butterfly: bits 4, 3, 2 of the lane index
    const int ph = 4 * ((lane >> 4) & 1) + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);
    const int c = ph & 3;
    double lna[2];
    bool va[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int a = 2 * h + (ph >> 2);
        int na = L - (I * NSUB + a) * SUB;
        na = na < 0 ? 0 : (na > SUB ? SUB : na);
        va[h] = na > 0;
        lna[h] = na > 0 ? log((double)na) : 0.0;
    }
    for (int t = 0; t < n_band; ++t) {
        const int J = slots[t];
        const double* k4 = kbase + (size_t)J * NSUB * D;
        int nc = L - (J * NSUB + c) * SUB;
        nc = nc < 0 ? 0 : (nc > SUB ? SUB : nc);
        const double lnc = nc > 0 ? log((double)nc) : 0.0;
        double x[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            double p[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) p[e] = 0.0;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const size_t d = (size_t)(lane + 32 * i) * NSUB;
                const double2 qq = *reinterpret_cast<const double2*>(q4 + d + 2 * h);
                const double2 u = *reinterpret_cast<const double2*>(k4 + d);
                const double2 w = *reinterpret_cast<const double2*>(k4 + d + 2);
                const double kv[4] = {u.x, u.y, w.x, w.y};
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    p[cc] = fma(qq.x, kv[cc], p[cc]);
                    p[4 + cc] = fma(qq.y, kv[cc], p[4 + cc]);
                }
            }
            double h4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool up = (lane >> 4) & 1;
                h4[e] = (up ? p[4 + e] : p[e]) + __shfl_xor_sync(0xffffffffu, up ? p[e] : p[4 + e], 16);
            }
            double h2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool up = (lane >> 3) & 1;
                h2[e] = (up ? h4[2 + e] : h4[e]) + __shfl_xor_sync(0xffffffffu, up ? h4[e] : h4[2 + e], 8);
            }
            const bool up2 = (lane >> 2) & 1;
            double dot = (up2 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, up2 ? h2[0] : h2[1], 4);
            dot += __shfl_xor_sync(0xffffffffu, dot, 2);
            dot += __shfl_xor_sync(0xffffffffu, dot, 1);
            x[h] = (va[h] && nc > 0) ? dot * inv + lna[h] + lnc : -INFINITY;
        }
        double m = fmax(x[0], x[1]);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
        double z = (x[0] != -INFINITY ? exp(x[0] - m) : 0.0) + (x[1] != -INFINITY ? exp(x[1] - m) : 0.0);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
        if (lane == 0) out[t] = m + log(z);
    }
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

// Largest key-mean norm of each (b, h) over its sample's pooled rows (blocks of
// `blk` tokens); one warp each.
__global__ void kmax_kernel(SelectWorkspace ws, const int32_t* __restrict__ valid_len, int H, int Npad,
                            int BH, int blk) {
    const int bh = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && threadIdx.x == 0) *ws.ovf_count = 0;  // the fused screen counts from here
    if (bh >= BH) return;
    const int nBmax = Npad / blk;
    const int nB = (sample_len(valid_len, bh / H, Npad) + blk - 1) / blk;
    double m = 0.0;
    for (int j = lane; j < nB; j += 32) m = fmax(m, ws.knorm[(size_t)bh * nBmax + j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) ws.kmaxn[bh] = m;
}

// Band members whose exact scores are cached (and ranked) in shared memory; a wider
// band falls back to a radix select that re-evaluates them.
constexpr int kBandCache = 64;

// Shared-memory bytes of one top-k warp: the screened row, a 256-bin histogram,
// the band's block indices and their exact scores.
__host__ __device__ inline size_t topk_warp_smem(int ld) {
    return (size_t)ld * 4 + 256 * 4 + kBandCache * 4 + kBandCache * 8;
}

// Shared-memory bytes of topk_kernel for `warps` warps per CTA.
__host__ __device__ inline size_t topk_smem(int warps, int ld) { return (size_t)warps * topk_warp_smem(ld); }

// Top-k routing of one (b, h, I) row per warp, from the screened scores.
//
// Screen error.  The scores come from select_fused_kernel: S = qhi.khi + qhi.klo +
// qlo.khi in fp32, with hi = bf16(x), lo = bf16(x - hi) (each through fp32).  Per
// term d the dropped parts (qlo.klo and the remainders of the split) are below
// 4 * 2^-16 |qbar_d kbar_d|; the products are exact in fp32 and the accumulation
// of the 3D products in fp32 adds at most 3D * 2^-22 of sum |qbar_d kbar_d| (two
// units in the last place per addition, whatever the order).  With Cauchy-Schwarz,
// |S - qbar.kbar| <= (4 * 2^-16 + 3D * 2^-22) |qbar_I| max_J |kbar_J|, doubled here
// for margin, plus an absolute term for values in the subnormal range.  (The fused
// screen accumulates all 3D products in one fp32 TMEM accumulator, which is the case
// this bound covers.)
//
// Log-sum-exp router (NSUB = 4).  The screen (score_lse_kernel) forms every
// sub-block logit in log2 units, y' = fp32(acc * fp32(log2(e) / sqrt(D))), where acc
// accumulates in fp32 first the 2D cross products hi.lo and lo.hi (each below
// 2^-8 |qbar_d kbar_d|), then the D products hi.hi.  Per logit, relative to
// R_ac = |qbar_a| |kbar_c| / sqrt(D), the error of x' = y' ln 2 is at most
//   dropped split terms              4 * 2^-16
//   hi.hi accumulation               1.02 D * 2^-22  (two ulps per addition of a
//                                    partial sum below 1.02 sum_d |qbar_d kbar_d|)
//   cross accumulation               1.01 D * 2^-28
//   scale constant and product       2 * 2^-24
// so |x' - x| <= (4 * 2^-16 + (D + 2) * 2^-22 + D * 2^-27) R, R = max_a |qbar_a| *
// max_c |kbar_c| / sqrt(D), plus the subnormal term.  The log-sum-exp is
// 1-Lipschitz in the largest logit error, so the block score inherits the bound.
// Its fp32 evaluation adds at most 2^-20 R + 2^-17: the max is exact; each gap to
// the max (one rounding of a value below 3R) moves its exponential by at most a
// relative 2^-21 R; ex2.approx is taken as accurate to 2^-20 relative; the
// count-weighted sum of at most 16 terms (at least 1, the term of the max) to
// 2^-19; log2 of a value below 4097 to two ulps; the last add and the product by
// ln 2 to 2^-23 (R + 12).  The total is multiplied by 1.25 for margin.
// One routing row `rid` = (bh, I) by one warp; `wsm` is the warp's topk_warp_smem bytes.
template <int D, int NSUB>
__device__ void topk_row(const SelectWorkspace& ws, const int32_t* __restrict__ valid_len, int H, int Npad,
                         double sparsity, int budget, int kmax, int32_t* __restrict__ kv_idx,
                         int32_t* __restrict__ kv_cnt, long long rid, unsigned char* wsm) {
    const int lane = threadIdx.x & 31;
    const int nBmax = Npad / kBlock;
    const int ld = ws.ld;
    const long long bh = rid / nBmax;
    const int I = (int)(rid % nBmax);
    const int L = sample_len(valid_len, (int)(bh / H), Npad);
    const int nB = (L + kBlock - 1) / kBlock;
    const int k = keep_count_budget(nB, sparsity, budget);
    int32_t* out = kv_idx + (size_t)rid * kmax;
    if (I >= nB) {
        if (lane == 0) kv_cnt[rid] = 0;
        return;
    }
    if (k >= nB) {  // nothing dropped: every block, ascending
        for (int j = lane; j < nB; j += 32) out[j] = j;
        if (lane == 0) kv_cnt[rid] = nB;
        return;
    }
    float* row = reinterpret_cast<float*>(wsm);
    uint32_t* whist = reinterpret_cast<uint32_t*>(row + ld);
    int32_t* wslots = reinterpret_cast<int32_t*>(whist + 256);
    double* bx = reinterpret_cast<double*>(wslots + kBandCache);  // 8-byte aligned: ld % 64 == 0
    float* bval = reinterpret_cast<float*>(bx);                    // bucket members' values (before bx is used)

    // ---- the screened row, with its smallest and largest value
    const float* src = ws.scores + (size_t)rid * ld;
    float vmin = INFINITY, vmax = -INFINITY;
    for (int j = lane; j < nB; j += 32) {
        const float f = __ldg(src + j);
        row[j] = f;
        vmin = fminf(vmin, f);
        vmax = fmaxf(vmax, f);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, off));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, off));
    }
    __syncwarp();

    // ---- tau = the k-th largest screened value.  A 256-bucket histogram between the
    // row's min and max finds the bucket holding it; when that bucket has at most
    // kBandCache members they are ranked directly, otherwise a radix select over
    // all the values decides.  Both give the same value.
    float tau = 0.f;
    bool have_tau = false;
    const float range = vmax - vmin;
    const float bscale = 256.0f / range;
    if (range > 0.f && range <= 3.0e38f && bscale <= 3.0e38f) {
        auto bucket = [&](float f) { return min(255, (int)((f - vmin) * bscale)); };
        for (int i = lane; i < 256; i += 32) whist[i] = 0u;
        __syncwarp();
        for (int j = lane; j < nB; j += 32) atomicAdd(&whist[bucket(row[j])], 1u);
        __syncwarp();
        // lane l holds buckets 255 - 8l - e (e = 0..7), highest first
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            c[e] = whist[255 - (8 * lane + e)];
            tot += c[e];
        }
        uint32_t incl = tot;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        const uint32_t excl = incl - tot;
        const uint32_t ball = __ballot_sync(0xffffffffu, excl < (uint32_t)k && (uint32_t)k <= incl);
        const int src_lane = ball ? __ffs(ball) - 1 : 31;
        int bstar = 0;
        uint32_t above = 0, bcount = 0;
        if (lane == src_lane) {
            uint32_t acc = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (acc + c[e] >= (uint32_t)k) {
                    bstar = 255 - (8 * lane + e);
                    above = acc;
                    bcount = c[e];
                    break;
                }
                acc += c[e];
            }
        }
        bstar = __shfl_sync(0xffffffffu, bstar, src_lane);
        above = __shfl_sync(0xffffffffu, above, src_lane);
        bcount = __shfl_sync(0xffffffffu, bcount, src_lane);
        if (bcount >= 1 && bcount <= (uint32_t)kBandCache) {
            // the bucket's values, then the (k - above)-th largest of them
            int base = 0;
            for (int j0 = 0; j0 < nB; j0 += 32) {
                const int j = j0 + lane;
                const bool in = j < nB && bucket(row[j]) == bstar;
                const uint32_t bb = __ballot_sync(0xffffffffu, in);
                if (in) bval[base + __popc(bb & lanemask_lt())] = row[j];
                base += __popc(bb);
            }
            __syncwarp();
            const int kk = k - (int)above;  // 1 <= kk <= bcount
            bool hit = false;
            float hv = 0.f;
            for (int t = lane; t < (int)bcount; t += 32) {
                const float vt = bval[t];
                int gt = 0, ge = 0;
                for (int u = 0; u < (int)bcount; ++u) {
                    const float vu = bval[u];
                    gt += vu > vt ? 1 : 0;
                    ge += vu >= vt ? 1 : 0;
                }
                if (gt < kk && kk <= ge) {
                    hit = true;
                    hv = vt;
                }
            }
            const uint32_t hb = __ballot_sync(0xffffffffu, hit);
            if (hb) {
                tau = __shfl_sync(0xffffffffu, hv, __ffs(hb) - 1);
                have_tau = true;
            }
            __syncwarp();
        }
    }
    if (!have_tau) {
        const uint32_t tau_key = warp_radix_select32(nB, k, whist, [&](int j, bool& ok) {
            ok = true;
            return f32_key(row[j]);
        });
        tau = key_to_f32(tau_key);
    }

    const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)D));
    const size_t prow = (size_t)bh * nBmax * NSUB + (size_t)I * NSUB;  // first pooled row of block I
    double qn = ws.qnorm[prow];
#pragma unroll
    for (int a = 1; a < NSUB; ++a) qn = fmax(qn, ws.qnorm[prow + a]);
    const double kmx = ws.kmaxn[bh];
    const double* qrow64 = ws.qmean64 + prow * D;
    const double* kbase64 = ws.kmean64 + (size_t)bh * nBmax * NSUB * D;
    auto exact = [&](int j) -> double {
        if constexpr (NSUB == 1)
            return exact_score(qrow64, kbase64 + (size_t)j * D, D, inv);
        else
            return exact_lse<NSUB>(qrow64, kbase64 + (size_t)j * NSUB * D, D, L, I, j, inv);
    };

    // screen error bound (see above); everything above the band [tau - 2 delta,
    // tau + 2 delta] is kept, everything below dropped, the band decided in fp64.
    // The edges are rounded outwards to fp32 so that the tests run in fp32; that can
    // only move values into the band.
    double delta;
    if constexpr (NSUB == 1)
        delta = 2.0 * (4.0 * 0x1p-16 + 3.0 * D * 0x1p-22) * qn * kmx + 3.0 * D * 0x1p-120 * (1.0 + qn + kmx);
    else
        delta = 1.25 * ((4.0 * 0x1p-16 + (D + 2.0) * 0x1p-22 + D * 0x1p-27 + 0x1p-20) * qn * kmx * inv +
                        3.0 * D * 0x1p-120 * (1.0 + qn + kmx) + 0x1p-17);
    const float hi = __double2float_ru((double)tau + 2.0 * delta);
    const float lo = __double2float_rd((double)tau - 2.0 * delta);

    // ---- classify: count the sure keeps, list the band (its first kBandCache members)
    int n_in = 0, n_band = 0;
    for (int j0 = 0; j0 < nB; j0 += 32) {
        const int j = j0 + lane;
        const float f = j < nB ? row[j] : -INFINITY;
        const bool in_a = j < nB && f > hi;
        const bool in_b = j < nB && !in_a && f >= lo;
        n_in += __popc(__ballot_sync(0xffffffffu, in_a));
        const uint32_t bb = __ballot_sync(0xffffffffu, in_b);
        const int slot = n_band + __popc(bb & lanemask_lt());
        if (in_b && slot < kBandCache) wslots[slot] = j;
        n_band += __popc(bb);
    }
    const int need = k - n_in;  // band members to keep, 1 <= need <= n_band
    __syncwarp();

    // mode 0: keep the whole band; 1: band of at most kBandCache, exact scores cached
    // and ranked in shared memory; 2: wide band, radix select
    const int mode = need >= n_band ? 0 : (n_band <= kBandCache ? 1 : 2);
    uint64_t chosen_mask = ~0ull;
    uint64_t tau_x = 0;
    int eq_take = 0;
    if (mode == 1) {
        if constexpr (NSUB == 1) {
            for (int t = lane; t < n_band; t += 32) bx[t] = exact(wslots[t]);
        } else {
            band_lse_warp<D>(qrow64, kbase64, L, I, inv, wslots, n_band, bx);
        }
        __syncwarp();
        // rank of each member: members with a higher exact score, or an equal one
        // and a lower block index, come first
        bool pick[kBandCache / 32];
#pragma unroll
        for (int h = 0; h < kBandCache / 32; ++h) {
            const int t = lane + 32 * h;
            pick[h] = false;
            if (t < n_band) {
                const double st = bx[t];
                const int jt = wslots[t];
                int rank = 0;
                for (int u = 0; u < n_band; ++u) {
                    const double su = bx[u];
                    rank += (su > st || (su == st && wslots[u] < jt)) ? 1 : 0;
                }
                pick[h] = rank < need;
            }
        }
        chosen_mask = 0ull;
#pragma unroll
        for (int h = 0; h < kBandCache / 32; ++h)
            chosen_mask |= (uint64_t)__ballot_sync(0xffffffffu, pick[h]) << (32 * h);
        __syncwarp();
    } else if (mode == 2) {
        auto band_key = [&](int j, bool& ok) -> uint64_t {
            const float f = row[j];
            ok = !(f > hi) && f >= lo;
            return ok ? f64_key(exact(j)) : 0ull;
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

    // ---- emit the kept blocks in ascending order
    int pos = 0, band_seen = 0, eq_seen = 0;
    for (int j0 = 0; j0 < nB; j0 += 32) {
        const int j = j0 + lane;
        const float f = j < nB ? row[j] : -INFINITY;
        const bool in_a = j < nB && f > hi;
        const bool in_b = j < nB && !in_a && f >= lo;
        const uint32_t bb = __ballot_sync(0xffffffffu, in_b);
        bool sel = in_a;
        if (mode == 0) {
            sel = sel || in_b;
        } else if (mode == 1) {
            const int slot = band_seen + __popc(bb & lanemask_lt());
            sel = sel || (in_b && ((chosen_mask >> slot) & 1ull));
        } else {
            uint64_t x = 0;
            if (in_b) x = f64_key(exact(j));
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
        kv_cnt[rid] = pos;
        if (pos != k) raise_device_error(kErrBadRouting);
    }
}

template <int D, int NSUB = 1>
__global__ void __launch_bounds__(256, NSUB == 1 ? 4 : 3) topk_kernel(SelectWorkspace ws, const int32_t* __restrict__ valid_len,
                                                   int H, int Npad, double sparsity, int budget, int kmax,
                                                   int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt,
                                                   long long rows) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5;
    const long long rid = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
    if (rid >= rows) return;
    topk_row<D, NSUB>(ws, valid_len, H, Npad, sparsity, budget, kmax, kv_idx, kv_cnt, rid,
                      smem_raw + (size_t)warp * topk_warp_smem(ws.ld));
}

// The rows that the fused screen left to the row routine above: ws.ovf_rows[0 ..
// *ws.ovf_count), their screened scores already in ws.scores.  Grid-stride over warps,
// so the grid need not know the count.
template <int D>
__global__ void __launch_bounds__(256, 4) topk_rest_kernel(SelectWorkspace ws, const int32_t* __restrict__ valid_len,
                                                           int H, int Npad, double sparsity, int budget, int kmax,
                                                           int32_t* __restrict__ kv_idx,
                                                           int32_t* __restrict__ kv_cnt) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, wpb = blockDim.x >> 5;
    const int n = *ws.ovf_count;
    for (int i = blockIdx.x * wpb + warp; i < n; i += gridDim.x * wpb)
        topk_row<D, 1>(ws, valid_len, H, Npad, sparsity, budget, kmax, kv_idx, kv_cnt, ws.ovf_rows[i],
                       smem_raw + (size_t)warp * topk_warp_smem(ws.ld));
}

}  // namespace sba

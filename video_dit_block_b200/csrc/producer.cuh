// producer.cuh -- the step before the router: QK RMSNorm + 3D RoPE with the block
// pooling done in the same pass, and the split of given block means for the screen.
//
// The page "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), the kernel layer,
// fuses the QK RMSNorm and the 3D RoPE of the attention inputs into one kernel
// (head dimension 128, RoPE dimension 96), on the rounding path that rounds the
// normalised value to bf16 before the rotation.  Per (b, h, token n):
//   y_d = bf16( x_d * rsqrt(mean_e x_e^2 + eps) * w_d )
//   channels [0, rope_dim): three axes of da = rope_dim / 3 channels for the token's
//   (t, y, x) position; pair (2i, 2i+1) of axis a turns by pos_a * base^(-2i/da):
//       o_2i = bf16(y_2i cos - y_2i+1 sin),  o_2i+1 = bf16(y_2i sin + y_2i+1 cos)
//   channels [rope_dim, D) pass through.
// The router pools these outputs over 64-token blocks; doing that here saves it a
// second pass over Q and K: the CTA of a block keeps its 64 output rows in shared
// memory and sums each channel over the valid rows in token order in fp64, the
// same sums, so the same fp64 means, as pool_kernel would form from the output.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <type_traits>

#include "select.cuh"  // kBlock, align256, SelectWorkspace

namespace sba {

constexpr int kMaxRopePairs = 64;  // per axis: rope_dim / 6

struct RopeFreqs {
    float inv_freq[kMaxRopePairs];  // base^(-2i/da), i < da / 2
};

// sin and cos of an fp32 angle: Cody-Waite reduction (W. J. Cody and W. Waite,
// "Software Manual for the Elementary Functions", 1980) by 2 pi split into a head
// with trailing zero bits and a tail, so k * head is exact for the |k| <= 2^12
// that positions times frequencies <= 1 reach, then the hardware approximations on
// [-pi, pi].  Absolute error about 1e-6 for |theta| < 2^12, far below one bf16 step.
// The nearest integer k is formed by adding and subtracting 1.5 * 2^23 (exact for
// |x| < 2^22), on the FMA pipe rather than the conversion pipe.
__device__ __forceinline__ void sincos_reduced(float theta, float* s, float* c) {
    constexpr float kInv2Pi = 0.15915494309189535f;
    constexpr float k2PiHi = 6.28125f;                 // 8 significant bits
    constexpr float k2PiLo = 1.9353071795864769e-3f;   // 2 pi - 6.28125
    constexpr float kRound = 12582912.0f;              // 1.5 * 2^23
    const float k = __fsub_rn(__fmaf_rn(theta, kInv2Pi, kRound), kRound);
    float r = fmaf(-k, k2PiHi, theta);
    r = fmaf(-k, k2PiLo, r);
    *s = __sinf(r);
    *c = __cosf(r);
}

// Packed fp32 product (mul.rn.f32x2), and the round trip of two fp32 values through
// bf16 (round to nearest even, as __float2bfloat16_rn) in one packed conversion.
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t bf16_round2(uint64_t v) {
    float a, b;
    unpack2(v, a, b);
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return pack2(__low2float(h), __high2float(h));
}

// One CTA of 256 threads per (bh, 64-token block).  A half-warp handles a row (lane l
// of the half owns channels [CPL l, CPL l + CPL), CPL = D / 16, an even count, so every
// RoPE pair is within a lane); warp w takes rows w, w + 8, ... two at a time, and all
// of its rows are loaded before any is processed.  Each lane then works on two of its
// rows at once in packed f32x2 arithmetic.  At D = 128 that takes up to 85 registers,
// three CTAs per SM; measured 11% faster than one row at a time in 64 registers.
template <int D>
__global__ void __launch_bounds__(256, D == 128 ? 3 : 4) qk_norm_rope_pool_kernel(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ valid_len, int H, int Npad, int rope_dim, const RopeFreqs freqs, float eps,
    __nv_bfloat16* __restrict__ out, double* __restrict__ means) {
    constexpr int CPL = D / 16;            // channels per lane: 8 (D = 128) or 4 (D = 64)
    constexpr int RPW = kBlock / 8 / 2;    // row pairs per warp
    using Vec = typename std::conditional<CPL == 8, uint4, uint2>::type;
    __shared__ __align__(16) __nv_bfloat16 tile[kBlock * D];
    const int nB = Npad / kBlock;
    const long long bh = blockIdx.x / nB;
    const int I = (int)(blockIdx.x % nB);
    const int b = (int)(bh / H);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hl = lane & 15, sub = lane >> 4;   // lane within the half, which half
    const int da = rope_dim / 3;
    const int c0 = CPL * hl;

    float wv[CPL];
#pragma unroll
    for (int e = 0; e < CPL; ++e) wv[e] = __bfloat162float(w[c0 + e]);
    // this lane's channel pairs never change: their axis (-1 = not rotated) and frequency
    int ax[CPL / 2];
    float fr[CPL / 2];
#pragma unroll
    for (int e = 0; e < CPL / 2; ++e) {
        const int c = c0 + 2 * e;
        ax[e] = c < rope_dim ? c / da : -1;
        fr[e] = c < rope_dim ? freqs.inv_freq[(c % da) >> 1] : 0.f;
    }

    Vec raw[RPW];
    float3 pp[RPW];  // positions as floats: small non-negative ints, converted through 2^23
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
        const int r = warp + 8 * (2 * j + sub);
        const int n = I * kBlock + r;
        raw[j] = *reinterpret_cast<const Vec*>(x + ((size_t)bh * Npad + n) * D + c0);
        const int32_t* q3 = pos + ((size_t)b * Npad + n) * 3;
        // int -> float for 0 <= v < 2^23: the bits of 2^23 + v, minus 2^23
        auto tof = [](int v) { return __fsub_rn(__int_as_float(0x4B000000 + v), 8388608.0f); };
        pp[j] = make_float3(tof(__ldg(q3)), tof(__ldg(q3 + 1)), tof(__ldg(q3 + 2)));
    }
    // Rows are taken two at a time (j and j + 1 of this lane), their arithmetic in packed
    // f32x2 operations: element by element the same operations, in the same order, as
    // one row at a time, so the same results, for about half the FMA-pipe instructions.
    const uint64_t kInv2Pi2 = pack2(0.15915494309189535f, 0.15915494309189535f);
    const uint64_t kRound2 = pack2(12582912.0f, 12582912.0f), kNegRound2 = pack2(-12582912.0f, -12582912.0f);
    const uint64_t kNeg2PiHi2 = pack2(-6.28125f, -6.28125f);
    const uint64_t kNeg2PiLo2 = pack2(-1.9353071795864769e-3f, -1.9353071795864769e-3f);
#pragma unroll
    for (int jj = 0; jj < RPW / 2; ++jj) {
        const int ja = 2 * jj, jb = 2 * jj + 1;
        float xa[CPL], xb[CPL];
        {
            const uint32_t* ua = reinterpret_cast<const uint32_t*>(&raw[ja]);
            const uint32_t* ub = reinterpret_cast<const uint32_t*>(&raw[jb]);
#pragma unroll
            for (int e = 0; e < CPL / 2; ++e) {
                const __nv_bfloat162 va = *reinterpret_cast<const __nv_bfloat162*>(&ua[e]);
                const __nv_bfloat162 vb = *reinterpret_cast<const __nv_bfloat162*>(&ub[e]);
                xa[2 * e] = __low2float(va);
                xa[2 * e + 1] = __high2float(va);
                xb[2 * e] = __low2float(vb);
                xb[2 * e + 1] = __high2float(vb);
            }
        }
        uint64_t ss2 = pack2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < CPL; ++e) {
            const uint64_t x2 = pack2(xa[e], xb[e]);
            ss2 = ffma2(x2, x2, ss2);
        }
        float ssa, ssb;
        unpack2(ss2, ssa, ssb);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) {
            ssa += __shfl_xor_sync(0xffffffffu, ssa, off);
            ssb += __shfl_xor_sync(0xffffffffu, ssb, off);
        }
        const uint64_t inv2 = pack2(rsqrtf(ssa / (float)D + eps), rsqrtf(ssb / (float)D + eps));
        uint32_t oa[CPL / 2], ob[CPL / 2];
#pragma unroll
        for (int e = 0; e < CPL; e += 2) {
            // the norm, rounded to bf16 before the rotation: y0 = channel e, y1 = e + 1,
            // rows a and b in the two halves
            const uint64_t t0 = fmul2(fmul2(pack2(xa[e], xb[e]), inv2), pack2(wv[e], wv[e]));
            const uint64_t t1 = fmul2(fmul2(pack2(xa[e + 1], xb[e + 1]), inv2), pack2(wv[e + 1], wv[e + 1]));
            const uint64_t y0 = bf16_round2(t0), y1 = bf16_round2(t1);
            const int a = ax[e / 2];
            const float pa_a = a == 0 ? pp[ja].x : (a == 1 ? pp[ja].y : pp[ja].z);
            const float pa_b = a == 0 ? pp[jb].x : (a == 1 ? pp[jb].y : pp[jb].z);
            const uint64_t ang = fmul2(pack2(pa_a, pa_b), pack2(fr[e / 2], fr[e / 2]));
            // sincos_reduced on both angles: the same Cody-Waite steps, packed
            const uint64_t k = fadd2(ffma2(ang, kInv2Pi2, kRound2), kNegRound2);
            uint64_t rr = ffma2(k, kNeg2PiHi2, ang);
            rr = ffma2(k, kNeg2PiLo2, rr);
            float ra, rb;
            unpack2(rr, ra, rb);
            const float sa = __sinf(ra), ca = __cosf(ra), sb = __sinf(rb), cb = __cosf(rb);
            const uint64_t cs = pack2(ca, cb), sn = pack2(sa, sb);
            const uint64_t r0 = ffma2(y0, cs, fmul2(y1, pack2(-sa, -sb)));
            const uint64_t r1 = ffma2(y0, sn, fmul2(y1, cs));
            float r0a, r0b, r1a, r1b, y0a, y0b, y1a, y1b;
            unpack2(r0, r0a, r0b);
            unpack2(r1, r1a, r1b);
            unpack2(y0, y0a, y0b);
            unpack2(y1, y1a, y1b);
            // channels past rope_dim keep y (a select: every lane evaluates the rotation)
            __nv_bfloat162 ha = __floats2bfloat162_rn(a >= 0 ? r0a : y0a, a >= 0 ? r1a : y1a);
            __nv_bfloat162 hb = __floats2bfloat162_rn(a >= 0 ? r0b : y0b, a >= 0 ? r1b : y1b);
            oa[e / 2] = *reinterpret_cast<uint32_t*>(&ha);
            ob[e / 2] = *reinterpret_cast<uint32_t*>(&hb);
        }
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            const int r = warp + 8 * (2 * (h2 ? jb : ja) + sub);
            const int n = I * kBlock + r;
            Vec ov;
            uint32_t* ou = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
            for (int e = 0; e < CPL / 2; ++e) ou[e] = h2 ? ob[e] : oa[e];
            *reinterpret_cast<Vec*>(out + ((size_t)bh * Npad + n) * D + c0) = ov;
            if (means) *reinterpret_cast<Vec*>(tile + r * D + c0) = ov;
        }
    }
    if (!means) return;
    __syncthreads();
    if (threadIdx.x < D) {
        const int L = valid_len ? valid_len[b] : Npad;
        int cnt = L - I * kBlock;
        cnt = cnt < 0 ? 0 : (cnt > kBlock ? kBlock : cnt);
        double s = 0.0;
        for (int r = 0; r < cnt; ++r) s = __dadd_rn(s, (double)__bfloat162float(tile[r * D + threadIdx.x]));
        means[((size_t)bh * nB + I) * D + threadIdx.x] = cnt > 0 ? __ddiv_rn(s, (double)cnt) : 0.0;
    }
}

// The screen's operands from given fp64 block means [BH][nB][D]: bf16 hi/lo split and
// the norm of each mean, with the same lane layout and arithmetic as pool_kernel's.
template <int D>
__global__ void __launch_bounds__(256) split_means_kernel(const double* __restrict__ mean64,
                                                          __nv_bfloat16* __restrict__ hi16,
                                                          __nv_bfloat16* __restrict__ lo16,
                                                          double* __restrict__ norm, long long n_groups) {
    constexpr int LPB = D / 8;
    long long grp = (long long)blockIdx.x * (256 / LPB) + threadIdx.x / LPB;
    const int g = threadIdx.x % LPB;
    const bool active = grp < n_groups;
    if (!active) grp = n_groups - 1;  // keep the shuffles below warp-uniform
    double m[8];
    const double* src = mean64 + (size_t)grp * D + 8 * g;
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        const double2 v = *reinterpret_cast<const double2*>(src + e);
        m[e] = v.x;
        m[e + 1] = v.y;
    }
    double sq = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) sq = fma(m[e], m[e], sq);
#pragma unroll
    for (int off = LPB / 2; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (!active) return;
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
    if (g == 0) norm[grp] = sqrt(sq);
}

}  // namespace sba

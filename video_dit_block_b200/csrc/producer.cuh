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

// One CTA of 256 threads per (bh, 64-token block).  A half-warp handles a row (lane l
// of the half owns channels [CPL l, CPL l + CPL), CPL = D / 16, an even count, so every
// RoPE pair is within a lane); warp w takes rows w, w + 8, ... two at a time, and all
// of its rows are loaded before any is processed.
template <int D>
__global__ void __launch_bounds__(256, 4) qk_norm_rope_pool_kernel(
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
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
        const int r = warp + 8 * (2 * j + sub);
        const int n = I * kBlock + r;
        float xv[CPL];
        const uint32_t* u = reinterpret_cast<const uint32_t*>(&raw[j]);
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) {
            const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&u[e]);
            xv[2 * e] = __low2float(v2);
            xv[2 * e + 1] = __high2float(v2);
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < CPL; ++e) ss = fmaf(xv[e], xv[e], ss);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float inv = rsqrtf(ss / (float)D + eps);
        uint32_t o2[CPL / 2];
#pragma unroll
        for (int e = 0; e < CPL; e += 2) {
            // the norm, rounded to bf16 before the rotation
            const float y0 = __bfloat162float(__float2bfloat16_rn(xv[e] * inv * wv[e]));
            const float y1 = __bfloat162float(__float2bfloat16_rn(xv[e + 1] * inv * wv[e + 1]));
            // every lane evaluates the rotation (no divergent branch); channels past
            // rope_dim then keep y by a select
            const int a = ax[e / 2];
            const float pa = a == 0 ? pp[j].x : (a == 1 ? pp[j].y : pp[j].z);
            float sn, cs;
            sincos_reduced(pa * fr[e / 2], &sn, &cs);
            const float r0 = a >= 0 ? fmaf(y0, cs, -y1 * sn) : y0;
            const float r1 = a >= 0 ? fmaf(y0, sn, y1 * cs) : y1;
            __nv_bfloat162 h2 = __floats2bfloat162_rn(r0, r1);
            o2[e / 2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        Vec ov;
        uint32_t* ou = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) ou[e] = o2[e];
        *reinterpret_cast<Vec*>(out + ((size_t)bh * Npad + n) * D + c0) = ov;
        if (means) *reinterpret_cast<Vec*>(tile + r * D + c0) = ov;
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

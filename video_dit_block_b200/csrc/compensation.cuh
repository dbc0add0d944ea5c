// compensation.cuh -- the rows the compensated attention walks after the kept blocks:
// the block means of K and V, rounded to bf16.
//
// Compensation of the dropped blocks follows PISA as the page "Sol Video Inference
// Engine" (sjmshsh.github.io), section 4.2.2, describes it: critical blocks exact,
// the others by a first-order Taylor approximation.  About a dropped block's mean
// key the expansion gives the block one softmax entry, logit s q.kbar_J + log(c_J)
// carrying vbar_J (the linear term of the normaliser sums to zero about the mean).
// The means are formed like the router's (fp64 sums over the valid tokens in token
// order, one correctly rounded division) and rounded once to bf16, the precision of
// the attention operands; blocks past a sample's length are zero rows.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "select.cuh"  // kBlock, sample_len

namespace sba {

// One group of D/8 lanes per (bh, J), J < nBpad (rows of [BH][nBpad][D]).
template <int D>
__global__ void __launch_bounds__(256) block_mean_bf16_kernel(const __nv_bfloat16* __restrict__ x,
                                                              const int32_t* __restrict__ valid_len, int H, int Npad,
                                                              int nBpad, __nv_bfloat16* __restrict__ out,
                                                              long long n_groups) {
    constexpr int LPB = D / 8;
    const long long grp = (long long)blockIdx.x * (256 / LPB) + threadIdx.x / LPB;
    if (grp >= n_groups) return;
    const int g = threadIdx.x % LPB;
    const long long bh = grp / nBpad;
    const int J = (int)(grp % nBpad);
    const int L = sample_len(valid_len, (int)(bh / H), Npad);
    int cnt = L - J * kBlock;
    cnt = cnt < 0 ? 0 : (cnt > kBlock ? kBlock : cnt);
    double s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) s[e] = 0.0;
    const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)bh * Npad + (size_t)J * kBlock) * D) + g;
    for (int n = 0; n < cnt; ++n) {
        const uint4 u = __ldg(src + (size_t)n * LPB);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            s[2 * e] = __dadd_rn(s[2 * e], (double)__uint_as_float(w[e] << 16));
            s[2 * e + 1] = __dadd_rn(s[2 * e + 1], (double)__uint_as_float(w[e] & 0xFFFF0000u));
        }
    }
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
        const __nv_bfloat16 a = __double2bfloat16(cnt > 0 ? __ddiv_rn(s[e], (double)cnt) : 0.0);
        const __nv_bfloat16 b = __double2bfloat16(cnt > 0 ? __ddiv_rn(s[e + 1], (double)cnt) : 0.0);
        __nv_bfloat162 h = __halves2bfloat162(a, b);
        pk[e / 2] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(out + (size_t)grp * D + 8 * g) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

}  // namespace sba

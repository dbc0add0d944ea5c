// attention3.cuh -- exact softmax attention over routed 64-token key blocks, sm_100a,
// two key blocks per step (D = 128).
//
// Same computation, tiling and routing as attn_kernel (attention.cuh; the block-sparse
// stage of the SubBlock router on the page "MiniMax-H3 on 8xH200 benchmark",
// section "How SubBlock sparse attention works"): a CTA owns two 64-row query blocks
// as one 128-row Q tile and walks the ascending union of their kept lists.  What
// differs is the step: two union blocks at a time.
//
// Why.  A tcgen05.mma with both operands in shared memory reads A and B through the
// one shared-memory port (about 128 B/clk per SM).  S = Q K^T with N = 64 keys reads
// 32 KB of Q per 16 KB of K, so S alone asks 192 B/clk at the full tensor rate; with
// the V operand and the TMA writes of K and V, a 64-key step moves 96 KB.  With N = 128
// (two key blocks) Q is read once per 128 keys: 80 KB per 64 keys.
//
// Layout.  TMEM (256 columns per CTA, two CTAs per SM): S at columns [0, 128) -- block
// a's logits in [0, 64), block b's in [64, 128) -- and O at [128, 256).  The softmax
// writes P (bf16 pairs) over columns [0, 64) once it has read S; the next S is issued
// after the PV that reads P, and tcgen05 MMAs of one thread run in issue order, so it
// never overwrites P too early.  S is single-buffered: within a CTA, S(t), the
// softmax, PV(t) and S(t+1) follow one another; the other CTA on the SM fills the
// tensor pipe meanwhile.  Shared memory: Q 32 KB, one 128-key stage of K (K-major,
// block a in rows 0-63, block b in rows 64-127) and one of V (MN-major, keys as rows),
// 32 KB each.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread t owns query row t = TMEM lane t.  Warps
//              0-1 serve query block I0, warps 2-3 query block I1; a block this half
//              does not keep costs no exponentials (P = 0 for its columns).
//   warp 4     builds the union list, then issues the TMA loads: Q once, then per step
//              K (once S of the previous step is done) and V (once its PV is done).
//   warp 5     allocates TMEM and issues the MMAs (one elected lane).
// A step with one block (the last of an odd union) uses N = 64 and K = 64.
//
// Every wait is bounded: on expiry the CTA records SBA_ERR_TIMEOUT, unwinds all
// roles, drains its own TMA loads and MMAs and frees its TMEM.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attention.cuh"
#include "common.cuh"

namespace sba {

struct Attn3Smem {
    static constexpr int kQ = 0;             // 2 chunks x 128 rows x 128 B
    static constexpr int kK = 32768;         // 2 chunks x 128 rows x 128 B
    static constexpr int kV = 65536;         // 2 chunks x 128 keys x 128 B
    static constexpr int kBars = 98304;
    // barriers: q_full, k_full, k_empty, v_full, v_empty, s_full, p_full, pv_done, drain
    static constexpr int kNumBars = 9;
    static constexpr int kCtl = kBars + kNumBars * 8;                 // tmem base, abort, n_union
    static constexpr int kBitmap = kCtl + 16;                         // uint32 [2][kMaxBlocks/32]
    static constexpr int kList = kBitmap + 2 * (kMaxBlocks / 32) * 4; // uint16 [kMaxBlocks]
    static constexpr int kTotal = kList + kMaxBlocks * 2;
    static constexpr int kAlloc = kTotal + 1024;                      // slack for 1024-byte alignment
};

__global__ void __launch_bounds__(192, 2)
    attn128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using SM = Attn3Smem;
    constexpr int D = 128;
    constexpr uint32_t kIdescS2 = idesc_bf16_f32(128, 128, 0, 0);   // two key blocks
    constexpr uint32_t kIdescS1 = idesc_bf16_f32(128, 64, 0, 0);    // one key block
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
    constexpr uint32_t kTmemCols = 256;
    constexpr uint32_t kBlockBytes = 64 * D * 2;                    // one key block of K or V

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sQ = smem_u32(sm + SM::kQ);
    const uint32_t sK = smem_u32(sm + SM::kK);
    const uint32_t sV = smem_u32(sm + SM::kV);
    const uint32_t bars = smem_u32(sm + SM::kBars);
    const uint32_t bar_q = bars, bar_kf = bars + 8, bar_ke = bars + 16, bar_vf = bars + 24, bar_ve = bars + 32;
    const uint32_t bar_sf = bars + 40, bar_pf = bars + 48, bar_pv = bars + 56, bar_drain = bars + 64;
    uint32_t* ctl = reinterpret_cast<uint32_t*>(sm + SM::kCtl);
    volatile uint32_t* abort_flag = ctl + 1;
    uint32_t* bm = reinterpret_cast<uint32_t*>(sm + SM::kBitmap);
    uint16_t* ulist = reinterpret_cast<uint16_t*>(sm + SM::kList);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int nQ = p.Npad / 64;
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
        mbar_init(bar_kf, 1);
        mbar_init(bar_ke, 1);
        mbar_init(bar_vf, 1);
        mbar_init(bar_ve, 1);
        mbar_init(bar_sf, 1);
        mbar_init(bar_pf, 128);
        mbar_init(bar_pv, 1);
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
            const uint32_t u = w < W ? (bm[w] | bm[kMaxBlocks / 32 + w]) : 0u;
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
    const int T = (n + 1) / 2;                 // steps of two union blocks
    const uint64_t lim = p.wait_limit;
    int issued_k = 0, issued_v = 0;           // steps whose K / V loads the producer has issued

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && T > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const bool q1 = qb[1] >= 0 && qb[1] < nQ;
            mbar_arrive_expect_tx(bar_q, (q1 ? 2 : 1) * (64 * D * 2));
            for (int h2 = 0; h2 < (q1 ? 2 : 1); ++h2)
                for (int c = 0; c < 2; ++c)
                    tma_load_3d(sQ + c * 16384 + h2 * 8192, &tmQ, bar_q, c * 64, qb[h2] * 64, bh);
            for (int t = 0; t < T; ++t) {
                const int nblk = (2 * t + 1 < n) ? 2 : 1;
                if (t > 0 && !wait_bounded(bar_ke, (t - 1) & 1, abort_flag, lim)) break;
                mbar_arrive_expect_tx(bar_kf, nblk * kBlockBytes);
                for (int e = 0; e < nblk; ++e)
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(sK + c * 16384 + e * 8192, &tmK, bar_kf, c * 64, ulist[2 * t + e] * 64, bh);
                issued_k = t + 1;
                if (t > 0 && !wait_bounded(bar_ve, (t - 1) & 1, abort_flag, lim)) break;
                mbar_arrive_expect_tx(bar_vf, nblk * kBlockBytes);
                for (int e = 0; e < nblk; ++e)
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(sV + c * 16384 + e * 8192, &tmV, bar_vf, c * 64, ulist[2 * t + e] * 64, bh);
                issued_v = t + 1;
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && T > 0) {
            bool ok = poll_bounded(bar_q, 0, abort_flag, lim);
            tc_fence_after();
            uint64_t dq[D / 16], dk[D / 16], dv[8];
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                dq[kk] = smem_desc_sw128(sQ + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
                dk[kk] = smem_desc_sw128(sK + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) dv[kk] = smem_desc_sw128(sV + kk * 2048, 16384, 1024);
            for (int t = 0; ok && t < T; ++t) {
                const bool two = 2 * t + 1 < n;
                if (!poll_bounded(bar_kf, t & 1, abort_flag, lim)) break;
                tc_fence_after();
                // S(t) into columns [0, 128) (or [0, 64)); issued after PV(t-1), which
                // reads P(t-1) from columns [0, 64)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_bf16_ss(tmem, dq[kk], dk[kk], two ? kIdescS2 : kIdescS1, kk > 0 ? 1u : 0u);
                mma_commit(bar_sf);
                mma_commit(bar_ke);
                if (!poll_bounded(bar_pf, t & 1, abort_flag, lim)) break;
                if (!poll_bounded(bar_vf, t & 1, abort_flag, lim)) break;
                tc_fence_after();
                const int nk = two ? 8 : 4;
                for (int kk = 0; kk < nk; ++kk)
                    mma_bf16_ts(tmem + 128, tmem + kk * 8, dv[kk], kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(bar_pv);
                mma_commit(bar_ve);
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
        for (int t = 0; t < T; ++t) {
            const bool two = 2 * t + 1 < n;
            const int Ja = ulist[2 * t], Jb = two ? ulist[2 * t + 1] : -1;
            const bool ka = (bmh[Ja >> 5] >> (Ja & 31)) & 1u;            // uniform over the warp
            const bool kb = two && ((bmh[Jb >> 5] >> (Jb & 31)) & 1u);
            int na = L - Ja * 64, nb = two ? L - Jb * 64 : 0;
            na = na > 64 ? 64 : na;
            nb = nb > 64 ? 64 : nb;
            if (!warp_wait_bounded(bar_sf, t & 1, abort_flag, lim)) { ok = false; break; }
            tc_fence_after();
            if (!ka && !kb) {
                // the other query block of the tile keeps these key blocks: P = 0 here
                uint32_t z[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) z[i] = 0u;
                tmem_st32(tl, z);
                if (two) tmem_st32(tl + 32, z);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar_pf);
                continue;
            }
            // the logits of the kept blocks (columns of an unkept block are not read)
            uint32_t u[128];
            if (ka) {
                tmem_ld32(tl, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
                tmem_ld32(tl + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
            }
            if (kb) {
                tmem_ld32(tl + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
                tmem_ld32(tl + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
            }
            tmem_wait_ld();
            constexpr uint32_t kNegInf = 0xff800000u;
            if (ka && na < 64) {  // ragged tail block of the sample
#pragma unroll
                for (int i = 0; i < 64; ++i) u[i] = i < na ? u[i] : kNegInf;
            }
            if (kb && nb < 64) {
#pragma unroll
                for (int i = 0; i < 64; ++i) u[64 + i] = i < nb ? u[64 + i] : kNegInf;
            }
            float mxa = -INFINITY, mxb = -INFINITY;
            if (ka) {
                float m0 = __uint_as_float(u[0]), m1 = __uint_as_float(u[1]);
#pragma unroll
                for (int i = 2; i < 62; i += 4) {
                    m0 = fmax3(m0, __uint_as_float(u[i]), __uint_as_float(u[i + 1]));
                    m1 = fmax3(m1, __uint_as_float(u[i + 2]), __uint_as_float(u[i + 3]));
                }
                mxa = fmax3(m0, m1, fmax3(__uint_as_float(u[62]), __uint_as_float(u[63]), -INFINITY));
            }
            if (kb) {
                float m0 = __uint_as_float(u[64]), m1 = __uint_as_float(u[65]);
#pragma unroll
                for (int i = 66; i < 126; i += 4) {
                    m0 = fmax3(m0, __uint_as_float(u[i]), __uint_as_float(u[i + 1]));
                    m1 = fmax3(m1, __uint_as_float(u[i + 2]), __uint_as_float(u[i + 3]));
                }
                mxb = fmax3(m0, m1, fmax3(__uint_as_float(u[126]), __uint_as_float(u[127]), -INFINITY));
            }
            const float m_new = fmaxf(m, fmaxf(mxa, mxb) * sc);
            const bool grow = m_new > m + 8.f;
            if (t > 0 && __any_sync(0xffffffffu, grow)) {
                // O holds sum P V with the old running max: move the max, rescale O and l.
                // (S(t) is complete, so PV(t-1), issued before it, is complete too.)
                if (!warp_wait_bounded(bar_pv, (t - 1) & 1, abort_flag, lim)) { ok = false; break; }
                tc_fence_after();
                const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m - m_new);
                // 8 columns at a time: the 128 logits of this step stay live meanwhile
#pragma unroll 1
                for (int ch = 0; ch < D / 8; ++ch) {
                    uint32_t o[8];
                    tmem_ld8(tl + 128 + ch * 8, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st8(tl + 128 + ch * 8, o);
                }
                l *= alpha;
                m = m_new;
            } else if (grow || t == 0) {
                m = m_new;
            }
            // p = 2^(s * scale * log2e - m), packed to bf16 pairs: block a -> columns
            // [0, 32), block b -> [32, 64); 8 columns per store
            const float nm = (m == -INFINITY) ? 0.f : -m;
            uint64_t acc = pack2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const bool kept = q < 4 ? ka : kb;
                if (q >= 4 && !two) break;
                uint32_t pk[8];
                if (!kept) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) pk[i] = 0u;
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float y0, y1;
                        unpack2(ffma2(pack2(__uint_as_float(u[16 * q + 2 * i]), __uint_as_float(u[16 * q + 2 * i + 1])),
                                      pack2(sc, sc), pack2(nm, nm)),
                                y0, y1);
                        const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
                        acc = fadd2(acc, pack2(p0, p1));
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                        pk[i] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                }
                tmem_st8(tl + 8 * q, pk);
            }
            {
                float a0, a1;
                unpack2(acc, a0, a1);
                l += a0 + a1;
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_pf);
        }

        // ------------------------------------------------------------ epilogue
        if (ok && T > 0) ok = warp_wait_bounded(bar_pv, (T - 1) & 1, abort_flag, lim);
        tc_fence_after();
        const bool in_range = qb[half] >= 0 && qb[half] < nQ;
        const bool valid = tok < L && l > 0.f;
        __nv_bfloat16* orow;
        float* lrow;
        if (p.n_shards > 0) {
            int sh = tok / p.shard_len;
            sh = sh < p.n_shards ? sh : p.n_shards - 1;
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
                if (T > 0) {
                    tmem_ld32(tl + 128 + ch * 32, o);
                    tmem_wait_ld();
                }
                if (in_range) {
                    uint32_t ob[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float o0 = (T > 0 && valid) ? __uint_as_float(o[2 * i]) * inv_l : 0.f;
                        const float o1 = (T > 0 && valid) ? __uint_as_float(o[2 * i + 1]) * inv_l : 0.f;
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(o0, o1);
                        ob[i] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(ob[4 * q4], ob[4 * q4 + 1], ob[4 * q4 + 2], ob[4 * q4 + 3]);
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
        if (warp == 4 && lane == 0 && T > 0) {
            wait_drain(bar_q, 0);
            if (issued_k > 0) wait_drain(bar_kf, (issued_k - 1) & 1);
            if (issued_v > 0) wait_drain(bar_vf, (issued_v - 1) & 1);
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

}  // namespace sba

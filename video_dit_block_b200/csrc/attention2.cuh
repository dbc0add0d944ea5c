// attention2.cuh -- the same exact attention over routed 64-token key blocks, run by
// a pair of SMs (a 2-CTA cluster issuing tcgen05 cta_group::2 MMAs), sm_100a, D = 128.
//
// What it computes is the block-sparse stage of the SubBlock router on the page
// "MiniMax-H3 on 8xH200 benchmark" (news.paixiangai.cn), section "How SubBlock
// sparse attention works", exactly as attn_kernel does; only the tiling differs.
//
// Why a pair.  A one-SM S = Q K^T MMA of M = 128, N = 64 re-reads the 128-row Q
// operand from shared memory for every 64 keys, and the shared-memory read port,
// shared with the TMA writes of K and V, limits it below the tensor rate.  A
// cta_group::2 MMA of M = 256, N = 128 splits A by rows (each SM reads its own 128
// Q rows) and B by columns (each SM reads one 64-key block), so each SM reads 6 KB
// per 16-deep K step for 64 tensor cycles instead of 6 KB per 32, and the step
// mix (S: M256 N128 K128, then O += P V: M256 N128 K128, P from TMEM), measured
// alone, runs at the full tensor rate with room left for the TMA writes.  Inside
// this kernel it runs at about half that rate; the softmax warps' TMEM stores and
// barrier waits account for part of the gap.
//
// Tiling.  A cluster owns four adjacent 64-row query blocks 4c .. 4c+3 of one (b, h);
// CTA r of the pair holds 2r and 2r+1 as its 128-row Q tile.  The pair walks the
// ascending union of the four kept lists two key blocks per step: step t covers
// u[2t] (S columns 0-63, K rows in CTA 0) and u[2t+1] (columns 64-127, K rows in
// CTA 1; u[2t] again, fully masked, when the union has odd length).  CTA r holds
// V columns 64r .. 64r+63 of both blocks.  A key block kept by only some of the four
// query blocks is masked for the others, so this tiling only suits routings that keep
// most blocks (every block, for dense attention).  Measured on B200 it is slower than
// attn_kernel even there, so it runs only when chosen (sba_set_attention_kernel).
//
// Warp roles (320 threads, one CTA per SM):
//   warps 0-7  softmax + epilogue.  Warp w serves TMEM lanes (query rows)
//              32 (w % 4) .. +31 and key block w / 4 of each step (S columns
//              64 (w / 4) .. +63); the two warps of a row quadrant agree on the
//              running max through shared memory every step, and each rescales
//              its half of O.  P (bf16) is written over the first 32 columns of
//              the warp's own S columns.
//   warp 8     builds the union list, then issues this CTA's TMA loads (Q once, then
//              K and V per step in NS-stage rings, K one step ahead of V)
//   warp 9     allocates TMEM for the pair (512 columns: S[3] at 0 / 128 / 256, O at
//              384);
//              in CTA 0 it issues every MMA of the pair; in CTA 1 it relays the
//              completion of that CTA's loads to CTA 0 (each CTA's loads complete on
//              its own barriers, so each drains its own copies on abort)
// Completion of an MMA group is multicast to the barrier of both CTAs; the P-ready
// barrier in CTA 0 counts one arrival per softmax warp of both CTAs.  S is triple
// buffered and the MMA warp issues S two steps ahead (S(t+2) before O += P(t) V(t)),
// so the next scores never wait on one step's softmax.  The epilogue waits on a
// one-phase barrier committed after the last PV, not on the two-phase PV barrier,
// whose parity a warp that keeps nothing in its last steps could read two phases
// early.
//
// A quarter of the exponentials run on the FMA pipe (exp2_fma2) instead of the MUFU:
// eight softmax warps exponentiate 128 x 128 scores per step, which at the MUFU's 16
// per cycle per SM is as long as the step's MMAs.
//
// Every wait is bounded, as in attn_kernel.  Both CTAs meet at a cluster barrier
// before any remote operation and again before TMEM is freed, so neither leaves
// while the other's MMAs, copies or arrivals may still touch it.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attention.cuh"

namespace sba {

template <int NS>
struct Attn2Smem {
    static constexpr int D = 128;
    static constexpr int kQBytes = 128 * D * 2;       // this CTA's 128 Q rows
    static constexpr int kKBytes = 64 * D * 2;        // one key block, all D
    static constexpr int kVBytes = 128 * 64 * 2;      // two key blocks, 64 of the D columns
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kQBytes;
    static constexpr int kV = kK + NS * kKBytes;
    static constexpr int kBars = kV + NS * kVBytes;
    // barriers: q_full, q_peer, k_full[NS], v_full[NS], k_peer[NS], v_peer[NS],
    //           k_empty[NS], v_empty[NS], s_full[3], p_full[3], pv_done[2], drain, o_full
    static constexpr int kNumBars = 2 + 6 * NS + 10;
    static constexpr int kCtl = kBars + kNumBars * 8;  // tmem base, abort, n_union, pad
    static constexpr int kXchg = kCtl + 16;            // float [2 parity][2 key block][128 rows]
    static constexpr int kFlags = kXchg + 2 * 2 * 128 * 4;                  // uint32 [2 parity][8 warps]
    static constexpr int kBitmap = kFlags + 2 * 8 * 4;                      // uint32 [4][kMaxBlocks/32]
    static constexpr int kList = kBitmap + 4 * (kMaxBlocks / 32) * 4;      // uint16 [kMaxBlocks]
    static constexpr int kTotal = kList + kMaxBlocks * 2;
    static constexpr int kAlloc = kTotal + 1024;
};

// 2^y for two values on the FMA pipe.  y = j + f with j = round(y), |f| <= 1/2; 2^f is
// a degree-3 polynomial with constant term 1 fitted for least maximum relative error
// on [-1/2, 1/2] (about 1.0e-4, below the bf16 rounding that P then takes), and j is
// added into the exponent field.  y is clamped at -127, where the result is exactly
// 0 (masked columns give y = -inf); above, no exponent field goes below 0 since
// j = -127 comes with f >= 0.  The softmax keeps y <= 8.
__device__ __forceinline__ void exp2_fma2(float y0, float y1, float& p0, float& p1) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
    constexpr float c1 = 0.69328287f, c2 = 0.24220999f, c3 = 0.05500843f;
    const uint64_t y = pack2(fmaxf(y0, -127.f), fmaxf(y1, -127.f));
    const uint64_t t = fadd2(y, pack2(kRound, kRound));        // j in the low mantissa bits
    const uint64_t j = fadd2(t, pack2(-kRound, -kRound));
    const uint64_t f = ffma2(j, pack2(-1.f, -1.f), y);
    uint64_t q = ffma2(pack2(c3, c3), f, pack2(c2, c2));
    q = ffma2(q, f, pack2(c1, c1));
    q = ffma2(q, f, pack2(1.f, 1.f));
    float qa, qb, ta, tb;
    unpack2(q, qa, qb);
    unpack2(t, ta, tb);
    p0 = __uint_as_float(__float_as_uint(qa) + (__float_as_uint(ta) << 23));
    p1 = __uint_as_float(__float_as_uint(qb) + (__float_as_uint(tb) << 23));
}

// Arrive once on a CTA-pair commit barrier without multicast (the drain of an
// aborted pair).
__device__ __forceinline__ void mma_pair_commit_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

template <int NS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    constexpr int D = 128;
    using SM = Attn2Smem<NS>;
    constexpr uint32_t kIdescS = idesc_bf16_f32(256, 128, 0, 0);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(256, D, 0, 1);
    constexpr uint32_t kTmemCols = 512;
    constexpr uint16_t kBoth = 0x3;

    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sQ = smem_u32(sm + SM::kQ);
    const uint32_t sK = smem_u32(sm + SM::kK);
    const uint32_t sV = smem_u32(sm + SM::kV);
    const uint32_t bars = smem_u32(sm + SM::kBars);
    const uint32_t bar_q = bars, bar_qp = bars + 8u;
    auto bar_kf = [&](int s) { return bars + 8u * (2 + s); };
    auto bar_vf = [&](int s) { return bars + 8u * (2 + NS + s); };
    auto bar_kp = [&](int s) { return bars + 8u * (2 + 2 * NS + s); };
    auto bar_vp = [&](int s) { return bars + 8u * (2 + 3 * NS + s); };
    auto bar_ke = [&](int s) { return bars + 8u * (2 + 4 * NS + s); };
    auto bar_ve = [&](int s) { return bars + 8u * (2 + 5 * NS + s); };
    auto bar_sf = [&](int s) { return bars + 8u * (2 + 6 * NS + s); };   // s < 3
    auto bar_pf = [&](int s) { return bars + 8u * (5 + 6 * NS + s); };   // s < 3
    auto bar_pv = [&](int s) { return bars + 8u * (8 + 6 * NS + s); };   // s < 2
    const uint32_t bar_drain = bars + 8u * (10 + 6 * NS);
    // O complete: one phase, committed after the last PV.  The epilogue cannot wait on
    // pv_done: a warp whose last steps keep nothing reaches it as soon as S(T-1) is
    // done, and S(T-1) is issued before PV(T-3), so pv_done may still be two phases
    // behind and its parity would read as complete.
    const uint32_t bar_of = bars + 8u * (11 + 6 * NS);
    uint32_t* ctl = reinterpret_cast<uint32_t*>(sm + SM::kCtl);
    volatile uint32_t* abort_flag = ctl + 1;
    float* xchg = reinterpret_cast<float*>(sm + SM::kXchg);
    volatile uint32_t* wflag = reinterpret_cast<uint32_t*>(sm + SM::kFlags);
    uint32_t* bm = reinterpret_cast<uint32_t*>(sm + SM::kBitmap);
    uint16_t* ulist = reinterpret_cast<uint16_t*>(sm + SM::kList);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int h = blockIdx.y, b = blockIdx.z;
    const int bh = b * p.H + h;
    const int nQ = p.Npad / 64;
    const int c4 = 4 * (int)(blockIdx.x >> 1);     // the cluster's first query block
    const int qb[2] = {c4 + 2 * (int)rank, c4 + 2 * (int)rank + 1};
    const int L = p.valid_len ? p.valid_len[b] : p.Npad;
    const int nB = (L + 63) / 64;
    const int W = (nB + 31) / 32;
    constexpr int BW = kMaxBlocks / 32;

    if (tid == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_qp, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar_kf(s), 1);
            mbar_init(bar_vf(s), 1);
            mbar_init(bar_kp(s), 1);
            mbar_init(bar_vp(s), 1);
            mbar_init(bar_ke(s), 1);
            mbar_init(bar_ve(s), 1);
        }
        for (int s = 0; s < 3; ++s) {
            mbar_init(bar_sf(s), 1);
            mbar_init(bar_pf(s), 16);  // 8 softmax warps in each CTA
        }
        for (int s = 0; s < 2; ++s) mbar_init(bar_pv(s), 1);
        mbar_init(bar_drain, 1);
        mbar_init(bar_of, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 9) tmem_alloc_pair(smem_u32(ctl), kTmemCols);
    if (warp == 8) {
        // kept-set bitmaps of the cluster's four query blocks, then their ascending union
        for (int w = lane; w < W; w += 32) {
            uint32_t full = 0;
            if (p.dense) full = (w * 32 + 32 <= nB) ? 0xffffffffu : ((1u << (nB - w * 32)) - 1u);
            for (int s = 0; s < 4; ++s) bm[s * BW + w] = (p.dense && c4 + s < nB) ? full : 0u;
        }
        __syncwarp();
        if (!p.dense) {
            for (int s = 0; s < 4; ++s) {
                const int I = c4 + s;
                if (I >= nQ) continue;
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
                        atomicOr(&bm[s * BW + (J >> 5)], 1u << (J & 31));
                    else
                        raise_device_error(kErrBadRouting);
                }
            }
        }
        __syncwarp();
        int base = 0;
        for (int w0 = 0; w0 < W; w0 += 32) {
            const int w = w0 + lane;
            const uint32_t u = w < W ? (bm[w] | bm[BW + w] | bm[2 * BW + w] | bm[3 * BW + w]) : 0u;
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
    // barriers initialised and TMEM allocated in both CTAs before any remote arrival
    // or pair MMA
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = ctl[0];
    const int n = static_cast<int>(ctl[2]);
    const int T = (n + 1) / 2;                      // steps of two key blocks
    const uint64_t lim = p.wait_limit;
    int issued_k = 0, issued_v = 0;
    auto step_block = [&](int t, int kb) {          // key block loaded for (step, half)
        const int i = 2 * t + kb;
        return static_cast<int>(ulist[i < n ? i : 2 * t]);
    };

    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && T > 0) {
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            const int nq = (qb[0] < nQ ? 1 : 0) + (qb[1] < nQ ? 1 : 0);
            if (nq > 0) {
                mbar_arrive_expect_tx(bar_q, nq * (64 * D * 2));
                for (int h2 = 0; h2 < nq; ++h2)
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(sQ + c * (128 * 128) + h2 * (64 * 128), &tmQ, bar_q, c * 64, qb[h2] * 64, bh);
            } else {
                mbar_arrive(bar_q);  // an empty tile: its rows only ever multiply P = 0
            }
            for (int t = 0; t <= T; ++t) {
                if (t < T) {
                    const int st = t % NS;
                    if (t >= NS && !wait_bounded(bar_ke(st), ((t / NS) - 1) & 1, abort_flag, lim)) break;
                    const int J = step_block(t, (int)rank);
                    mbar_arrive_expect_tx(bar_kf(st), SM::kKBytes);
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(sK + st * SM::kKBytes + c * (64 * 128), &tmK, bar_kf(st), c * 64, J * 64, bh);
                    issued_k = t + 1;
                }
                if (t >= 1) {
                    const int tv = t - 1, st = tv % NS;
                    if (tv >= NS && !wait_bounded(bar_ve(st), ((tv / NS) - 1) & 1, abort_flag, lim)) break;
                    mbar_arrive_expect_tx(bar_vf(st), SM::kVBytes);
                    for (int kb = 0; kb < 2; ++kb)
                        tma_load_3d(sV + st * SM::kVBytes + kb * (64 * 128), &tmV, bar_vf(st), 64 * (int)rank,
                                    step_block(tv, kb) * 64, bh);
                    issued_v = tv + 1;
                }
            }
        }
    } else if (warp == 9) {
        if (leader) {
            // -------------------------------------------------------- MMA issuer (pair)
            // The tensor pipe holds only a few queued MMAs, so this thread must issue
            // without stalls: descriptors are precomputed (a shared-memory descriptor
            // steps by adding (byte offset >> 4) to its start-address field), the
            // barriers the next group needs are tested (non-blocking) before the current
            // group issues and read only after it, and it waits -- by polling, which
            // resumes at once -- only for a barrier that is really pending.
            if (lane == 0 && T > 0) {
                bool ok = poll_bounded(bar_q, 0, abort_flag, lim) && poll_bounded(bar_qp, 0, abort_flag, lim);
                uint64_t dq[D / 16], dk[D / 16], dv[8];
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    dq[kk] = smem_desc_sw128(sQ + (kk / 4) * (128 * 128) + (kk % 4) * 32, 16, 1024);
                    dk[kk] = smem_desc_sw128(sK + (kk / 4) * (64 * 128) + (kk % 4) * 32, 16, 1024);
                }
#pragma unroll
                for (int k2 = 0; k2 < 8; ++k2) dv[k2] = smem_desc_sw128(sV + k2 * (16 * 128), 128 * 128, 1024);
                constexpr uint64_t kKStep = SM::kKBytes >> 4, kVStep = SM::kVBytes >> 4;
                // S(j) = Q K(j)^T into S buffer j % 3 (its last P was read by PV(j - 3),
                // issued before); K(j) in stage j % NS
                auto s_group = [&](int kst, int sbuf) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_pair_bf16_ss(tmem + sbuf * 128, dq[kk], dk[kk] + kst * kKStep, kIdescS, kk > 0 ? 1u : 0u);
                    mma_pair_commit(bar_sf(sbuf), kBoth);
                    mma_pair_commit(bar_ke(kst), kBoth);
                };
                auto k_wait = [&](int j) {
                    const int st = j % NS;
                    const uint32_t par = (j / NS) & 1;
                    return poll_bounded(bar_kf(st), par, abort_flag, lim) &&
                           poll_bounded(bar_kp(st), par, abort_flag, lim);
                };
                for (int j = 0; ok && j < 2 && j < T; ++j) {
                    ok = k_wait(j);
                    if (!ok) break;
                    tc_fence_after();
                    s_group(j % NS, j);
                }
                int done_pv = 0;
                bool k_pre = false;  // K(t + 2) seen ready during the previous PV group
                int sb = 0;          // S buffer of step t (t % 3)
                for (int t = 0; ok && t < T; ++t) {
                    const int sv = t % NS;
                    const uint32_t pv_par = (t / NS) & 1;
                    const uint32_t p_par = (t / 3) & 1;
                    bool p_ok = false, vf_ok = false, vp_ok = false;
                    if (t + 2 < T) {
                        if (!k_pre && !k_wait(t + 2)) break;
                        tc_fence_after();
                        p_ok = mbar_test_wait(bar_pf(sb), p_par);
                        vf_ok = mbar_test_wait(bar_vf(sv), pv_par);
                        vp_ok = mbar_test_wait(bar_vp(sv), pv_par);
                        s_group((t + 2) % NS, sb == 0 ? 2 : sb - 1);
                    }
                    if (!p_ok && !poll_bounded(bar_pf(sb), p_par, abort_flag, lim)) break;
                    if (!vf_ok && !poll_bounded(bar_vf(sv), pv_par, abort_flag, lim)) break;
                    if (!vp_ok && !poll_bounded(bar_vp(sv), pv_par, abort_flag, lim)) break;
                    tc_fence_after();
                    const int jn = t + 3;
                    bool kf_ok = false, kp_ok = false;
                    if (jn < T) {
                        kf_ok = mbar_test_wait(bar_kf(jn % NS), (jn / NS) & 1);
                        kp_ok = mbar_test_wait(bar_kp(jn % NS), (jn / NS) & 1);
                    }
                    const uint32_t pa = tmem + sb * 128;
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2)
                        mma_pair_bf16_ts(tmem + 384, pa + (k2 < 4 ? k2 * 8 : 64 + (k2 - 4) * 8), dv[k2] + sv * kVStep,
                                         kIdescPV, (t > 0 || k2 > 0) ? 1u : 0u);
                    mma_pair_commit(bar_pv(t & 1), kBoth);
                    mma_pair_commit(bar_ve(sv), kBoth);
                    done_pv = t + 1;
                    k_pre = kf_ok && kp_ok;
                    sb = sb == 2 ? 0 : sb + 1;
                }
                if (done_pv == T) mma_pair_commit(bar_of, kBoth);
            }
        } else {
            // -------------------------------------------------------- relay (CTA 1)
            // CTA 0's MMAs read this CTA's Q, K and V: tell it when each has landed.
            if (lane == 0 && T > 0) {
                bool ok = wait_bounded(bar_q, 0, abort_flag, lim);
                if (ok) mbar_arrive_remote(mapa_shared(bar_qp, 0));
                for (int t = 0; ok && t < T; ++t) {
                    const int st = t % NS;
                    const uint32_t par = (t / NS) & 1;
                    if (!wait_bounded(bar_kf(st), par, abort_flag, lim)) break;
                    mbar_arrive_remote(mapa_shared(bar_kp(st), 0));
                    if (!wait_bounded(bar_vf(st), par, abort_flag, lim)) break;
                    mbar_arrive_remote(mapa_shared(bar_vp(st), 0));
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps
        const int qd = warp & 3, kb = warp >> 2;
        const int r = qd * 32 + lane;           // query row of this CTA's tile = TMEM lane
        const int half = r >> 6;
        const int I = qb[half];
        const bool slot_ok = I < nB;            // this row's query block has keys in the sample
        const int tok = I * 64 + (r & 63);
        const uint32_t* bmh = bm + (2 * (int)rank + half) * BW;
        const uint32_t tl = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const uint32_t pf_remote = leader ? 0u : mapa_shared(bar_pf(0), 0);
        const float sc = p.scale_log2;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        // The two warps of a row quadrant pass the same named barriers in the same
        // order whatever happens: a failed wait is carried to the next exchange, where
        // both see it and leave the loop together.
        bool failed = false;
        for (int t = 0; t < T; ++t) {
            const int i = 2 * t + kb;
            const int J = i < n ? static_cast<int>(ulist[i]) : -1;
            const bool kept = slot_ok && J >= 0 && ((bmh[J >> 5] >> (J & 31)) & 1u);  // uniform over the warp
            int ncol = kept ? L - J * 64 : 0;
            ncol = ncol > 64 ? 64 : ncol;
            if (!failed && !warp_wait_bounded(bar_sf(t % 3), (t / 3) & 1, abort_flag, lim)) failed = true;
            tc_fence_after();
            const uint32_t sbuf = tl + (t % 3) * 128 + kb * 64;
            float x[64];
            float mx = -INFINITY;
            if (kept && !failed) {
                uint32_t a[32], c[32];
                tmem_ld32(sbuf, a);
                tmem_ld32(sbuf + 32, c);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    x[k] = __uint_as_float(a[k]);
                    x[32 + k] = __uint_as_float(c[k]);
                }
                if (ncol < 64) {
#pragma unroll
                    for (int k = 0; k < 64; ++k) x[k] = k < ncol ? x[k] : -INFINITY;
                }
                float mx0 = x[0], mx1 = x[1];
#pragma unroll
                for (int k = 2; k < 62; k += 4) {
                    mx0 = fmax3(mx0, x[k], x[k + 1]);
                    mx1 = fmax3(mx1, x[k + 2], x[k + 3]);
                }
                mx0 = fmax3(mx0, x[62], x[63]);
                mx = fmaxf(mx0, mx1) * sc;
            }
            // the row's max over both key blocks of the step, from the partner warp
            float* xs = xchg + (t & 1) * 256;
            xs[kb * 128 + r] = mx;
            if (lane == 0) wflag[(t & 1) * 8 + warp] = failed ? 1u : 0u;
            named_bar_sync(1 + qd, 64);
            if (wflag[(t & 1) * 8 + qd] | wflag[(t & 1) * 8 + qd + 4]) {
                ok = false;
                break;
            }
            const float m_new = fmaxf(m, fmaxf(xs[r], xs[128 + r]));
            const bool grow = m_new > m + 8.f;
            if (t > 0 && __any_sync(0xffffffffu, grow)) {
                // O holds sum P V with the old running max: move it, rescale this warp's
                // half of O and its part of l
                // (the barrier's previous phase, PV(t-3), finished before S(t), issued after it)
                if (!warp_wait_bounded(bar_pv((t - 1) & 1), ((t - 1) >> 1) & 1, abort_flag, lim)) {
                    failed = true;
                    continue;
                }
                tc_fence_after();
                const float alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m - m_new);
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    uint32_t o[32];
                    const uint32_t oa = tl + 384 + kb * 64 + ch * 32;
                    tmem_ld32(oa, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    tmem_st32(oa, o);
                }
                l *= alpha;
                m = m_new;
            } else if (grow || t == 0) {
                m = m_new;
            }
            uint32_t pk[32];
            if (kept) {
                const float nm = (m == -INFINITY) ? 0.f : -m;
                const uint64_t sc2 = pack2(sc, sc), nm2 = pack2(nm, nm);
                uint64_t acc0 = pack2(0.f, 0.f), acc1 = acc0;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    float y0, y1, p0, p1;
                    unpack2(ffma2(pack2(x[2 * k], x[2 * k + 1]), sc2, nm2), y0, y1);
                    if ((k & 3) == 3) {
                        exp2_fma2(y0, y1, p0, p1);
                    } else {
                        p0 = ex2_approx(y0);
                        p1 = ex2_approx(y1);
                    }
                    if (k & 1) acc1 = fadd2(acc1, pack2(p0, p1));
                    else acc0 = fadd2(acc0, pack2(p0, p1));
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    pk[k] = *reinterpret_cast<uint32_t*>(&h2);
                }
                float a0, a1, b0, b1;
                unpack2(acc0, a0, a1);
                unpack2(acc1, b0, b1);
                l += (a0 + a1) + (b0 + b1);
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) pk[k] = 0u;
            }
            tmem_st32(sbuf, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(bar_pf(t % 3));
                else mbar_arrive_remote(pf_remote + 8u * (t % 3));
            }
        }

        // ------------------------------------------------------------ epilogue
        ok = ok && !failed;
        if (ok && T > 0) ok = warp_wait_bounded(bar_of, 0, abort_flag, lim);
        tc_fence_after();
        // l over both key-block halves (the exchange slots of step parity T & 1 are free:
        // the partner passed this step's barrier before reaching the epilogue)
        float* xs = xchg + (T & 1) * 256;
        xs[kb * 128 + r] = l;
        named_bar_sync(1 + qd, 64);
        const float lt = xs[r] + xs[128 + r];
        const bool in_range = I < nQ;
        const bool valid = tok < L && lt > 0.f;
        __nv_bfloat16* orow = p.o + ((size_t)bh * p.Npad + tok) * D + kb * 64;
        if (ok) {
            const float inv_l = valid ? 1.f / lt : 0.f;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t o[32];
                if (T > 0) {
                    tmem_ld32(tl + 384 + kb * 64 + ch * 32, o);
                    tmem_wait_ld();
                }
                if (in_range) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float o0 = (T > 0 && valid) ? __uint_as_float(o[2 * k]) * inv_l : 0.f;
                        const float o1 = (T > 0 && valid) ? __uint_as_float(o[2 * k + 1]) * inv_l : 0.f;
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(o0, o1);
                        pk[k] = *reinterpret_cast<uint32_t*>(&h2);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            if (in_range && kb == 0 && p.lse)
                p.lse[(size_t)bh * p.Npad + tok] = valid ? (m + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        // this CTA's own copies land, and CTA 0's MMAs finish, before TMEM is freed
        if (warp == 8 && lane == 0 && T > 0) {
            wait_drain(bar_q, 0);
            for (int t = issued_k > NS ? issued_k - NS : 0; t < issued_k; ++t)
                wait_drain(bar_kf(t % NS), (t / NS) & 1);
            for (int t = issued_v > NS ? issued_v - NS : 0; t < issued_v; ++t)
                wait_drain(bar_vf(t % NS), (t / NS) & 1);
        }
        if (warp == 9 && lane == 0 && leader) {
            mma_pair_commit_local(bar_drain);
            wait_drain(bar_drain, 0);
        }
        __syncthreads();
    }
    tc_fence_before();
    cluster_sync();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace sba

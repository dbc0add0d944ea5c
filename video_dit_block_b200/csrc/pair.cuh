// pair.cuh -- choose which two query blocks share a 128-row attention tile.
//
// The attention kernel runs two 64-row query blocks per tile over the union of
// their kept key blocks; a key block kept by only one of them is masked work for
// the other.  Pairing query blocks whose kept lists overlap most cuts that waste.
// This pass is a heuristic on top of the routing and never changes any result,
// only which query blocks share a tile:
//   1. a bitmap of each query block's kept key blocks;
//   2. a few rounds of mutual-best matching: every unmatched query block proposes
//      the unmatched block within +-64 positions whose kept set overlaps its own
//      most (ties: nearer, then lower), and mutual proposals are matched.  Overlaps
//      are computed once; later rounds walk each block's 16 best candidates, all
//      rounds of a (b, h) in one CTA with its proposals in shared memory.  The
//      window reaches the same position one frame later in the raster order of
//      these latent grids (25-57 blocks per frame), where the kept sets are most
//      alike;
//   3. the tile list: matched pairs in order, then the leftovers two by two, then
//      the blocks past the sample's valid length; an odd count leaves one slot -1.
#pragma once
#include <cstdint>

#include "select.cuh"  // align256

namespace sba {

constexpr int kPairWindow = 64;  // a multiple of 32
constexpr int kPairRounds = 4;

constexpr int kPairCands = 16;  // candidates kept per query block after the overlap pass
static_assert(kPairCands % 4 == 0, "a row of candidates is read as 16-byte vectors");

struct PairWorkspace {
    uint32_t* bits;     // [BH][nQ][W] kept-set bitmaps, W = ceil(nQ / 32)
    int32_t* proposal;  // [BH][nQ]
    int32_t* partner;   // [BH][nQ], -1 = unmatched
    int32_t* cand;      // [BH][nQ][kPairCands] best candidates in preference order, -1 = none
};

__host__ __device__ inline size_t pair_workspace_bytes(size_t BH, size_t nQ) {
    const size_t W = (nQ + 31) / 32;
    return align256(BH * nQ * W * 4) + 2 * align256(BH * nQ * 4) + align256(BH * nQ * kPairCands * 4);
}

__host__ __device__ inline PairWorkspace carve_pair_workspace(void* base, size_t BH, size_t nQ) {
    const size_t W = (nQ + 31) / 32;
    char* p = static_cast<char*>(base);
    PairWorkspace w;
    w.bits = reinterpret_cast<uint32_t*>(p);
    p += align256(BH * nQ * W * 4);
    w.proposal = reinterpret_cast<int32_t*>(p);
    p += align256(BH * nQ * 4);
    w.partner = reinterpret_cast<int32_t*>(p);
    p += align256(BH * nQ * 4);
    w.cand = reinterpret_cast<int32_t*>(p);
    return w;
}

// One warp per routing row (bh, I): its kept-set bitmap (built in shared memory,
// then written out word by word).
__global__ void __launch_bounds__(256) pair_bitmap_kernel(PairWorkspace ws, const int32_t* __restrict__ kv_idx,
                                                          const int32_t* __restrict__ kv_cnt, int nQ, int kmax,
                                                          long long rows) {
    extern __shared__ uint32_t srow[];  // [8 warps][W]
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + warp;
    if (row >= rows) return;
    const int W = (nQ + 31) / 32;
    uint32_t* bm = srow + warp * W;
    for (int w = lane; w < W; w += 32) bm[w] = 0u;
    __syncwarp();
    int cnt = kv_cnt[row];
    cnt = cnt < 0 ? 0 : (cnt > kmax ? kmax : cnt);
    const int32_t* lst = kv_idx + (size_t)row * kmax;
    constexpr int kLoads = 8;  // entries of a lane loaded before their bits are set
    for (int t0 = 0; t0 < cnt; t0 += 32 * kLoads) {
        int J[kLoads];
#pragma unroll
        for (int u = 0; u < kLoads; ++u) {
            const int t = t0 + 32 * u + lane;
            J[u] = t < cnt ? lst[t] : -1;
        }
#pragma unroll
        for (int u = 0; u < kLoads; ++u)
            if (J[u] >= 0 && J[u] < nQ) atomicOr(&bm[J[u] >> 5], 1u << (J[u] & 31));
    }
    __syncwarp();
    uint32_t* out = ws.bits + (size_t)row * W;
    for (int w = lane; w < W; w += 32) out[w] = bm[w];
}

// A CTA of 16 warps proposes for 16 consecutive query blocks a0..a0+15 of one (b, h);
// the bitmaps of their joint window [a0 - 64, a0 + 79] are staged in shared memory
// once.  A query block that keeps every key block (dense routing) has the same
// overlap with every candidate and proposes nothing, so it stays in order.
constexpr int kPairWarps = 16;
constexpr int kPairSpan = 2 * kPairWindow + kPairWarps;  // blocks staged per CTA
static_assert(kPairSpan % kPairWarps == 0, "the staging gives each warp the same number of rows");

// Words per staged bitmap row: W rounded up to a multiple of 4 (16-byte vector reads)
// and, if that is a multiple of 8, 4 more, so that the rows read by 8 consecutive lanes
// start in different banks.
__host__ __device__ inline int pair_row_words(int W) {
    int p = (W + 3) / 4 * 4;
    if (p % 8 == 0) p += 4;
    return p;
}

__global__ void __launch_bounds__(32 * kPairWarps) pair_propose_kernel(PairWorkspace ws,
                                                           const int32_t* __restrict__ kv_cnt,
                                                           const int32_t* __restrict__ valid_len,
                                                           int H, int nQ, int tiles_per_bh) {
    extern __shared__ __align__(16) uint32_t sbits[];  // [kPairSpan][Wp], zero-padded
    const int bh = blockIdx.x / tiles_per_bh;
    const int a0 = (blockIdx.x % tiles_per_bh) * kPairWarps;
    const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int L = valid_len ? valid_len[bh / H] : nQ * 64;
    const int nB = (L + 63) / 64;
    const int W = (nQ + 31) / 32;
    const int Wp = pair_row_words(W);
    const uint32_t* gbits = ws.bits + (size_t)bh * nQ * W;
    const int lo = a0 - kPairWindow;
    // warp w stages rows w, w + 16, ...: five loads of a lane in flight before their stores
    constexpr int kRowsPerWarp = kPairSpan / kPairWarps, kGroup = 5;
    for (int w = lane; w < Wp; w += 32) {
#pragma unroll 1
        for (int i0 = 0; i0 < kRowsPerWarp; i0 += kGroup) {
            uint32_t v[kGroup];
#pragma unroll
            for (int j = 0; j < kGroup; ++j) {
                const int c = lo + warp + kPairWarps * (i0 + j);
                v[j] = (i0 + j < kRowsPerWarp && c >= 0 && c < nB && w < W) ? gbits[(size_t)c * W + w] : 0u;
            }
#pragma unroll
            for (int j = 0; j < kGroup; ++j)
                if (i0 + j < kRowsPerWarp) sbits[(warp + kPairWarps * (i0 + j)) * Wp + w] = v[j];
        }
    }
    __syncthreads();
    const int a = a0 + warp;
    if (a >= nQ) return;
    const size_t row = (size_t)bh * nQ + a;
    int32_t* cand = ws.cand + row * kPairCands;
    if (a >= nB || kv_cnt[row] >= nB) {
        if (lane < kPairCands) cand[lane] = -1;
        if (lane == 0) ws.proposal[row] = -1;
        return;
    }
    const uint32_t* ba = sbits + (size_t)(a - lo) * Wp;
    // lane l scores a - 64 + l, a - 32 + l, a + 1 + l, a + 33 + l.  Preference as one
    // ordered 32-bit key: larger overlap, then smaller distance, then the lower index
    // (of the two candidates at one distance, the one before a); 0 = no candidate.
    constexpr int kSlots = 2 * kPairWindow / 32;
    uint32_t key[kSlots];
#pragma unroll
    for (int slot = 0; slot < kSlots; ++slot) {
        const int half = kPairWindow / 32;
        const int c = slot < half ? a - kPairWindow + 32 * slot + lane : a + 1 + 32 * (slot - half) + lane;
        key[slot] = 0u;
        if (c < 0 || c >= nB) continue;
        const uint32_t* bc = sbits + (size_t)(c - lo) * Wp;
        int ov = 0;
        for (int w = 0; w < Wp; w += 4) {  // four words per read; the padding is zero
            const uint4 x = *reinterpret_cast<const uint4*>(ba + w);
            const uint4 y = *reinterpret_cast<const uint4*>(bc + w);
            ov += __popc(x.x & y.x) + __popc(x.y & y.y) + __popc(x.z & y.z) + __popc(x.w & y.w);
        }
        const int dist = c > a ? c - a : a - c;  // 1 .. kPairWindow
        key[slot] = ((uint32_t)(ov + 1) << 8) | ((uint32_t)(kPairWindow - dist) << 1) | (c < a ? 1u : 0u);
    }
    // the kPairCands best candidates, best first
    for (int r = 0; r < kPairCands; ++r) {
        uint32_t mine = key[0];
#pragma unroll
        for (int slot = 1; slot < kSlots; ++slot) mine = max(mine, key[slot]);
        const uint32_t best = __reduce_max_sync(0xffffffffu, mine);
        if (best != 0u && mine == best) {
#pragma unroll
            for (int slot = 0; slot < kSlots; ++slot) key[slot] = key[slot] == best ? 0u : key[slot];
        }
        if (lane == 0) {
            const int dist = kPairWindow - (int)((best >> 1) & 0x7Fu);
            cand[r] = best == 0u ? -1 : ((best & 1u) ? a - dist : a + dist);
        }
    }
    if (lane == 0) ws.proposal[row] = cand[0];
}

// One CTA per (b, h) for the matching rounds and the tile list, with the head's
// proposals and partners in shared memory and a block barrier between the steps of
// a round (so every step sees the whole previous step, as separate launches would):
//   resolve    a proposal returned by its target matches the two;
//   repropose  (rounds after the first) every unmatched block proposes its first
//              cached candidate that is still unmatched;
// then warp 0 writes the tile list pair_order[bh][2 * nP] (nP = ceil(nQ / 2)).
constexpr int kPairMatchThreads = 1024;

__global__ void __launch_bounds__(kPairMatchThreads) pair_match_kernel(PairWorkspace ws,
                                                                     const int32_t* __restrict__ valid_len,
                                                                     int H, int nQ,
                                                                     int32_t* __restrict__ pair_order) {
    extern __shared__ int32_t pm_smem[];  // proposal [nQ], partner [nQ]
    int32_t* prop = pm_smem;
    int32_t* part = pm_smem + nQ;
    const int bh = blockIdx.x;
    const int L = valid_len ? valid_len[bh / H] : nQ * 64;
    const int nB = (L + 63) / 64;
    const size_t base = (size_t)bh * nQ;
    for (int a = threadIdx.x; a < nQ; a += blockDim.x) {
        prop[a] = ws.proposal[base + a];
        part[a] = -1;
    }
    __syncthreads();
    for (int r = 0; r < kPairRounds; ++r) {
        if (r > 0) {
            for (int a = threadIdx.x; a < nQ; a += blockDim.x) {
                int p = -1;
                if (part[a] < 0) {
                    // the row's candidates in four 16-byte loads, then scanned in order
                    const int4* c4 = reinterpret_cast<const int4*>(ws.cand + (base + a) * kPairCands);
                    int cs[kPairCands];
#pragma unroll
                    for (int v = 0; v < kPairCands / 4; ++v) {
                        const int4 x = c4[v];
                        cs[4 * v] = x.x;
                        cs[4 * v + 1] = x.y;
                        cs[4 * v + 2] = x.z;
                        cs[4 * v + 3] = x.w;
                    }
#pragma unroll
                    for (int i = 0; i < kPairCands; ++i) {
                        if (p < 0 && cs[i] >= 0 && cs[i] < nQ && part[cs[i]] < 0) p = cs[i];
                    }
                }
                prop[a] = p;
            }
            __syncthreads();
        }
        for (int a = threadIdx.x; a < nQ; a += blockDim.x) {
            const int c = prop[a];
            if (c >= 0 && c < nQ && part[a] < 0 && prop[c] == a) part[a] = c;
        }
        __syncthreads();
    }
    for (int a = threadIdx.x; a < nQ; a += blockDim.x) ws.partner[base + a] = part[a];
    if (threadIdx.x >= 32) return;

    const int lane = threadIdx.x;
    const int nP = (nQ + 1) / 2;
    int32_t* out = pair_order + (size_t)bh * 2 * nP;
    int pos = 0;
    // matched pairs, by their lower block
    for (int a0 = 0; a0 < nQ; a0 += 32) {
        const int a = a0 + lane;
        const int pa = a < nB ? part[a] : -1;
        const bool lead = a < nB && pa > a;
        const uint32_t bal = __ballot_sync(0xffffffffu, lead);
        if (lead) {
            const int slot = pos + 2 * __popc(bal & ((1u << lane) - 1u));
            out[slot] = a;
            out[slot + 1] = pa;
        }
        pos += 2 * __popc(bal);
    }
    // unmatched valid blocks, then blocks past the valid length, two by two
    for (int pass = 0; pass < 2; ++pass) {
        for (int a0 = 0; a0 < nQ; a0 += 32) {
            const int a = a0 + lane;
            const bool take = pass == 0 ? (a < nB && part[a] < 0) : (a >= nB && a < nQ);
            const uint32_t bal = __ballot_sync(0xffffffffu, take);
            if (take) out[pos + __popc(bal & ((1u << lane) - 1u))] = a;
            pos += __popc(bal);
        }
    }
    if (lane == 0 && pos < 2 * nP) out[pos] = -1;
}

}  // namespace sba

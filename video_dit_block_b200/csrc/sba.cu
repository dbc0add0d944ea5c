// sba.cu -- host side of the C ABI declared in include/sba.h: argument checks,
// TMA tensor-map encoding, launches and the device status word.  The whole
// library is this one translation unit (kernels come from the .cuh files).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/sba.h"
#include "attention.cuh"
#include "attention2.cuh"
#include "common.cuh"
#include "select.cuh"
#include "select_fused.cuh"
#include "score_lse.cuh"
#include "pair.cuh"
#include "producer.cuh"
#include "compensation.cuh"
#include "prune.cuh"

namespace {

constexpr uint64_t kDefaultWaitLimit = 1ull << 32;  // clock cycles, ~2 s at 2 GHz
uint64_t g_wait_limit = kDefaultWaitLimit;
int g_attn_kernel = SBA_ATTN_KERNEL_AUTO;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up_256(size_t x) { return (x + 255) & ~size_t(255); }

sba_status check_shape(int B, int H, int Npad, int D, int block) {
    if (B <= 0 || H <= 0 || Npad <= 0) return SBA_ERR_INVALID_ARG;
    if (B > 65535 || H > 65535) return SBA_ERR_UNSUPPORTED;
    if (D != 64 && D != 128) return SBA_ERR_UNSUPPORTED;
    if (block != 64) return SBA_ERR_UNSUPPORTED;
    if (Npad % block != 0) return SBA_ERR_INVALID_ARG;
    if (Npad > SBA_MAX_NPAD) return SBA_ERR_UNSUPPORTED;
    return SBA_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [B*H, Npad, D] bf16 viewed as a 3-D tensor; box = 64 columns (128 B) x rows x 1,
// 128-byte swizzle (the canonical K-major / MN-major SW128 operand layout).
bool make_map(CUtensorMap* map, const void* base, int BH, int Npad, int D, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Npad, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Npad * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Row-major [rows][cols] bf16 as a 2-D tensor; box = 64 columns (128 B) x box_rows,
// 128-byte swizzle.
bool make_map_2d(CUtensorMap* map, const void* base, long long rows, int cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The key means of one head sampled every `stride` blocks: [BH][nB][D] bf16 viewed as
// 3-D (D, floor(nB / stride), BH) with row pitch stride * D * 2 bytes; box 64 x 128 rows.
bool make_map_sample(CUtensorMap* map, const void* base, int BH, int nB, int D, int stride) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)(nB / stride), (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)stride * D * 2, (cuuint64_t)nB * D * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Where the epilogue stores the output when it goes straight to sequence shards.
struct ShardOut {
    int n;
    int h_total;
    int h_first;
    void* const* o;
    float* const* lse;  // NULL: no lse
};

// kbar / vbar (kMeanComp only): bf16 [BH][nBpad][D] block means for the compensation steps.
template <int D, int NS, int MODE = sba::kPlain>
sba_status launch_attention(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int H, int Npad, const int32_t* valid_len,
                            const int32_t* kv_idx, const int32_t* kv_cnt, int kmax, int dense,
                            const int32_t* pair_order, float softmax_scale, cudaStream_t stream,
                            const void* kbar = nullptr, const void* vbar = nullptr, int nBpad = 0,
                            const ShardOut* shards = nullptr) {
    using SM = sba::AttnSmem<D, NS>;
    CUtensorMap tq, tk, tv, tkb, tvb;
    const int BH = B * H;
    if (!make_map(&tq, q, BH, Npad, D, 64) || !make_map(&tk, k, BH, Npad, D, 64) ||
        !make_map(&tv, v, BH, Npad, D, 64))
        return SBA_ERR_CUDA;
    if (MODE == sba::kMeanComp) {
        if (!make_map(&tkb, kbar, BH, nBpad, D, 64) || !make_map(&tvb, vbar, BH, nBpad, D, 64)) return SBA_ERR_CUDA;
    } else {
        tkb = tk;
        tvb = tv;
    }
    const void* fn = MODE == sba::kMeanComp      ? (const void*)sba::attn_comp_kernel<D, NS>
                     : MODE == sba::kFirstOrder ? (const void*)sba::attn_first_order_kernel<D, NS>
                                                : (const void*)sba::attn_kernel<D, NS>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc) != cudaSuccess)
        return SBA_ERR_CUDA;
    sba::AttnParams p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.valid_len = valid_len;
    p.kv_idx = kv_idx;
    p.kv_cnt = kv_cnt;
    p.pair_order = pair_order;
    p.H = H;
    p.Npad = Npad;
    p.kmax = kmax;
    p.dense = dense;
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)D);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.wait_limit = g_wait_limit;
    if (shards) {
        p.n_shards = shards->n;
        p.shard_len = Npad / shards->n;
        p.h_total = shards->h_total;
        p.h_first = shards->h_first;
        for (int i = 0; i < shards->n; ++i) {
            p.o_shard[i] = static_cast<__nv_bfloat16*>(shards->o[i]);
            p.lse_shard[i] = shards->lse ? shards->lse[i] : nullptr;
        }
    }
    dim3 grid((Npad / 64 + 1) / 2, H, B);
    if (MODE == sba::kMeanComp)
        sba::attn_comp_kernel<D, NS><<<grid, 192, SM::kAlloc, stream>>>(tq, tk, tv, tkb, tvb, p);
    else if (MODE == sba::kFirstOrder)
        sba::attn_first_order_kernel<D, NS><<<grid, 192, SM::kAlloc, stream>>>(tq, tk, tv, p);
    else
        sba::attn_kernel<D, NS><<<grid, 192, SM::kAlloc, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

// The CTA-pair kernel (D = 128): four query blocks per 2-SM cluster, two key blocks
// per step.
template <int NS>
sba_status launch_attention_pair(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                 int Npad, const int32_t* valid_len, const int32_t* kv_idx, const int32_t* kv_cnt,
                                 int kmax, int dense, float softmax_scale, cudaStream_t stream) {
    using SM = sba::Attn2Smem<NS>;
    CUtensorMap tq, tk, tv;
    const int BH = B * H;
    if (!make_map(&tq, q, BH, Npad, 128, 64) || !make_map(&tk, k, BH, Npad, 128, 64) ||
        !make_map(&tv, v, BH, Npad, 128, 64))
        return SBA_ERR_CUDA;
    if (cudaFuncSetAttribute(sba::attn_pair_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kAlloc) !=
        cudaSuccess)
        return SBA_ERR_CUDA;
    sba::AttnParams p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.valid_len = valid_len;
    p.kv_idx = kv_idx;
    p.kv_cnt = kv_cnt;
    p.pair_order = nullptr;
    p.H = H;
    p.Npad = Npad;
    p.kmax = kmax;
    p.dense = dense;
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(128.0f);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.wait_limit = g_wait_limit;
    const int nQ = Npad / 64;
    dim3 grid(2 * ((nQ + 3) / 4), H, B);
    sba::attn_pair_kernel<NS><<<grid, 320, SM::kAlloc, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

// Routing launches shared by both routers: pool Q and K (blocks, or NSUB
// sub-blocks per block), largest key norm, screened scores on the tensor cores
// (skipped when nothing is dropped), then the per-row top-k.  Arguments checked
// by the caller.
// With qmean/kmean given (fp64 block means [BH][nB][D], NSUB = 1), pooling is replaced
// by splitting those means for the screen, and the top-k re-scores from them.
template <int D, int NSUB>
sba_status run_select(const void* q, const void* k, int B, int H, int Npad, const int32_t* valid_len,
                      double sparsity, int budget, int kmax, int32_t* kv_idx, int32_t* kv_cnt,
                      void* workspace, cudaStream_t s, const double* qmean = nullptr,
                      const double* kmean = nullptr) {
    constexpr int BLK = 64 / NSUB;
    const size_t BH = (size_t)B * H;
    const int nB = Npad / 64;
    const int nP = nB * NSUB;
    sba::SelectWorkspace ws = sba::carve_select_workspace(workspace, BH, nB, D, NSUB);
    const long long pgroups = (long long)BH * nP;
    const int gpc = 256 / (D / 8);  // pooled rows per CTA
    const unsigned pool_grid = (unsigned)((pgroups + gpc - 1) / gpc);
    const long long rows = (long long)BH * nB;
    const int wpb = 8;              // top-k: one warp per routing row
    const size_t tsmem = sba::topk_smem(wpb, ws.ld);
    if (tsmem > 227 * 1024) return SBA_ERR_UNSUPPORTED;
    const unsigned tgrid = (unsigned)((rows + wpb - 1) / wpb);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const bool need_scores = sparsity > 0.0;
    CUtensorMap tqh, tql, tkh, tkl, tks;
    const int sample_stride = nB / 128 > 1 ? nB / 128 : 1;  // the fused screen's range sample
    if (NSUB == 1 && BH > 65535) return SBA_ERR_UNSUPPORTED;  // grid.y of the fused screen
    if ((need_scores || NSUB == 1) &&
        (!make_map(&tqh, ws.qhi, (int)BH, nP, D, 128) || !make_map(&tql, ws.qlo, (int)BH, nP, D, 128) ||
         !make_map(&tkh, ws.khi, (int)BH, nP, D, 128) || !make_map(&tkl, ws.klo, (int)BH, nP, D, 128) ||
         (NSUB == 1 && !make_map_sample(&tks, ws.khi, (int)BH, nB, D, sample_stride))))
        return SBA_ERR_CUDA;
    if (qmean && kmean) {
        ws.qmean64 = const_cast<double*>(qmean);
        ws.kmean64 = const_cast<double*>(kmean);
        sba::split_means_kernel<D><<<pool_grid, 256, 0, s>>>(qmean, ws.qhi, ws.qlo, ws.qnorm, pgroups);
        sba::split_means_kernel<D><<<pool_grid, 256, 0, s>>>(kmean, ws.khi, ws.klo, ws.knorm, pgroups);
    } else {
        // Q and K in one launch: the CTAs past pool_grid pool K
        const sba::PoolSecond kside{kb, ws.kmean64, ws.khi, ws.klo, ws.knorm, pool_grid};
        sba::pool_kernel<D, BLK><<<2 * pool_grid, 256, 0, s>>>(qb, valid_len, H, Npad, ws.qmean64, ws.qhi, ws.qlo,
                                                               ws.qnorm, pgroups, kside);
    }
    sba::kmax_kernel<<<(unsigned)((BH + 7) / 8), 256, 0, s>>>(ws, valid_len, H, Npad, (int)BH, BLK);
    if (NSUB == 1) {
        // screen and top-k in one kernel; the rows it hands back finish in topk_rest_kernel
        using SM = sba::FusedSmem<D>;
        if (cudaFuncSetAttribute(sba::select_fused_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SM::kAlloc) != cudaSuccess ||
            cudaFuncSetAttribute(sba::topk_rest_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tsmem) != cudaSuccess)
            return SBA_ERR_CUDA;
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return SBA_ERR_CUDA;
        const dim3 fgrid((unsigned)((nB + 127) / 128), (unsigned)BH);
        sba::select_fused_kernel<D><<<fgrid, sba::kFusedThreads, SM::kAlloc, s>>>(
            tqh, tql, tkh, tkl, tks, ws, valid_len, H, Npad, sample_stride, sparsity, budget, kmax, kv_idx, kv_cnt,
            g_wait_limit);
        using FS = sba::FinishSmem<D>;
        if (cudaFuncSetAttribute(sba::select_finish_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 FS::kTotal) != cudaSuccess)
            return SBA_ERR_CUDA;
        sba::select_finish_kernel<D><<<(unsigned)((rows + sba::kFinishWarps - 1) / sba::kFinishWarps),
                                       32 * sba::kFinishWarps, FS::kTotal, s>>>(ws, valid_len, H, Npad, sparsity,
                                                                               budget, kmax, kv_idx, kv_cnt, rows);
        sba::topk_rest_kernel<D><<<(unsigned)(2 * sms), 32 * wpb, tsmem, s>>>(ws, valid_len, H, Npad, sparsity,
                                                                              budget, kmax, kv_idx, kv_cnt);
        return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
    } else if (need_scores) {
        // persistent: one CTA per SM over the (b, h, query tile) items
        using SM = sba::LseSmem<D>;
        if (cudaFuncSetAttribute(sba::score_lse_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SM::kAlloc) != cudaSuccess)
            return SBA_ERR_CUDA;
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return SBA_ERR_CUDA;
        const long long items = (long long)BH * ((nP + 127) / 128);
        const unsigned grid = (unsigned)(items < sms ? items : sms);
        sba::score_lse_kernel<D><<<grid, 320, SM::kAlloc, s>>>(tqh, tql, tkh, tkl, ws.scores, nB, ws.ld, valid_len,
                                                               H, Npad, (int)BH, g_wait_limit);
    }
    if (cudaFuncSetAttribute(sba::topk_kernel<D, NSUB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsmem) !=
        cudaSuccess)
        return SBA_ERR_CUDA;
    sba::topk_kernel<D, NSUB><<<tgrid, 32 * wpb, tsmem, s>>>(ws, valid_len, H, Npad, sparsity, budget, kmax, kv_idx,
                                                             kv_cnt, rows);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

}  // namespace

extern "C" {

int32_t sba_keep_count(int32_t n_blocks, double sparsity) {
    return sba::keep_count(n_blocks, sparsity);
}

int32_t sba_keep_count_budget(int32_t n_blocks, double sparsity, int32_t budget) {
    if (budget < 1) return 0;
    return sba::keep_count_budget(n_blocks, sparsity, budget);
}

size_t sba_pool_select_workspace_size(int B, int H, int Npad, int D, int block) {
    if (check_shape(B, H, Npad, D, block) != SBA_OK) return 0;
    return sba::select_workspace_bytes((size_t)B * H, (size_t)Npad / block, (size_t)D);
}

sba_status sba_pool_select(const void* q, const void* k, int B, int H, int Npad, int D,
                           const int32_t* valid_len, int block, double sparsity, int kmax,
                           int32_t* kv_idx, int32_t* kv_cnt, void* workspace,
                           size_t workspace_bytes, void* stream) {
    sba_status st = check_shape(B, H, Npad, D, block);
    if (st != SBA_OK) return st;
    if (!q || !k || !kv_idx || !kv_cnt || !workspace) return SBA_ERR_INVALID_ARG;
    if (!(sparsity >= 0.0 && sparsity < 1.0)) return SBA_ERR_INVALID_ARG;
    const int nB = Npad / block;
    if (kmax < sba::keep_count(nB, sparsity)) return SBA_ERR_INVALID_ARG;
    if (workspace_bytes < sba::select_workspace_bytes((size_t)B * H, nB, D)) return SBA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(workspace) || !aligned16(valid_len))
        return SBA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (D == 128)
        return run_select<128, 1>(q, k, B, H, Npad, valid_len, sparsity, 1, kmax, kv_idx, kv_cnt, workspace, s);
    return run_select<64, 1>(q, k, B, H, Npad, valid_len, sparsity, 1, kmax, kv_idx, kv_cnt, workspace, s);
}

sba_status sba_pool_select_means(const double* qmean, const double* kmean, int B, int H, int Npad, int D,
                                 const int32_t* valid_len, int block, double sparsity, int kmax,
                                 int32_t* kv_idx, int32_t* kv_cnt, void* workspace, size_t workspace_bytes,
                                 void* stream) {
    sba_status st = check_shape(B, H, Npad, D, block);
    if (st != SBA_OK) return st;
    if (!qmean || !kmean || !kv_idx || !kv_cnt || !workspace) return SBA_ERR_INVALID_ARG;
    if (!(sparsity >= 0.0 && sparsity < 1.0)) return SBA_ERR_INVALID_ARG;
    const int nB = Npad / block;
    if (kmax < sba::keep_count(nB, sparsity)) return SBA_ERR_INVALID_ARG;
    if (workspace_bytes < sba::select_workspace_bytes((size_t)B * H, nB, D)) return SBA_ERR_INVALID_ARG;
    if (!aligned16(qmean) || !aligned16(kmean) || !aligned16(workspace) || !aligned16(valid_len))
        return SBA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (D == 128)
        return run_select<128, 1>(nullptr, nullptr, B, H, Npad, valid_len, sparsity, 1, kmax, kv_idx, kv_cnt,
                                  workspace, s, qmean, kmean);
    return run_select<64, 1>(nullptr, nullptr, B, H, Npad, valid_len, sparsity, 1, kmax, kv_idx, kv_cnt, workspace,
                             s, qmean, kmean);
}

sba_status sba_qk_norm_rope_pool(const void* x, const void* weight, const int32_t* pos, int B, int H, int Npad,
                                 int D, const int32_t* valid_len, int block, int rope_dim, double rope_base,
                                 float eps, void* out, double* means, void* stream) {
    sba_status st = check_shape(B, H, Npad, D, block);
    if (st != SBA_OK) return st;
    if (!x || !weight || !pos || !out) return SBA_ERR_INVALID_ARG;
    if (rope_dim < 0 || rope_dim > D || rope_dim % 6 != 0 || rope_dim / 6 > sba::kMaxRopePairs)
        return SBA_ERR_INVALID_ARG;
    if (!(rope_base > 0.0) || !std::isfinite(rope_base) || !(eps >= 0.f) || !std::isfinite(eps))
        return SBA_ERR_INVALID_ARG;
    if ((long long)B * H * (Npad / block) > 0x7fffffffll) return SBA_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(out) || !aligned16(weight) || !aligned16(means) || !aligned16(valid_len) ||
        (reinterpret_cast<uintptr_t>(pos) & 3u))
        return SBA_ERR_ALIGNMENT;
    sba::RopeFreqs f;
    const int da = rope_dim / 3;
    for (int i = 0; i < sba::kMaxRopePairs; ++i)
        f.inv_freq[i] = (da > 0 && 2 * i < da) ? (float)std::pow(rope_base, -2.0 * i / da) : 0.f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)((long long)B * H * (Npad / block));
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    const auto* wb = static_cast<const __nv_bfloat16*>(weight);
    auto* ob = static_cast<__nv_bfloat16*>(out);
    if (D == 128)
        sba::qk_norm_rope_pool_kernel<128><<<grid, 256, 0, s>>>(xb, wb, pos, valid_len, H, Npad, rope_dim, f, eps, ob,
                                                                means);
    else
        sba::qk_norm_rope_pool_kernel<64><<<grid, 256, 0, s>>>(xb, wb, pos, valid_len, H, Npad, rope_dim, f, eps, ob,
                                                               means);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

size_t sba_pool_select_lse_workspace_size(int B, int H, int Npad, int D, int block, int nsub) {
    if (check_shape(B, H, Npad, D, block) != SBA_OK || nsub != sba::kNsub) return 0;
    return sba::select_workspace_bytes((size_t)B * H, (size_t)Npad / block, (size_t)D, (size_t)nsub);
}

sba_status sba_pool_select_lse(const void* q, const void* k, int B, int H, int Npad, int D,
                               const int32_t* valid_len, int block, int nsub, double sparsity, int budget,
                               int kmax, int32_t* kv_idx, int32_t* kv_cnt, void* workspace,
                               size_t workspace_bytes, void* stream) {
    sba_status st = check_shape(B, H, Npad, D, block);
    if (st != SBA_OK) return st;
    if (nsub != sba::kNsub) return SBA_ERR_UNSUPPORTED;
    if (!q || !k || !kv_idx || !kv_cnt || !workspace) return SBA_ERR_INVALID_ARG;
    if (!(sparsity >= 0.0 && sparsity < 1.0) || budget < 1) return SBA_ERR_INVALID_ARG;
    const int nB = Npad / block;
    if (kmax < sba::keep_count_budget(nB, sparsity, budget)) return SBA_ERR_INVALID_ARG;
    if (workspace_bytes < sba::select_workspace_bytes((size_t)B * H, nB, D, nsub)) return SBA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(workspace) || !aligned16(valid_len))
        return SBA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (D == 128)
        return run_select<128, sba::kNsub>(q, k, B, H, Npad, valid_len, sparsity, budget, kmax, kv_idx, kv_cnt,
                                           workspace, s);
    return run_select<64, sba::kNsub>(q, k, B, H, Npad, valid_len, sparsity, budget, kmax, kv_idx, kv_cnt,
                                      workspace, s);
}

sba_status sba_block_means(const void* x, int B, int H, int Npad, int D, const int32_t* valid_len,
                           int block, double* out, void* stream) {
    sba_status st = check_shape(B, H, Npad, D, block);
    if (st != SBA_OK) return st;
    if (!x || !out) return SBA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out) || !aligned16(valid_len)) return SBA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long groups = (long long)B * H * (Npad / block);
    const int gpc = 256 / (D / 8);
    const unsigned grid = (unsigned)((groups + gpc - 1) / gpc);
    if (D == 128)
        sba::pool_kernel<128><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), valid_len, H,
                                                   Npad, out, nullptr, nullptr, nullptr, groups,
                                                   sba::PoolSecond{nullptr, nullptr, nullptr, nullptr, nullptr, grid});
    else
        sba::pool_kernel<64><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), valid_len, H,
                                                  Npad, out, nullptr, nullptr, nullptr, groups,
                                                   sba::PoolSecond{nullptr, nullptr, nullptr, nullptr, nullptr, grid});
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

static sba_status attention_common(const void* q, const void* k, const void* v, void* o, float* lse,
                                   int B, int H, int Npad, int D, const int32_t* valid_len,
                                   int block, const int32_t* kv_idx, const int32_t* kv_cnt,
                                   int kmax, int dense, const int32_t* pair_order,
                                   float softmax_scale, void* stream, void* comp_ws = nullptr,
                                   size_t comp_ws_bytes = 0, const ShardOut* shards = nullptr,
                                   bool first_order = false) {
    sba_status st = check_shape(B, H, Npad, D, block);
    if (st != SBA_OK) return st;
    if (!q || !k || !v || !o) return SBA_ERR_INVALID_ARG;
    if (!dense && (!kv_idx || !kv_cnt || kmax <= 0)) return SBA_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return SBA_ERR_INVALID_ARG;
    if ((long long)B * H * Npad > (1ll << 31)) return SBA_ERR_UNSUPPORTED;  // 3-D TMA row index
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(valid_len) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (kv_idx && (reinterpret_cast<uintptr_t>(kv_idx) & 3u)) ||
        (kv_cnt && (reinterpret_cast<uintptr_t>(kv_cnt) & 3u)) ||
        (pair_order && (reinterpret_cast<uintptr_t>(pair_order) & 3u)))
        return SBA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (comp_ws) {
        // compensated: the bf16 block means of K and V, then the attention with the
        // mean steps after the kept blocks
        if (dense) return SBA_ERR_INVALID_ARG;
        if (!aligned16(comp_ws)) return SBA_ERR_ALIGNMENT;
        const int nBpad = (Npad / 64 + 63) / 64 * 64;
        const size_t half = align_up_256((size_t)B * H * nBpad * D * 2);
        if (comp_ws_bytes < 2 * half) return SBA_ERR_INVALID_ARG;
        char* kbar = static_cast<char*>(comp_ws);
        char* vbar = kbar + half;
        const long long groups = (long long)B * H * nBpad;
        const int gpc = 256 / (D / 8);
        const unsigned mgrid = (unsigned)((groups + gpc - 1) / gpc);
        if (D == 128) {
            sba::block_mean_bf16_kernel<128><<<mgrid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(k), valid_len, H,
                                                                    Npad, nBpad, reinterpret_cast<__nv_bfloat16*>(kbar),
                                                                    groups);
            sba::block_mean_bf16_kernel<128><<<mgrid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(v), valid_len, H,
                                                                    Npad, nBpad, reinterpret_cast<__nv_bfloat16*>(vbar),
                                                                    groups);
            return launch_attention<128, 2, sba::kMeanComp>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt,
                                                            kmax, 0, pair_order, softmax_scale, s, kbar, vbar, nBpad);
        }
        sba::block_mean_bf16_kernel<64><<<mgrid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(k), valid_len, H, Npad,
                                                               nBpad, reinterpret_cast<__nv_bfloat16*>(kbar), groups);
        sba::block_mean_bf16_kernel<64><<<mgrid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(v), valid_len, H, Npad,
                                                               nBpad, reinterpret_cast<__nv_bfloat16*>(vbar), groups);
        return launch_attention<64, 4, sba::kMeanComp>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt, kmax,
                                                       0, pair_order, softmax_scale, s, kbar, vbar, nBpad);
    }
    if (first_order) {
        if (dense) return SBA_ERR_INVALID_ARG;
        if (D == 128)
            return launch_attention<128, 2, sba::kFirstOrder>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt,
                                                              kmax, 0, pair_order, softmax_scale, s);
        return launch_attention<64, 4, sba::kFirstOrder>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt, kmax,
                                                         0, pair_order, softmax_scale, s);
    }
    if (shards) {
        if (D == 128)
            return launch_attention<128, 2>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt, kmax, dense,
                                            pair_order, softmax_scale, s, nullptr, nullptr, 0, shards);
        return launch_attention<64, 4>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt, kmax, dense,
                                       pair_order, softmax_scale, s, nullptr, nullptr, 0, shards);
    }
    // the CTA-pair kernel only when chosen: on B200 it is slower than the query pairs on
    // every workload measured, dense included
    if (D == 128 && g_attn_kernel == SBA_ATTN_KERNEL_CTA_PAIR)
        return launch_attention_pair<4>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt, kmax, dense,
                                        softmax_scale, s);
    if (D == 128)
        return launch_attention<128, 2>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt, kmax,
                                        dense, pair_order, softmax_scale, s);
    return launch_attention<64, 4>(q, k, v, o, lse, B, H, Npad, valid_len, kv_idx, kv_cnt, kmax, dense,
                                   pair_order, softmax_scale, s);
}

sba_status sba_attention(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Npad, int D, const int32_t* valid_len, int block,
                         const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                         float softmax_scale, void* stream) {
    return attention_common(q, k, v, o, lse, B, H, Npad, D, valid_len, block, kv_idx, kv_cnt, kmax,
                            0, nullptr, softmax_scale, stream);
}

sba_status sba_attention_paired(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int Npad, int D, const int32_t* valid_len, int block,
                                const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                const int32_t* pair_order, float softmax_scale, void* stream) {
    if (!pair_order) return SBA_ERR_INVALID_ARG;
    return attention_common(q, k, v, o, lse, B, H, Npad, D, valid_len, block, kv_idx, kv_cnt, kmax,
                            0, pair_order, softmax_scale, stream);
}

sba_status sba_dense_attention(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int Npad, int D, const int32_t* valid_len,
                               float softmax_scale, void* stream) {
    return attention_common(q, k, v, o, lse, B, H, Npad, D, valid_len, 64, nullptr, nullptr, 0, 1,
                            nullptr, softmax_scale, stream);
}

sba_status sba_attention_to_shards(const void* q, const void* k, const void* v, void* const* o_shards,
                                   float* const* lse_shards, int n_shards, int h_total, int h_first, int B,
                                   int H, int Npad, int D, const int32_t* valid_len, int block,
                                   const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                   const int32_t* pair_order, float softmax_scale, void* stream) {
    if (!o_shards || n_shards < 1 || n_shards > sba::kMaxShards) return SBA_ERR_INVALID_ARG;
    if (Npad <= 0 || Npad % n_shards != 0 || h_first < 0 || H < 1 || h_total < h_first + H)
        return SBA_ERR_INVALID_ARG;
    for (int i = 0; i < n_shards; ++i) {
        if (!o_shards[i] || (lse_shards && !lse_shards[i])) return SBA_ERR_INVALID_ARG;
        if (!aligned16(o_shards[i]) || (lse_shards && (reinterpret_cast<uintptr_t>(lse_shards[i]) & 3u)))
            return SBA_ERR_ALIGNMENT;
    }
    if ((long long)B * h_total * (Npad / n_shards) > (1ll << 31)) return SBA_ERR_UNSUPPORTED;
    const ShardOut sh{n_shards, h_total, h_first, o_shards, lse_shards};
    // o is not written; any 16-byte aligned pointer passes the common checks
    return attention_common(q, k, v, o_shards[0], nullptr, B, H, Npad, D, valid_len, block, kv_idx, kv_cnt, kmax, 0,
                            pair_order, softmax_scale, stream, nullptr, 0, &sh);
}

size_t sba_mean_compensation_workspace_size(int B, int H, int Npad, int D, int block) {
    if (check_shape(B, H, Npad, D, block) != SBA_OK) return 0;
    const int nBpad = (Npad / 64 + 63) / 64 * 64;
    return 2 * align_up_256((size_t)B * H * nBpad * D * 2);
}

sba_status sba_attention_mean_compensated(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                          int H, int Npad, int D, const int32_t* valid_len, int block,
                                          const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                          const int32_t* pair_order, float softmax_scale, void* workspace,
                                          size_t workspace_bytes, void* stream) {
    if (!workspace) return SBA_ERR_INVALID_ARG;
    return attention_common(q, k, v, o, lse, B, H, Npad, D, valid_len, block, kv_idx, kv_cnt, kmax, 0,
                            pair_order, softmax_scale, stream, workspace, workspace_bytes);
}

sba_status sba_attention_compensated(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                     int H, int Npad, int D, const int32_t* valid_len, int block,
                                     const int32_t* kv_idx, const int32_t* kv_cnt, int kmax,
                                     const int32_t* pair_order, float softmax_scale, void* stream) {
    return attention_common(q, k, v, o, lse, B, H, Npad, D, valid_len, block, kv_idx, kv_cnt, kmax, 0,
                            pair_order, softmax_scale, stream, nullptr, 0, nullptr, true);
}

sba_status sba_get_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SBA_ERR_CUDA;
    int word = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&word, sba::g_device_error, sizeof(int)) != cudaSuccess) return SBA_ERR_CUDA;
    if (cudaMemcpyToSymbol(sba::g_device_error, &zero, sizeof(int)) != cudaSuccess) return SBA_ERR_CUDA;
    if (word == sba::kErrTimeout) return SBA_ERR_TIMEOUT;
    if (word != 0) return SBA_ERR_DEVICE_FLAG;
    return SBA_OK;
}

void sba_set_wait_limit(uint64_t cycles) { g_wait_limit = cycles ? cycles : kDefaultWaitLimit; }

sba_status sba_set_attention_kernel(int which) {
    if (which != SBA_ATTN_KERNEL_AUTO && which != SBA_ATTN_KERNEL_QUERY_PAIRS && which != SBA_ATTN_KERNEL_CTA_PAIR)
        return SBA_ERR_INVALID_ARG;
    g_attn_kernel = which;
    return SBA_OK;
}

const char* sba_strerror(sba_status status) {
    switch (status) {
        case SBA_OK: return "ok";
        case SBA_ERR_INVALID_ARG: return "invalid argument";
        case SBA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
        case SBA_ERR_ALIGNMENT: return "misaligned device pointer";
        case SBA_ERR_CUDA: return "CUDA call failed";
        case SBA_ERR_TIMEOUT: return "a kernel wait gave up";
        case SBA_ERR_DEVICE_FLAG: return "a kernel found an invalid routing entry";
        case SBA_ERR_SCRATCH_TOO_SMALL: return "problem needs more scratch than the fixed no-allocation buffer holds";
    }
    return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------- token pruning
extern "C" int32_t sba_keep_token_count(int32_t n_tokens, double keep_ratio) {
    if (!(keep_ratio >= 0.0 && keep_ratio <= 1.0)) return 0;
    return sba::keep_tokens(n_tokens, keep_ratio);
}

extern "C" size_t sba_token_prune_workspace_size(int B, int N) {
    if (B <= 0 || N <= 0 || (long long)B * N > 0x7fffffffll) return 0;
    return align_up_256((size_t)B * N * sizeof(double));
}

extern "C" sba_status sba_token_prune_select(const void* x, int B, int N, int C, const int32_t* valid_len,
                                             double keep_ratio, int Npad_out, int32_t* idx, int32_t* valid_len_out,
                                             void* workspace, size_t workspace_bytes, void* stream) {
    if (B <= 0 || N <= 0 || C <= 0 || Npad_out <= 0) return SBA_ERR_INVALID_ARG;
    if ((long long)B * N > 0x7fffffffll || B > 65535 || C > (1 << 20)) return SBA_ERR_UNSUPPORTED;
    if (C % 8 != 0) return SBA_ERR_UNSUPPORTED;
    if (!x || !idx || !valid_len_out || !workspace) return SBA_ERR_INVALID_ARG;
    if (!(keep_ratio >= 0.0 && keep_ratio <= 1.0)) return SBA_ERR_INVALID_ARG;
    if (Npad_out < sba::keep_tokens(N, keep_ratio)) return SBA_ERR_INVALID_ARG;
    if (workspace_bytes < (size_t)B * N * sizeof(double)) return SBA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(workspace) || !aligned16(valid_len) ||
        (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(valid_len_out) & 3u))
        return SBA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap tx;
    const long long rows = (long long)B * N;
    if (!make_map_2d(&tx, x, rows, C, sba::kNormRows)) return SBA_ERR_CUDA;
    if (cudaFuncSetAttribute(sba::token_norm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sba::kNormSmem) !=
        cudaSuccess)
        return SBA_ERR_CUDA;
    double* norm2 = static_cast<double*>(workspace);
    const unsigned grid = (unsigned)((rows + sba::kNormRows - 1) / sba::kNormRows);
    sba::token_norm_kernel<<<grid, 160, sba::kNormSmem, s>>>(tx, valid_len, N, C, rows, norm2, g_wait_limit);
    sba::prune_select_kernel<<<(unsigned)B, 1024, 0, s>>>(norm2, valid_len, N, keep_ratio, Npad_out, idx,
                                                           valid_len_out);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

extern "C" sba_status sba_gather_tokens(const void* src, int B, int H, int N, int row_bytes, const int32_t* idx,
                                        const int32_t* valid_len_out, int Npad_out, void* dst, void* stream) {
    if (B <= 0 || H <= 0 || N <= 0 || Npad_out <= 0 || row_bytes <= 0) return SBA_ERR_INVALID_ARG;
    if (row_bytes % 4 != 0) return SBA_ERR_UNSUPPORTED;
    if ((long long)B * H > 65535 || (long long)Npad_out * (row_bytes / 4) > 0x7fffffffll ||
        (long long)N * (row_bytes / 4) > 0x7fffffffll)
        return SBA_ERR_UNSUPPORTED;
    if (!src || !dst || !idx || !valid_len_out) return SBA_ERR_INVALID_ARG;
    const int unit = row_bytes % 16 == 0 ? 16 : 4;
    const uintptr_t am = (uintptr_t)unit - 1;
    if ((reinterpret_cast<uintptr_t>(src) & am) || (reinterpret_cast<uintptr_t>(dst) & am) ||
        (reinterpret_cast<uintptr_t>(idx) & 3u) || (reinterpret_cast<uintptr_t>(valid_len_out) & 3u))
        return SBA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const long long units = (long long)Npad_out * (row_bytes / unit);   // per (b, h)
    const dim3 grid((unsigned)((units + 4 * 256 - 1) / (4 * 256)), (unsigned)(B * H));
    const auto* sp = static_cast<const unsigned char*>(src);
    auto* dp = static_cast<unsigned char*>(dst);
    if (unit == 16)
        sba::gather_rows_kernel<16><<<grid, 256, 0, s>>>(sp, dp, idx, valid_len_out, H, N, row_bytes, Npad_out);
    else
        sba::gather_rows_kernel<4><<<grid, 256, 0, s>>>(sp, dp, idx, valid_len_out, H, N, row_bytes, Npad_out);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

// ---------------------------------------------------------------- query-block pairing
extern "C" size_t sba_pair_workspace_size(int B, int H, int Npad, int block) {
    if (check_shape(B, H, Npad, 64, block) != SBA_OK) return 0;
    return sba::pair_workspace_bytes((size_t)B * H, (size_t)Npad / block);
}

extern "C" sba_status sba_pair_query_blocks(const int32_t* kv_idx, const int32_t* kv_cnt, int B, int H,
                                            int Npad, int kmax, const int32_t* valid_len, int block,
                                            int32_t* pair_order, void* workspace,
                                            size_t workspace_bytes, void* stream) {
    sba_status st = check_shape(B, H, Npad, 64, block);
    if (st != SBA_OK) return st;
    if (!kv_idx || !kv_cnt || !pair_order || !workspace || kmax <= 0) return SBA_ERR_INVALID_ARG;
    const int nQ = Npad / block;
    const size_t BH = (size_t)B * H;
    if (workspace_bytes < sba::pair_workspace_bytes(BH, nQ)) return SBA_ERR_INVALID_ARG;
    if (!aligned16(workspace) || !aligned16(valid_len) || (reinterpret_cast<uintptr_t>(kv_idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(kv_cnt) & 3u) || (reinterpret_cast<uintptr_t>(pair_order) & 3u))
        return SBA_ERR_ALIGNMENT;
    const long long rows = (long long)BH * nQ;
    const int tiles_per_bh = (nQ + sba::kPairWarps - 1) / sba::kPairWarps;
    // every grid below is one dimension of at most 2^31 - 1 CTAs
    if ((rows + 7) / 8 > 0x7fffffffLL || (long long)BH * tiles_per_bh > 0x7fffffffLL) return SBA_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    sba::PairWorkspace ws = sba::carve_pair_workspace(workspace, BH, nQ);
    const unsigned wgrid = (unsigned)((rows + 7) / 8);   // 8 warps per 256-thread CTA
    sba::pair_bitmap_kernel<<<wgrid, 256, 8 * ((nQ + 31) / 32) * 4, s>>>(ws, kv_idx, kv_cnt, nQ, kmax, rows);
    const int W = (nQ + 31) / 32;
    const size_t psmem = (size_t)sba::kPairSpan * sba::pair_row_words(W) * 4;  // <= 144 x 132 x 4 = 76 KB
    if (cudaFuncSetAttribute(sba::pair_propose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)psmem) != cudaSuccess)
        return SBA_ERR_CUDA;
    sba::pair_propose_kernel<<<(unsigned)(BH * tiles_per_bh), 32 * sba::kPairWarps, psmem, s>>>(
        ws, kv_cnt, valid_len, H, nQ, tiles_per_bh);
    const size_t msmem = (size_t)2 * nQ * 4;  // <= 2 x 4096 x 4 = 32 KB
    if (cudaFuncSetAttribute(sba::pair_match_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)msmem) != cudaSuccess)
        return SBA_ERR_CUDA;
    sba::pair_match_kernel<<<(unsigned)BH, sba::kPairMatchThreads, msmem, s>>>(ws, valid_len, H, nQ, pair_order);
    return cudaGetLastError() == cudaSuccess ? SBA_OK : SBA_ERR_CUDA;
}

// ---------------------------------------------------------------- routing without allocation
// Scratch for sba_pool_select_noalloc: a fixed array in device memory that every
// GPU loading this library holds until the process exits.  In host code its name is
// only a handle; host code resolves its device address with cudaGetSymbolAddress
// and passes that address to sba_pool_select as the workspace.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device, resolved once per device
// (on the first call there, under the lock).
sba_status noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SBA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SBA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SBA_OK;
}
}  // namespace

extern "C" size_t sba_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" sba_status sba_pool_select_noalloc(const void* q, const void* k, int B, int H, int Npad,
                                              int D, const int32_t* valid_len, int block,
                                              double sparsity, int kmax, int32_t* kv_idx,
                                              int32_t* kv_cnt, void* stream) {
    // the argument checks of sba_pool_select first, so that a bad argument is reported
    // as such whatever the problem size
    sba_status st = check_shape(B, H, Npad, D, block);
    if (st != SBA_OK) return st;
    if (!q || !k || !kv_idx || !kv_cnt) return SBA_ERR_INVALID_ARG;
    if (!(sparsity >= 0.0 && sparsity < 1.0)) return SBA_ERR_INVALID_ARG;
    if (kmax < sba::keep_count(Npad / block, sparsity)) return SBA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(valid_len)) return SBA_ERR_ALIGNMENT;
    const size_t need = sba::select_workspace_bytes((size_t)B * H, (size_t)Npad / block, (size_t)D);
    if (need > kNoAllocScratchBytes) return SBA_ERR_SCRATCH_TOO_SMALL;
    void* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != SBA_OK) return st;
    return sba_pool_select(q, k, B, H, Npad, D, valid_len, block, sparsity, kmax, kv_idx, kv_cnt,
                           scratch, kNoAllocScratchBytes, stream);
}

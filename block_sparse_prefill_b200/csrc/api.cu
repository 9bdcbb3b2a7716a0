// api.cu -- the C ABI (include/fp2.h): argument checks, workspace layout,
// TMA descriptors and kernel launches.  No allocation; the only global state is
// the cached driver entry point of cuTensorMapEncodeTiled and, for the
// allocation-free entry point, its static device scratch array and the cached
// addresses of that array per device.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace fp2;

namespace {

constexpr size_t kMaxSmem = 232448;  // 227 KB opt-in per CTA on sm_100

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
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

// 3-D map over [rows, heads, 128] (token-major) with 128-byte-swizzled boxes of
// 128 rows x one head x 128 bytes.
bool make_map(CUtensorMap* m, const void* base, bool e4m3, int64_t heads, int64_t rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t esz = e4m3 ? 1 : 2;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(heads),
                                static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
    const cuuint64_t strides[2] = {kHeadDim * esz, kHeadDim * esz * static_cast<cuuint64_t>(heads)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [rows, heads, d] without swizzle, box of 32 rows x hb heads x d (the pooling stages).
bool make_map_pool(CUtensorMap* m, const void* base, bool e4m3, int64_t heads, int64_t rows,
                   int32_t hb) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t esz = e4m3 ? 1 : 2;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(heads),
                                static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
    const cuuint64_t strides[2] = {kHeadDim * esz, kHeadDim * esz * static_cast<cuuint64_t>(heads)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kHeadDim), static_cast<cuuint32_t>(hb), 32};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 map over [rows, 128] with 128-byte-swizzled boxes of 128 rows x 64 columns.
bool make_map_2d(CUtensorMap* m, const void* base, int64_t rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
    const cuuint64_t strides[1] = {kHeadDim * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int32_t esize(const fp2_params* p) { return p->dtype == FP2_E4M3 ? 1 : 2; }

fp2_status check_params(const fp2_params* p) {
    if (!p) return FP2_ERR_INVALID_ARG;
    if (p->num_q_heads < 1 || p->num_kv_heads < 1 || p->num_q_heads % p->num_kv_heads != 0)
        return FP2_ERR_INVALID_ARG;
    if (p->dtype != FP2_BF16 && p->dtype != FP2_E4M3) return FP2_ERR_INVALID_ARG;
    if (p->correction < 0 || p->correction > 2) return FP2_ERR_INVALID_ARG;
    if (std::isnan(p->alpha) || p->alpha > 1.f) return FP2_ERR_INVALID_ARG;
    if (!std::isfinite(p->sm_scale) || p->sm_scale < 0.f) return FP2_ERR_INVALID_ARG;
    if (p->head_dim <= 0 || p->block_size <= 0) return FP2_ERR_INVALID_ARG;
    if (p->head_dim != kHeadDim || p->block_size != kBlock) return FP2_ERR_UNSUPPORTED;
    if (p->dtype == FP2_E4M3 && (!p->q_scale || !p->k_scale || !p->v_scale))
        return FP2_ERR_INVALID_ARG;
    return FP2_OK;
}

float tau_of(const fp2_params* p) {
    return p->sm_scale > 0.f ? p->sm_scale : 1.f / std::sqrt(static_cast<float>(p->head_dim));
}

struct Problem {
    int32_t batch;
    int64_t total_q;      // query rows (= total_k for plain prefill)
    int64_t total_k;      // keys
    int32_t max_seqlen;   // >= every request's keys
    int64_t max_blocks;   // host bound of the key blocks sum_b ceil(Lk_b / bs) (>= q-blocks)
    int64_t max_qblocks;  // host bound of the q-blocks (<= max_blocks)
    int32_t nb_need;      // ceil(max_seqlen / block)
    WsLayout ws;
};

// Plain prefill passes the same cu_seqlens and total for queries and keys.
fp2_status check_problem(const fp2_params* p, const void* q, const void* k, const void* v,
                         const int32_t* cu_q, const int32_t* cu_k, int32_t batch, int64_t total_q,
                         int64_t total_k, int32_t max_seqlen, void* workspace, size_t ws_bytes,
                         Problem* out) {
    fp2_status st = check_params(p);
    if (st != FP2_OK) return st;
    if (batch < 0 || total_q < 0 || total_k < 0 || max_seqlen < 0) return FP2_ERR_INVALID_ARG;
    if (total_q > total_k) return FP2_ERR_INVALID_ARG;
    if (total_k > (int64_t(1) << 31) - 1) return FP2_ERR_UNSUPPORTED;
    if (batch > 0 && (!cu_q || !cu_k)) return FP2_ERR_INVALID_ARG;
    if ((total_q > 0 && !q) || (total_k > 0 && (!k || !v))) return FP2_ERR_INVALID_ARG;
    if ((q && !aligned(q, 16)) || (k && !aligned(k, 16)) || (v && !aligned(v, 16)))
        return FP2_ERR_INVALID_ARG;
    out->batch = batch;
    out->total_q = total_q;
    out->total_k = total_k;
    out->max_seqlen = max_seqlen;
    out->max_blocks = fp2_max_blocks(batch, total_k, kBlock);
    // a request's q-blocks: at most ceil(Lq / bs) + 1 (the first one partial)
    out->max_qblocks = std::min<int64_t>(out->max_blocks, fp2_max_blocks(batch, total_q, kBlock) + batch);
    out->nb_need = (max_seqlen + kBlock - 1) / kBlock;
    out->ws = ws_layout(batch, out->max_blocks, p->num_q_heads, p->num_kv_heads, esize(p));
    if (!workspace || !aligned(workspace, 256) || ws_bytes < out->ws.total) return FP2_ERR_WORKSPACE;
    return FP2_OK;
}

fp2_status check_meta(const fp2_blockmeta* m, const fp2_params* p, const Problem& pr, bool need_v) {
    if (!m || !m->kept_cnt || !m->kept_idx || !m->k_mean) return FP2_ERR_INVALID_ARG;
    if (need_v && p->correction && !m->v_mean) return FP2_ERR_INVALID_ARG;
    if (need_v && p->correction == 2 && !m->k_var) return FP2_ERR_INVALID_ARG;
    if (m->nb_max < pr.nb_need || m->nb_max < 1) return FP2_ERR_INVALID_ARG;
    if (m->max_blocks < 0) return FP2_ERR_INVALID_ARG;
    if (!aligned(m->k_mean, 16) || (m->v_mean && !aligned(m->v_mean, 16))) return FP2_ERR_INVALID_ARG;
    return FP2_OK;
}

template <class T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

fp2_status launched(cudaError_t e) { return e == cudaSuccess ? FP2_OK : FP2_ERR_CUDA; }

// Score-kernel tiling: q-blocks per 128-row tile (rows = q-block x query head).
bool score_tiling(int32_t G, int32_t* qt) {
    if (G < 1 || G > 128) return false;
    *qt = 128 / G;
    return true;
}

// Size limits of the kernels, checked before anything is enqueued: the setup
// kernel's per-index histogram and the attention kernel's per-item kept-list
// staging live in shared memory, and the score kernel's grid has at most 65535
// tiles in y.
fp2_status check_limits(const fp2_params* p, const Problem& pr, bool estimate, bool attention) {
    const int32_t nb_cap = pr.nb_need > 0 ? pr.nb_need : 1;
    if (sizeof(int32_t) * (setup_bins(nb_cap, attention) + 1) > kMaxSmem) return FP2_ERR_UNSUPPORTED;
    if (estimate) {
        int32_t qt;
        if (!score_tiling(p->num_q_heads / p->num_kv_heads, &qt)) return FP2_ERR_UNSUPPORTED;
        if ((pr.max_qblocks + qt - 1) / qt + pr.batch > 65535) return FP2_ERR_UNSUPPORTED;
    }
    if (attention && attn_smem_bytes(p->dtype == FP2_E4M3, pr.nb_need, p->correction == 2) > kMaxSmem)
        return FP2_ERR_UNSUPPORTED;
    return FP2_OK;
}

// kept_cnt != NULL (the attention call): work items ordered by cost.
fp2_status run_setup(const Problem& pr, void* ws, const int32_t* cu_q, const int32_t* cu_k, int32_t qt,
                     bool paged, int32_t mbps, int64_t meta_blocks, cudaStream_t s,
                     const int32_t* kept_cnt = nullptr, int32_t hkv = 0, int32_t correction = 0) {
    SetupArgs sa;
    sa.cu_q = cu_q;
    sa.cu_k = cu_k;
    sa.batch = pr.batch;
    sa.total_q = pr.total_q;
    sa.total_k = pr.total_k;
    sa.max_seqlen = pr.max_seqlen;
    sa.qt = qt;
    sa.paged = paged ? 1 : 0;
    sa.max_blocks_per_seq = mbps;
    sa.max_blocks = meta_blocks < pr.max_blocks ? meta_blocks : pr.max_blocks;
    sa.nb_cap = pr.nb_need > 0 ? pr.nb_need : 1;
    sa.hdr = at<WsHeader>(ws, 0);
    sa.cu_blocks = at<int32_t>(ws, pr.ws.cu_blocks);
    sa.cu_qblocks = at<int32_t>(ws, pr.ws.cu_qblocks);
    sa.cu_tiles = at<int32_t>(ws, pr.ws.cu_tiles);
    sa.blk_req = at<int32_t>(ws, pr.ws.blk_req);
    sa.blk_req_q = at<int32_t>(ws, pr.ws.blk_req_q);
    sa.order = at<int32_t>(ws, pr.ws.order);
    sa.kept_cnt = kept_cnt;
    sa.hkv = hkv;
    sa.correction = correction;
    const size_t hist_bytes = sizeof(int32_t) * (setup_bins(sa.nb_cap, kept_cnt != nullptr) + 1);
    if (hist_bytes > kMaxSmem) return FP2_ERR_UNSUPPORTED;
    if (hist_bytes > 48 * 1024 &&
        cudaFuncSetAttribute(setup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(hist_bytes)) != cudaSuccess)
        return FP2_ERR_CUDA;
    setup_kernel<<<1, 256, hist_bytes, s>>>(sa);
    return launched(cudaGetLastError());
}

fp2_status run_estimate(const fp2_params* p, const void* q, const void* k, const void* v,
                        const int32_t* cu_q, const int32_t* cu_k, const Problem& pr,
                        const int32_t* block_table, int32_t mbps, int32_t num_pages,
                        fp2_blockmeta* meta, void* ws, cudaStream_t s) {
    const int32_t G = p->num_q_heads / p->num_kv_heads;
    fp2_status st = check_limits(p, pr, true, false);
    if (st != FP2_OK) return st;
    int32_t qt;
    score_tiling(G, &qt);
    st = run_setup(pr, ws, cu_q, cu_k, qt, block_table != nullptr, mbps, meta->max_blocks, s);
    // a batch without query rows ends after the setup kernel has checked the
    // cu_seqlens arrays: there is no q-block to score
    if (st != FP2_OK || pr.batch == 0 || pr.total_q == 0) return st;

    const bool e4m3 = p->dtype == FP2_E4M3;
    WsHeader* hdr = at<WsHeader>(ws, 0);
    PoolArgs pa;
    memset(&pa, 0, sizeof(pa));
    pa.out[0] = nullptr;
    pa.out[1] = meta->k_mean;
    pa.out[2] = meta->v_mean;
    pa.kvar = meta->k_var;
    pa.split[0] = at<uint16_t>(ws, pr.ws.qsplit);
    pa.split[1] = at<uint16_t>(ws, pr.ws.ksplit);
    pa.G = G;
    pa.max_blocks = pr.max_blocks;
    pa.scale[0] = e4m3 ? p->q_scale : nullptr;
    pa.scale[1] = e4m3 ? p->k_scale : nullptr;
    pa.scale[2] = e4m3 ? p->v_scale : nullptr;
    pa.heads[0] = p->num_q_heads;
    pa.heads[1] = p->num_kv_heads;
    pa.heads[2] = p->num_kv_heads;
    // a slab is at most 2 KB of a row (8 bf16 or 16 e4m3 heads): 32 rows = one 64 KB stage
    const int32_t hb_max = e4m3 ? 16 : 8;
    for (int x = 0; x < 3; ++x) {
        pa.hb[x] = pa.heads[x] < hb_max ? pa.heads[x] : hb_max;
        pa.slabs[x] = (pa.heads[x] + pa.hb[x] - 1) / pa.hb[x];
    }
    pa.paged[0] = 0;
    pa.paged[1] = pa.paged[2] = block_table ? 1 : 0;
    pa.first = 0;
    pa.last = meta->v_mean ? 3 : 2;
    pa.cu_q = cu_q;
    pa.cu_k = cu_k;
    pa.cu_blocks = at<int32_t>(ws, pr.ws.cu_blocks);
    pa.cu_qblocks = at<int32_t>(ws, pr.ws.cu_qblocks);
    pa.blk_req = at<int32_t>(ws, pr.ws.blk_req);
    pa.blk_req_q = at<int32_t>(ws, pr.ws.blk_req_q);
    pa.block_table = block_table;
    pa.max_blocks_per_seq = mbps;
    pa.num_pages = num_pages;
    pa.hdr = hdr;
    const int32_t yskv = pa.slabs[1] + (pa.last == 3 ? pa.slabs[2] : 0);
    const int64_t kv_rows = block_table ? int64_t(num_pages) * kBlock : pr.total_k;
    CUtensorMap pq, pk, pv;
    if (!make_map_pool(&pq, q, e4m3, p->num_q_heads, pr.total_q, pa.hb[0]) ||
        !make_map_pool(&pk, k, e4m3, p->num_kv_heads, kv_rows, pa.hb[1]) ||
        !make_map_pool(&pv, v, e4m3, p->num_kv_heads, kv_rows, pa.hb[2]))
        return FP2_ERR_CUDA;
    // persistent: one CTA per SM (the stage ring fills most of shared memory)
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return FP2_ERR_CUDA;
    const int64_t units = pr.max_qblocks * pa.slabs[0] + pr.max_blocks * yskv;
    const unsigned pgrid = static_cast<unsigned>(units < sms ? units : sms);
    const size_t psmem = pool_smem_bytes(e4m3);
    if (cudaFuncSetAttribute(e4m3 ? pool_kernel<true> : pool_kernel<false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(psmem)) != cudaSuccess)
        return FP2_ERR_CUDA;
    if (e4m3)
        pool_kernel<true><<<pgrid, kPoolThreads, psmem, s>>>(pa, pq, pk, pv);
    else
        pool_kernel<false><<<pgrid, kPoolThreads, psmem, s>>>(pa, pq, pk, pv);
    if ((st = launched(cudaGetLastError())) != FP2_OK) return st;

    ScoreArgs sa;
    sa.cu_q = cu_q;
    sa.cu_k = cu_k;
    sa.cu_blocks = at<int32_t>(ws, pr.ws.cu_blocks);
    sa.cu_qblocks = at<int32_t>(ws, pr.ws.cu_qblocks);
    sa.cu_tiles = at<int32_t>(ws, pr.ws.cu_tiles);
    sa.batch = pr.batch;
    sa.hq = p->num_q_heads;
    sa.hkv = p->num_kv_heads;
    sa.G = G;
    sa.qt = qt;
    sa.max_blocks = pr.max_blocks;
    sa.nb_max = meta->nb_max;
    sa.tau = tau_of(p);
    sa.keep_all = p->alpha <= 0.f ? 1 : 0;
    sa.ln_alpha = p->alpha > 0.f ? std::log(p->alpha) : 0.f;
    sa.kept_cnt = meta->kept_cnt;
    sa.kept_idx = meta->kept_idx;
    sa.score_dbg = meta->score_dbg;
    sa.hdr = hdr;
    uint16_t* qs = at<uint16_t>(ws, pr.ws.qsplit);
    uint16_t* ks = at<uint16_t>(ws, pr.ws.ksplit);
    const int64_t qrows = pr.max_blocks * p->num_q_heads;
    const int64_t krows = pr.max_blocks * p->num_kv_heads;
    CUtensorMap tqh, tql, tkh, tkl;
    if (!make_map_2d(&tqh, qs, qrows) || !make_map_2d(&tql, qs + qrows * kHeadDim, qrows) ||
        !make_map_2d(&tkh, ks, krows) || !make_map_2d(&tkl, ks + krows * kHeadDim, krows))
        return FP2_ERR_CUDA;
    const size_t smem = score_smem_bytes();
    if (cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return FP2_ERR_CUDA;
    const int64_t tiles = (pr.max_qblocks + qt - 1) / qt + pr.batch;  // <= 65535 (check_limits)
    score_kernel<<<dim3(static_cast<unsigned>(p->num_kv_heads), static_cast<unsigned>(tiles)),
                   kScoreThreads, smem, s>>>(sa, tqh, tql, tkh, tkl);
    return launched(cudaGetLastError());
}

fp2_status run_attention(const fp2_params* p, const void* q, const void* k, const void* v,
                         const int32_t* cu_q, const int32_t* cu_k, const Problem& pr,
                         const int32_t* block_table,
                         int32_t mbps, int32_t num_pages, const fp2_blockmeta* meta, void* out,
                         float* lse, void* ws, cudaStream_t s) {
    const bool e4m3 = p->dtype == FP2_E4M3;
    fp2_status st = check_limits(p, pr, false, true);
    if (st != FP2_OK) return st;
    st = run_setup(pr, ws, cu_q, cu_k, 1, block_table != nullptr, mbps, meta->max_blocks, s,
                   meta->kept_cnt, p->num_kv_heads, p->correction);
    if (st != FP2_OK) return st;
    if (pr.batch == 0 || pr.total_q == 0) return FP2_OK;  // no rows to attend
    WsHeader* hdr = at<WsHeader>(ws, 0);
    void* kb_lp = at<void>(ws, pr.ws.kbar_lp);
    void* vb_lp = at<void>(ws, pr.ws.vbar_lp);
    if (p->correction) {
        MeanLpArgs ma;
        ma.k_mean = meta->k_mean;
        ma.v_mean = meta->v_mean;
        ma.k_lp = kb_lp;
        ma.v_lp = vb_lp;
        ma.k_scale = p->k_scale;
        ma.v_scale = p->v_scale;
        ma.hkv = p->num_kv_heads;
        ma.e4m3 = e4m3 ? 1 : 0;
        ma.max_blocks = pr.max_blocks;
        ma.hdr = hdr;
        meanlp_kernel<<<592, 256, 0, s>>>(ma);
        if ((st = launched(cudaGetLastError())) != FP2_OK) return st;
    }
    const int64_t kv_rows = block_table ? int64_t(num_pages) * kBlock : pr.total_k;
    CUtensorMap tq, tk, tv, tkb, tvb;
    if (!make_map(&tq, q, e4m3, p->num_q_heads, pr.total_q) ||
        !make_map(&tk, k, e4m3, p->num_kv_heads, kv_rows) ||
        !make_map(&tv, v, e4m3, p->num_kv_heads, kv_rows) ||
        !make_map(&tkb, kb_lp, e4m3, p->num_kv_heads, pr.max_blocks) ||
        !make_map(&tvb, vb_lp, e4m3, p->num_kv_heads, pr.max_blocks))
        return FP2_ERR_CUDA;
    AttnArgs a;
    a.cu_q = cu_q;
    a.cu_k = cu_k;
    a.cu_blocks = at<int32_t>(ws, pr.ws.cu_blocks);
    a.cu_qblocks = at<int32_t>(ws, pr.ws.cu_qblocks);
    a.blk_req_q = at<int32_t>(ws, pr.ws.blk_req_q);
    a.order = at<int32_t>(ws, pr.ws.order);
    a.block_table = block_table;
    a.max_blocks_per_seq = mbps;
    a.num_pages = num_pages;
    a.kept_cnt = meta->kept_cnt;
    a.kept_idx = meta->kept_idx;
    a.nb_max = meta->nb_max;
    a.nb_cap = pr.nb_need > 0 ? pr.nb_need : 1;
    a.hq = p->num_q_heads;
    a.hkv = p->num_kv_heads;
    a.G = p->num_q_heads / p->num_kv_heads;
    a.pairs = (a.G + 1) / 2;
    a.correction = p->correction;
    a.k_var = meta->k_var;
    a.var_coef = 0.5f * tau_of(p) * tau_of(p) * 1.4426950408889634f;
    // test hook (tests/test_gpu_errors.py): make one bounded wait run out
    a.test_wait_timeout = std::getenv("FP2_TEST_WAIT_TIMEOUT") != nullptr ? 1 : 0;
    a.scale_log2 = tau_of(p) * 1.4426950408889634f;
    a.q_scale = p->q_scale;
    a.k_scale = p->k_scale;
    a.v_scale = p->v_scale;
    a.out = out;
    a.out_align32 = aligned(out, 32) ? 1 : 0;
    a.lse = lse;
    a.hdr = hdr;
    return launched(launch_attention(e4m3, a, tq, tk, tv, tkb, tvb, pr.max_qblocks, s));
}

}  // namespace

extern "C" {

int64_t fp2_max_blocks(int32_t batch, int64_t total_tokens, int32_t block_size) {
    if (batch < 0 || total_tokens < 0 || block_size <= 0) return 0;
    return total_tokens / block_size + batch;
}

size_t fp2_workspace_bytes(const fp2_params* params, int32_t batch, int64_t total_tokens,
                           int32_t max_seqlen) {
    if (check_params(params) != FP2_OK || batch < 0 || total_tokens < 0 || max_seqlen < 0) return 0;
    return ws_layout(batch, fp2_max_blocks(batch, total_tokens, kBlock), params->num_q_heads,
                     params->num_kv_heads, esize(params))
        .total;
}

fp2_status fp2_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
    if (!workspace || !aligned(workspace, 256) || ws_bytes < sizeof(WsHeader)) return FP2_ERR_WORKSPACE;
    return launched(cudaMemsetAsync(workspace, 0, sizeof(WsHeader), static_cast<cudaStream_t>(stream)));
}

fp2_status fp2_estimate_chunked(const fp2_params* params, const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch,
                                int64_t total_q, int64_t total_k, int32_t max_seqlen_k,
                                const int32_t* block_table, int32_t max_blocks_per_seq, int32_t num_pages,
                                fp2_blockmeta* meta, void* workspace, size_t ws_bytes, void* stream) {
    Problem pr;
    fp2_status st = check_problem(params, q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                  max_seqlen_k, workspace, ws_bytes, &pr);
    if (st != FP2_OK) return st;
    if ((st = check_meta(meta, params, pr, false)) != FP2_OK) return st;
    if (block_table && (max_blocks_per_seq < 1 || num_pages < 1)) return FP2_ERR_INVALID_ARG;
    // page rows are int32 inside the kernels (TMA coordinates)
    if (block_table && int64_t(num_pages) * kBlock > (int64_t(1) << 31) - 1) return FP2_ERR_UNSUPPORTED;
    return run_estimate(params, q, k, v, cu_seqlens_q, cu_seqlens_k, pr, block_table, max_blocks_per_seq,
                        num_pages, meta, workspace, static_cast<cudaStream_t>(stream));
}

fp2_status fp2_estimate(const fp2_params* params, const void* q, const void* k, const void* v,
                        const int32_t* cu_seqlens, int32_t batch, int64_t total_tokens,
                        int32_t max_seqlen, const int32_t* block_table, int32_t max_blocks_per_seq,
                        int32_t num_pages, fp2_blockmeta* meta, void* workspace, size_t ws_bytes,
                        void* stream) {
    return fp2_estimate_chunked(params, q, k, v, cu_seqlens, cu_seqlens, batch, total_tokens, total_tokens,
                                max_seqlen, block_table, max_blocks_per_seq, num_pages, meta, workspace,
                                ws_bytes, stream);
}

fp2_status fp2_prefill_chunked(const fp2_params* params, const void* q, const void* k, const void* v,
                               const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t batch,
                               int64_t total_q, int64_t total_k, int32_t max_seqlen_k,
                               const int32_t* block_table, int32_t max_blocks_per_seq, int32_t num_pages,
                               const fp2_blockmeta* meta, void* out, float* lse, void* workspace,
                               size_t ws_bytes, void* stream) {
    Problem pr;
    fp2_status st = check_problem(params, q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                  max_seqlen_k, workspace, ws_bytes, &pr);
    if (st != FP2_OK) return st;
    if ((st = check_meta(meta, params, pr, true)) != FP2_OK) return st;
    if (block_table && (max_blocks_per_seq < 1 || num_pages < 1)) return FP2_ERR_INVALID_ARG;
    // page rows are int32 inside the kernels (TMA coordinates)
    if (block_table && int64_t(num_pages) * kBlock > (int64_t(1) << 31) - 1) return FP2_ERR_UNSUPPORTED;
    if (total_q > 0 && (!out || !aligned(out, 16))) return FP2_ERR_INVALID_ARG;
    if (lse && !aligned(lse, 4)) return FP2_ERR_INVALID_ARG;
    return run_attention(params, q, k, v, cu_seqlens_q, cu_seqlens_k, pr, block_table, max_blocks_per_seq,
                         num_pages, meta, out, lse, workspace, static_cast<cudaStream_t>(stream));
}

fp2_status fp2_sparse_prefill(const fp2_params* params, const void* q, const void* k, const void* v,
                              const int32_t* cu_seqlens, int32_t batch, int64_t total_tokens,
                              int32_t max_seqlen, const fp2_blockmeta* meta, void* out, float* lse,
                              void* workspace, size_t ws_bytes, void* stream) {
    return fp2_prefill_chunked(params, q, k, v, cu_seqlens, cu_seqlens, batch, total_tokens, total_tokens,
                               max_seqlen, nullptr, 0, 0, meta, out, lse, workspace, ws_bytes, stream);
}

fp2_status fp2_prefill_paged(const fp2_params* params, const void* q, const void* k_pool,
                             const void* v_pool, const int32_t* cu_seqlens, int32_t batch,
                             int64_t total_tokens, int32_t max_seqlen, const int32_t* block_table,
                             int32_t max_blocks_per_seq, int32_t num_pages, const fp2_blockmeta* meta,
                             void* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
    if (batch > 0 && !block_table) return FP2_ERR_INVALID_ARG;
    if (batch > 0 && (max_blocks_per_seq < 1 || num_pages < 1)) return FP2_ERR_INVALID_ARG;
    return fp2_prefill_chunked(params, q, k_pool, v_pool, cu_seqlens, cu_seqlens, batch, total_tokens,
                               total_tokens, max_seqlen, block_table, max_blocks_per_seq, num_pages, meta,
                               out, lse, workspace, ws_bytes, stream);
}

fp2_status fp2_get_error(void* workspace, void* stream) {
    if (!workspace || !aligned(workspace, 256)) return FP2_ERR_WORKSPACE;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h[2] = {0, 0};
    if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return FP2_ERR_CUDA;
    if (h[0] != 0) {
        if (cudaMemsetAsync(workspace, 0, 2 * sizeof(int32_t), s) != cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return FP2_ERR_CUDA;
    }
    return static_cast<fp2_status>(h[0]);
}

const char* fp2_status_string(fp2_status status) {
    switch (status) {
        case FP2_OK: return "ok";
        case FP2_ERR_INVALID_ARG: return "invalid argument";
        case FP2_ERR_UNSUPPORTED: return "unsupported configuration";
        case FP2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case FP2_ERR_CUDA: return "CUDA call or kernel launch failed";
        case FP2_ERR_TIMEOUT: return "device pipeline wait timed out";
        case FP2_ERR_BAD_INDEX: return "bad cu_seqlens or page index";
    }
    return "unknown status";
}

int32_t fp2_version(void) { return 200; }

}  // extern "C"

// ---------------------------------------------------------------------------
// fp2_sparse_prefill_noalloc: the same attention call with its scratch in a
// file-scope device array instead of a caller workspace.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[FP2_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};  // device address of the array, per device ordinal

// Device address of the scratch array on the current device.  Host code must
// not hand `g_noalloc_scratch` itself to a kernel: on the host that name is a
// stand-in, not a device address.
fp2_status noalloc_scratch(void** addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FP2_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *addr = g_noalloc_addr[dev];
    return FP2_OK;
}

}  // namespace

extern "C" fp2_status fp2_sparse_prefill_noalloc(const fp2_params* params, const void* q,
                                                 const void* k, const void* v,
                                                 const int32_t* cu_seqlens, int32_t batch,
                                                 int64_t total_tokens, int32_t max_seqlen,
                                                 const fp2_blockmeta* meta, void* out, float* lse,
                                                 int32_t* device_status, void* stream) {
    fp2_status st = check_params(params);
    if (st != FP2_OK) return st;
    if (batch < 0 || total_tokens < 0 || max_seqlen < 0) return FP2_ERR_INVALID_ARG;
    if (total_tokens > (int64_t(1) << 31) - 1) return FP2_ERR_UNSUPPORTED;
    if (batch > 0 && !cu_seqlens) return FP2_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!q || !k || !v)) return FP2_ERR_INVALID_ARG;
    if ((q && !aligned(q, 16)) || (k && !aligned(k, 16)) || (v && !aligned(v, 16)))
        return FP2_ERR_INVALID_ARG;
    if (total_tokens > 0 && (!out || !aligned(out, 16))) return FP2_ERR_INVALID_ARG;
    if (lse && !aligned(lse, 4)) return FP2_ERR_INVALID_ARG;
    if (device_status && !aligned(device_status, 4)) return FP2_ERR_INVALID_ARG;
    Problem pr;
    pr.batch = batch;
    pr.total_q = total_tokens;
    pr.total_k = total_tokens;
    pr.max_seqlen = max_seqlen;
    pr.max_blocks = fp2_max_blocks(batch, total_tokens, kBlock);
    pr.max_qblocks = pr.max_blocks;
    pr.nb_need = (max_seqlen + kBlock - 1) / kBlock;
    // the attention call reads none of the estimator's split means
    pr.ws = ws_layout(batch, pr.max_blocks, params->num_q_heads, params->num_kv_heads, esize(params),
                      false);
    if (pr.ws.total > FP2_NOALLOC_SCRATCH_BYTES) return FP2_ERR_WORKSPACE;  // over the static maximum
    if ((st = check_meta(meta, params, pr, true)) != FP2_OK) return st;
    // every host-side rejection before anything is enqueued
    if ((st = check_limits(params, pr, false, true)) != FP2_OK) return st;
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != FP2_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the error flag is the only scratch state that must start at zero; every
    // other region is rewritten by the kernels of this call
    if (cudaMemsetAsync(scratch, 0, sizeof(WsHeader), s) != cudaSuccess) return FP2_ERR_CUDA;
    st = run_attention(params, q, k, v, cu_seqlens, cu_seqlens, pr, nullptr, 0, 0, meta, out, lse, scratch,
                       s);
    if (st != FP2_OK) return st;
    if (device_status &&
        cudaMemcpyAsync(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
        return FP2_ERR_CUDA;
    return FP2_OK;
}

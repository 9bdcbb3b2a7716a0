// kernels.h -- argument blocks and declarations of the device kernels.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "common.cuh"

namespace fp2 {

constexpr int kPoolThreads = 544;  // 16 consumer warps (4 row groups x 128 column lanes) + TMA warp
constexpr int kScoreThreads = 160; // score_kernel: 4 epilogue warps + 1 TMA/MMA warp

struct SetupArgs {
    const int32_t* cu_q;     // [batch + 1] query rows
    const int32_t* cu_k;     // [batch + 1] keys (= cu_q for plain prefill)
    int32_t batch;
    int64_t total_q;
    int64_t total_k;
    int32_t max_seqlen;      // >= every request's keys
    int32_t qt;  // q-blocks per estimator tile
    int32_t paged;
    int32_t max_blocks_per_seq;
    int64_t max_blocks;
    int32_t nb_cap;  // >= blocks of the longest request (histogram bins)
    // attention call: order the (q-block, KV head) work items by their cost
    // (kept tiles + correction tiles), heaviest first; NULL (the estimator
    // call): no work order
    const int32_t* kept_cnt;   // [max_blocks, hkv]
    int32_t hkv;
    int32_t correction;
    WsHeader* hdr;
    int32_t* cu_blocks;   // key blocks
    int32_t* cu_qblocks;  // q-blocks
    int32_t* cu_tiles;    // estimator tiles of q-blocks
    int32_t* blk_req;     // request of every key block
    int32_t* blk_req_q;   // request of every q-block
    int32_t* order;  // codes t * hkv + g (t a q-block), heaviest first (attention call)
};

// Histogram bins of the setup kernel's cost order (kept tiles <= nb_cap,
// correction tiles <= ceil(nb_cap / 128), fill 2); the estimator call has none.
__host__ __device__ inline int32_t setup_bins(int32_t nb_cap, bool cost) {
    return cost ? nb_cap + (nb_cap + 127) / 128 + 3 : 0;
}

struct PoolArgs {
    float* out[3];           // fp32 means (NULL = not written): -, k_mean, v_mean
    float* kvar;             // NULL, or [max_blocks, Hkv]: key variance of every block, averaged
                             // over the dimensions (dequantised)
    uint16_t* split[2];      // bf16 hi/lo means of q (grouped rows) and k, see WsLayout
    const float* scale[3];   // per-head dequantisation scales (NULL = 1)
    int32_t heads[3];
    int32_t hb[3];           // heads per column slab (one TMA box: 32 rows x hb heads x d)
    int32_t slabs[3];        // column slabs per block of each tensor
    int32_t paged[3];
    int32_t first, last;     // tensors [first, last) of q, k, v are pooled
    const int32_t* cu_q;
    const int32_t* cu_k;
    const int32_t* cu_blocks;
    const int32_t* cu_qblocks;
    const int32_t* blk_req;
    const int32_t* blk_req_q;
    const int32_t* block_table;
    int32_t max_blocks_per_seq;
    int32_t num_pages;
    int32_t G;                 // query heads per KV head
    int64_t max_blocks;        // row capacity of the split arrays
    WsHeader* hdr;
};

struct ScoreArgs {
    const int32_t* cu_q;
    const int32_t* cu_k;
    const int32_t* cu_blocks;
    const int32_t* cu_qblocks;
    const int32_t* cu_tiles;
    int32_t batch;
    int32_t hq, hkv, G;
    int32_t qt;          // q-blocks per tile: floor(128 / G)
    int64_t max_blocks;  // row capacity of the split mean arrays
    int32_t nb_max;
    float tau, ln_alpha;
    int32_t keep_all;
    int32_t* kept_cnt;
    int32_t* kept_idx;
    float* score_dbg;
    WsHeader* hdr;
};

struct MeanLpArgs {
    const float* k_mean;
    const float* v_mean;
    void* k_lp;
    void* v_lp;
    const float* k_scale;
    const float* v_scale;
    int32_t hkv;
    int32_t e4m3;
    int64_t max_blocks;   // rows of k_lp / v_lp; rows past the last block are zeroed
    WsHeader* hdr;
};

struct AttnArgs {
    const int32_t* cu_q;
    const int32_t* cu_k;
    const int32_t* cu_blocks;    // key blocks (rows of the correction operands)
    const int32_t* cu_qblocks;
    const int32_t* blk_req_q;
    const int32_t* order;        // work items t * hkv + g (q-block, KV head), heaviest first
    const int32_t* block_table;  // NULL = contiguous K/V
    int32_t max_blocks_per_seq;
    int32_t num_pages;
    const int32_t* kept_cnt;
    const int32_t* kept_idx;
    int32_t nb_max;              // row stride of kept_idx
    int32_t nb_cap;              // >= key blocks of the longest request (shared-memory lists)
    int32_t hq, hkv, G, pairs;   // pairs = ceil(G / 2) CTAs per (q-block, KV head)
    int32_t correction;          // 0 none, 1 mean, 2 mean with the variance term
    const float* k_var;          // correction 2: [max_blocks, Hkv] mean key variance per block
    float var_coef;              // correction 2: tau^2 / 2 * log2(e)
    int32_t test_wait_timeout;   // 1: the MMA issuer waits on a barrier nothing completes
                                 // (tests the bounded-wait timeout and abort path)
    float scale_log2;            // tau * log2(e)
    const float* q_scale;        // e4m3 only
    const float* k_scale;
    const float* v_scale;
    void* out;                   // bf16 [T, Hq, d]
    int32_t out_align32;         // 1: out is 32-byte aligned (each output row is then
                                 // written with 256-bit stores, else 128-bit ones)
    float* lse;                  // [T, Hq] or NULL
    WsHeader* hdr;
};

__global__ void setup_kernel(SetupArgs a);
template <bool kE4M3>
__global__ void pool_kernel(const __grid_constant__ PoolArgs a, const __grid_constant__ CUtensorMap tq,
                            const __grid_constant__ CUtensorMap tk,
                            const __grid_constant__ CUtensorMap tv);
size_t pool_smem_bytes(bool e4m3);
__global__ void score_kernel(const __grid_constant__ ScoreArgs a,
                             const __grid_constant__ CUtensorMap tqh,
                             const __grid_constant__ CUtensorMap tql,
                             const __grid_constant__ CUtensorMap tkh,
                             const __grid_constant__ CUtensorMap tkl);
size_t score_smem_bytes();
__global__ void meanlp_kernel(MeanLpArgs a);

// Shared-memory bytes of the attention kernel for a kept-list capacity (var:
// correction 2, which stages one variance per pruned block).
size_t attn_smem_bytes(bool e4m3, int32_t nb_cap, bool var);
// Launches the persistent attention kernel: one CTA per SM, taking work items
// (q-block, KV head, query-head pair) from a counter in the workspace.
cudaError_t launch_attention(bool e4m3, const AttnArgs& a, const CUtensorMap& tq,
                             const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& tkb, const CUtensorMap& tvb, int64_t max_blocks,
                             cudaStream_t stream);

}  // namespace fp2

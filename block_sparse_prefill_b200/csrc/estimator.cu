// estimator.cu -- the block-score estimator of block-sparse prefill
// ("computes a small sample of attention scores, finds the maximum, and attends
// only to tokens that exceed a threshold relative to that max", lode.cx write-up
// of FlashPrefill V2, section "How It Works"; "estimating scores at the block
// level", aipulsen.com write-up), plus the small set-up and conversion passes
// the attention call needs.
//
//   setup_kernel   validates cu_seqlens, numbers the blocks of the ragged batch
//   pool_kernel    block means of Q, K, V (HBM-bound streaming pass, every input
//                  byte read once with 16-byte loads)
//   score_kernel   s = tau * qbar . kbar for the causal block pairs of a tile of
//                  q-blocks (fp32 FMA from shared memory), per-head row max,
//                  exp(s - m) >= alpha threshold, union over the G query heads of
//                  a KV head, forced diagonal, ascending compaction
//   meanlp_kernel  block means -> bf16 / e4m3 operands of the correction MMA
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace fp2 {

// ---------------------------------------------------------------------------
// set-up
// ---------------------------------------------------------------------------
__global__ void setup_kernel(SetupArgs a) {
    extern __shared__ int32_t hist[];  // [nb_cap + 1]
    __shared__ int32_t ok;
    if (threadIdx.x == 0) {
        int32_t good = 1, bad = -1;
        int32_t nb_acc = 0, nt_acc = 0;
        if (a.cu[0] != 0) { good = 0; bad = 0; }
        a.cu_blocks[0] = 0;
        a.cu_tiles[0] = 0;
        for (int32_t b = 0; good && b < a.batch; ++b) {
            const int32_t L = a.cu[b + 1] - a.cu[b];
            if (L < 0 || L > a.max_seqlen) { good = 0; bad = b + 1; break; }
            const int32_t nb = (L + kBlock - 1) / kBlock;
            if (a.paged && nb > a.max_blocks_per_seq) { good = 0; bad = b + 1; break; }
            nb_acc += nb;
            nt_acc += (nb + a.qt - 1) / a.qt;
            a.cu_blocks[b + 1] = nb_acc;
            a.cu_tiles[b + 1] = nt_acc;
        }
        if (good && a.cu[a.batch] != a.total_tokens) { good = 0; bad = a.batch; }
        if (good && nb_acc > a.max_blocks) { good = 0; bad = a.batch; }
        a.hdr->valid = good;
        a.hdr->total_blocks = good ? nb_acc : 0;
        a.hdr->work_next = 0;
        if (!good) set_error(a.hdr, FP2_ERR_BAD_INDEX, bad);
        ok = good;
    }
    for (int32_t e = threadIdx.x; e <= a.nb_cap; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    if (!ok) return;
    for (int32_t b = 0; b < a.batch; ++b)
        for (int32_t t = a.cu_blocks[b] + threadIdx.x; t < a.cu_blocks[b + 1]; t += blockDim.x) {
            a.blk_req[t] = b;
            atomicAdd(&hist[t - a.cu_blocks[b]], 1);
        }
    __syncthreads();
    // order: blocks sorted by their index in the request, largest first (the
    // causal kept lists grow with it), so the persistent attention kernel
    // takes the longest work items first
    if (threadIdx.x == 0) {
        int32_t run = 0;
        for (int32_t j = a.nb_cap - 1; j >= 0; --j) {
            const int32_t c = hist[j];
            hist[j] = run;
            run += c;
        }
    }
    __syncthreads();
    for (int32_t b = 0; b < a.batch; ++b)
        for (int32_t t = a.cu_blocks[b] + threadIdx.x; t < a.cu_blocks[b + 1]; t += blockDim.x)
            a.order[atomicAdd(&hist[t - a.cu_blocks[b]], 1)] = t;
}

// ---------------------------------------------------------------------------
// pooling: mean over the valid rows of every block, per column
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <bool kE4M3>
struct PoolVec;
template <>
struct PoolVec<false> {  // 8 bf16 per 16 bytes
    static constexpr int N = 8;
    __device__ static void add(float* acc, uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(w[i] << 16);
            acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct PoolVec<true> {  // 16 e4m3 per 16 bytes
    static constexpr int N = 16;
    __device__ static void add(float* acc, uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFF), __NV_E4M3);
            __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
            float2 a = __half22float2(*reinterpret_cast<__half2*>(&lo));
            float2 b = __half22float2(*reinterpret_cast<__half2*>(&hi));
            acc[4 * i] += a.x;
            acc[4 * i + 1] += a.y;
            acc[4 * i + 2] += b.x;
            acc[4 * i + 3] += b.y;
        }
    }
};

template <bool kE4M3>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(PoolArgs a) {
    using V = PoolVec<kE4M3>;
    constexpr int N = V::N;
    constexpr int kRowGroups = kPoolThreads / 128;
    __shared__ float red[kRowGroups - 1][128][N + 1];

    const int32_t t = blockIdx.x;
    if (!a.hdr->valid || t >= a.hdr->total_blocks) return;
    // which tensor / column slab
    int32_t y = blockIdx.y, x = 0;
    while (x < 2 && y >= a.slabs[x]) { y -= a.slabs[x]; ++x; }
    if (x >= a.ntensors) return;
    const int32_t b = a.blk_req[t];
    const int32_t j = t - a.cu_blocks[b];
    const int32_t L = a.cu[b + 1] - a.cu[b];
    const int32_t n = min(kBlock, L - j * kBlock);
    const int32_t ncols = a.heads[x] * kHeadDim;
    const int32_t tc = threadIdx.x & 127;
    const int32_t rg = threadIdx.x >> 7;
    const int32_t col = (y * 128 + tc) * N;
    const bool active = col < ncols;

    int64_t row0;
    if (a.paged[x]) {
        int32_t page = a.block_table[static_cast<int64_t>(b) * a.max_blocks_per_seq + j];
        if (page < 0 || page >= a.num_pages) {
            if (threadIdx.x == 0) set_error(a.hdr, FP2_ERR_BAD_INDEX, t);
            page = 0;
        }
        row0 = static_cast<int64_t>(page) * kBlock;
    } else {
        row0 = a.cu[b] + static_cast<int64_t>(j) * kBlock;
    }

    float acc[N];
#pragma unroll
    for (int e = 0; e < N; ++e) acc[e] = 0.f;
    if (active) {
        const char* base = static_cast<const char*>(a.x[x]) +
                           (row0 * ncols + col) * static_cast<int64_t>(kE4M3 ? 1 : 2);
        const int64_t rstride = static_cast<int64_t>(ncols) * (kE4M3 ? 1 : 2);
        int32_t r = rg;
        for (; r + 7 * kRowGroups < n; r += 8 * kRowGroups) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = ld_stream16(base + (r + u * kRowGroups) * rstride);
#pragma unroll
            for (int u = 0; u < 8; ++u) V::add(acc, v[u]);
        }
        for (; r < n; r += kRowGroups) V::add(acc, ld_stream16(base + r * rstride));
    }
    if (rg > 0) {
#pragma unroll
        for (int e = 0; e < N; ++e) red[rg - 1][tc][e] = acc[e];
    }
    __syncthreads();
    if (rg == 0 && active) {
#pragma unroll
        for (int g = 0; g < kRowGroups - 1; ++g)
#pragma unroll
            for (int e = 0; e < N; ++e) acc[e] += red[g][tc][e];
        const int32_t h = col / kHeadDim;
        const float s = (a.scale[x] ? a.scale[x][h] : 1.f) / static_cast<float>(n);
        float* out = a.out[x] + static_cast<int64_t>(t) * ncols + col;
#pragma unroll
        for (int e = 0; e < N; e += 4)
            *reinterpret_cast<float4*>(out + e) =
                make_float4(acc[e] * s, acc[e + 1] * s, acc[e + 2] * s, acc[e + 3] * s);
    }
}

// ---------------------------------------------------------------------------
// scores, threshold, union, compaction
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) score_kernel(ScoreArgs a) {
    extern __shared__ __align__(16) float smem[];
    const int32_t RP = a.rp;                  // padded rows (multiple of 4)
    float* qs = smem;                         // [d][RP]
    float* ks = qs + kHeadDim * RP;           // [d][KC + 4]
    float* sc = ks + kHeadDim * (kScoreKC + 4);  // [RP][ncap]
    float* rowmax = sc + static_cast<size_t>(RP) * a.ncap;  // [RP]

    if (!a.hdr->valid) return;
    const int32_t total_tiles = a.cu_tiles[a.batch];
    if (static_cast<int32_t>(blockIdx.x) >= total_tiles) return;
    const int32_t tile = total_tiles - 1 - blockIdx.x;  // late (long-row) tiles first
    int32_t lo = 0, hi = a.batch - 1;                   // request owning this tile
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (a.cu_tiles[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int32_t b = lo;
    const int32_t g = blockIdx.y;
    const int32_t G = a.G;
    const int32_t cb = a.cu_blocks[b];
    const int32_t nb = a.cu_blocks[b + 1] - cb;
    const int32_t i0 = (tile - a.cu_tiles[b]) * a.qt;
    const int32_t nqb = min(a.qt, nb - i0);
    const int32_t nrows = nqb * G;
    const int32_t ncols = i0 + nqb;
    const int32_t tid = threadIdx.x;
    const int32_t nthr = blockDim.x;

    // q rows, transposed: qs[c][rho], rho = ii * G + hh
    for (int32_t e = tid; e < RP * kHeadDim; e += nthr) {
        const int32_t rho = e / kHeadDim, c = e % kHeadDim;
        float v = 0.f;
        if (rho < nrows) {
            const int32_t ii = rho / G, hh = rho % G;
            v = a.qbar[(static_cast<int64_t>(cb + i0 + ii) * a.hq + g * G + hh) * kHeadDim + c];
        }
        qs[c * RP + rho] = v;
    }
    const int32_t tr = tid / 32;  // 4-row group
    const int32_t tcg = tid % 32;  // 2-column group
    for (int32_t kc0 = 0; kc0 < ncols; kc0 += kScoreKC) {
        __syncthreads();
        for (int32_t e = tid; e < kScoreKC * kHeadDim; e += nthr) {
            const int32_t jj = e / kHeadDim, c = e % kHeadDim;
            const int32_t j = kc0 + jj;
            ks[c * (kScoreKC + 4) + jj] =
                j < ncols ? a.kbar[(static_cast<int64_t>(cb + j) * a.hkv + g) * kHeadDim + c] : 0.f;
        }
        __syncthreads();
        float acc[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 8
        for (int32_t c = 0; c < kHeadDim; ++c) {
            const float4 q4 = *reinterpret_cast<const float4*>(qs + c * RP + 4 * tr);
            const float2 k2 = *reinterpret_cast<const float2*>(ks + c * (kScoreKC + 4) + 2 * tcg);
            acc[0][0] = fmaf(q4.x, k2.x, acc[0][0]);
            acc[0][1] = fmaf(q4.x, k2.y, acc[0][1]);
            acc[1][0] = fmaf(q4.y, k2.x, acc[1][0]);
            acc[1][1] = fmaf(q4.y, k2.y, acc[1][1]);
            acc[2][0] = fmaf(q4.z, k2.x, acc[2][0]);
            acc[2][1] = fmaf(q4.z, k2.y, acc[2][1]);
            acc[3][0] = fmaf(q4.w, k2.x, acc[3][0]);
            acc[3][1] = fmaf(q4.w, k2.y, acc[3][1]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int32_t j = kc0 + 2 * tcg + cc;
                if (j < a.ncap) sc[(4 * tr + r) * a.ncap + j] = a.tau * acc[r][cc];
            }
    }
    __syncthreads();

    const int32_t warp = tid / 32, lane = tid % 32, nwarps = nthr / 32;
    for (int32_t rho = warp; rho < nrows; rho += nwarps) {
        const int32_t i = i0 + rho / G;
        float m = -INFINITY;
        for (int32_t j = lane; j <= i; j += 32) m = fmaxf(m, sc[rho * a.ncap + j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) rowmax[rho] = m;
        if (a.score_dbg) {
            const int32_t h = g * G + rho % G;
            float* dst = a.score_dbg + (static_cast<int64_t>(cb + i) * a.hq + h) * a.nb_max;
            for (int32_t j = lane; j <= i; j += 32) dst[j] = sc[rho * a.ncap + j] - m;
        }
    }
    __syncthreads();
    for (int32_t ii = warp; ii < nqb; ii += nwarps) {
        const int32_t i = i0 + ii;
        const int64_t row = static_cast<int64_t>(cb + i) * a.hkv + g;
        int32_t* dst = a.kept_idx + row * a.nb_max;
        int32_t base = 0;
        for (int32_t j0 = 0; j0 <= i; j0 += 32) {
            const int32_t j = j0 + lane;
            bool keep = false;
            if (j <= i) {
                if (a.keep_all || j == i) {
                    keep = true;
                } else {
                    for (int32_t hh = 0; hh < G; ++hh) {
                        const int32_t rho = ii * G + hh;
                        keep |= (sc[rho * a.ncap + j] - rowmax[rho]) >= a.ln_alpha;
                    }
                }
            }
            const uint32_t mask = __ballot_sync(0xffffffffu, keep);
            if (keep) dst[base + __popc(mask & ((1u << lane) - 1u))] = j;
            base += __popc(mask);
        }
        if (lane == 0) a.kept_cnt[row] = base;
    }
}

// ---------------------------------------------------------------------------
// block means -> MMA operand precision
// ---------------------------------------------------------------------------
__global__ void meanlp_kernel(MeanLpArgs a) {
    if (!a.hdr->valid) return;
    const int64_t per = static_cast<int64_t>(a.hkv) * kHeadDim;
    const int64_t n4 = static_cast<int64_t>(a.hdr->total_blocks) * per / 4;
    const int64_t all4 = a.max_blocks * per / 4;
    // rows past the last block are zero: the correction MMA reads whole
    // 128-row tiles and multiplies masked (zero-weight) rows by them
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < all4;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int32_t g = static_cast<int32_t>((e * 4 / kHeadDim) % a.hkv);
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const float* src = which ? a.v_mean : a.k_mean;
            if (!src) continue;
            const float4 x = e < n4 ? reinterpret_cast<const float4*>(src)[e] : make_float4(0.f, 0.f, 0.f, 0.f);
            if (a.e4m3) {
                const float inv = 1.f / (which ? a.v_scale[g] : a.k_scale[g]);
                reinterpret_cast<uint32_t*>(which ? a.v_lp : a.k_lp)[e] =
                    pack_e4m3x4(x.x * inv, x.y * inv, x.z * inv, x.w * inv);
            } else {
                reinterpret_cast<uint2*>(which ? a.v_lp : a.k_lp)[e] =
                    make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
            }
        }
    }
}

template __global__ void pool_kernel<false>(PoolArgs);
template __global__ void pool_kernel<true>(PoolArgs);

}  // namespace fp2

// estimator.cu -- the block-score estimator of block-sparse prefill: a cheap
// estimate of the attention scores, their maximum, and the blocks whose score
// clears a threshold set relative to that maximum (lode.cx write-up of
// FlashPrefill V2, section "How It Works"; the aipulsen.com write-up makes the
// estimate per block), plus the small set-up and conversion passes the
// attention call needs.
//
//   setup_kernel   validates cu_seqlens, numbers the blocks of the ragged batch
//   pool_kernel    block means of Q, K, V (HBM-bound streaming pass, every input
//                  byte read once, TMA into a ring of shared-memory stages)
//   score_kernel   s = tau * qbar . kbar for the causal block pairs of a tile of
//                  q-blocks (tcgen05 MMAs on bf16 hi/lo parts of the means, fp32
//                  accumulation in TMEM), per-head row max, exp(s - m) >= alpha
//                  threshold, union over the G query heads of a KV head, forced
//                  diagonal, ascending compaction
//   meanlp_kernel  block means -> bf16 / e4m3 operands of the correction MMA
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace fp2 {

// ---------------------------------------------------------------------------
// set-up
// ---------------------------------------------------------------------------
// Cost of the attention work item (q-block t = block i of its request, KV
// head g) in tile steps: its kept tiles, its correction tiles (128 pruned-block
// means each, when the correction is on) and 2 steps of pipeline fill.  The kept
// count is clamped to [1, i + 1]; the attention kernel checks the list itself.
__device__ __forceinline__ int32_t item_cost(const SetupArgs& a, int32_t t, int32_t i, int32_t g) {
    const int32_t c = min(max(a.kept_cnt[static_cast<int64_t>(t) * a.hkv + g], 1), i + 1);
    const int32_t pruned = i + 1 - c;
    const int32_t corr = (a.correction && pruned > 0) ? min((i + 127) / 128, pruned) : 0;
    return c + corr + 2;
}

__global__ void setup_kernel(SetupArgs a) {
    extern __shared__ int32_t hist[];  // [setup_bins(nb_cap, cost) + 1]
    __shared__ int32_t ok;
    const bool cost = a.kept_cnt != nullptr;
    const int32_t nbins = setup_bins(a.nb_cap, cost);
    if (threadIdx.x == 0) {
        int32_t good = 1, bad = -1;
        int32_t nb_acc = 0, nq_acc = 0, nt_acc = 0;
        if (a.cu_q[0] != 0 || a.cu_k[0] != 0) { good = 0; bad = 0; }
        a.cu_blocks[0] = 0;
        a.cu_qblocks[0] = 0;
        a.cu_tiles[0] = 0;
        for (int32_t b = 0; good && b < a.batch; ++b) {
            const int32_t lk = a.cu_k[b + 1] - a.cu_k[b];
            const int32_t lq = a.cu_q[b + 1] - a.cu_q[b];
            if (lq < 0 || lk < lq || lk > a.max_seqlen) { good = 0; bad = b + 1; break; }
            const int32_t nb = (lk + kBlock - 1) / kBlock;
            if (a.paged && nb > a.max_blocks_per_seq) { good = 0; bad = b + 1; break; }
            const int32_t nq = nb - req_span(a.cu_q, a.cu_k, b).i0;
            nb_acc += nb;
            nq_acc += nq;
            nt_acc += (nq + a.qt - 1) / a.qt;
            a.cu_blocks[b + 1] = nb_acc;
            a.cu_qblocks[b + 1] = nq_acc;
            a.cu_tiles[b + 1] = nt_acc;
        }
        if (good && (a.cu_q[a.batch] != a.total_q || a.cu_k[a.batch] != a.total_k)) { good = 0; bad = a.batch; }
        if (good && nb_acc > a.max_blocks) { good = 0; bad = a.batch; }
        a.hdr->valid = good;
        a.hdr->total_blocks = good ? nb_acc : 0;
        a.hdr->total_qblocks = good ? nq_acc : 0;
        a.hdr->work_next = 0;
        if (!good) set_error(a.hdr, FP2_ERR_BAD_INDEX, bad);
        ok = good;
    }
    if (cost)
        for (int32_t e = threadIdx.x; e <= nbins; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    if (!ok) return;
    // request of every key block and q-block; for the attention call, the
    // histogram of the work items' costs
    for (int32_t b = 0; b < a.batch; ++b) {
        for (int32_t t = a.cu_blocks[b] + threadIdx.x; t < a.cu_blocks[b + 1]; t += blockDim.x)
            a.blk_req[t] = b;
        const int32_t i0 = req_span(a.cu_q, a.cu_k, b).i0, cq = a.cu_qblocks[b];
        for (int32_t t = cq + threadIdx.x; t < a.cu_qblocks[b + 1]; t += blockDim.x) {
            a.blk_req_q[t] = b;
            if (cost)
                for (int32_t g = 0; g < a.hkv; ++g) atomicAdd(&hist[item_cost(a, t, i0 + t - cq, g)], 1);
        }
    }
    // the estimator call needs no work order
    if (!cost) return;
    __syncthreads();
    // order: largest cost first, so the persistent attention kernel takes the
    // longest work items first.  Exclusive scan of the histogram in descending
    // cost order: each thread scans a contiguous run of bins, the runs' totals
    // are scanned across the block.
    {
        __shared__ int32_t wsum[32];
        const int32_t tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
        const int32_t nwarps = (blockDim.x + 31) >> 5;
        const int32_t per = (nbins + blockDim.x - 1) / blockDim.x;
        const int32_t p0 = min(nbins, tid * per), p1 = min(nbins, p0 + per);
        int32_t local = 0;
        for (int32_t p = p0; p < p1; ++p) local += hist[nbins - 1 - p];
        int32_t incl = local;
        for (int32_t o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int32_t v = lane < nwarps ? wsum[lane] : 0;
            int32_t vi = v;
            for (int32_t o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, vi, o);
                if (lane >= o) vi += y;
            }
            wsum[lane] = vi - v;
        }
        __syncthreads();
        int32_t run = wsum[warp] + incl - local;
        for (int32_t p = p0; p < p1; ++p) {
            const int32_t j = nbins - 1 - p;
            const int32_t c = hist[j];
            hist[j] = run;
            run += c;
        }
    }
    __syncthreads();
    for (int32_t b = 0; b < a.batch; ++b) {
        const int32_t i0 = req_span(a.cu_q, a.cu_k, b).i0, cq = a.cu_qblocks[b];
        for (int32_t t = cq + threadIdx.x; t < a.cu_qblocks[b + 1]; t += blockDim.x)
            for (int32_t g = 0; g < a.hkv; ++g)
                a.order[atomicAdd(&hist[item_cost(a, t, i0 + t - cq, g)], 1)] = t * a.hkv + g;
    }
}

// ---------------------------------------------------------------------------
// pooling: mean over the valid rows of every block, per column
//
// Persistent: one CTA per SM walks the units (block t, column slab y of
// tensor x).  A producer warp streams each unit's rows into a ring of
// shared-memory stages with TMA (32 rows of one slab, up to 64 KB per stage),
// so the bytes in flight per SM do not depend on the consumers' registers.
// 16 consumer warps (4 row groups x 128 lanes of 16 bytes) accumulate in fp32
// and, after the unit's last stage, reduce the row groups through shared
// memory.  Rows past a request's end are loaded (or zero-filled past the
// tensor) but not summed; pages are checked against the pool size.
// ---------------------------------------------------------------------------
namespace {
constexpr int kPoolStages = 3;
constexpr int kPoolStageRows = 32;
constexpr int kPoolStageBytes = 65536;
constexpr int kPoolConsumers = kPoolThreads - 32;
static_assert(kPoolConsumers == 512, "4 row groups x 128 column lanes");

struct PoolSmem {
    uint64_t full[kPoolStages];
    uint64_t empty[kPoolStages];
    int32_t abort;
};

struct PoolUnit {
    int32_t x, y, t, b;  // tensor, column slab, block (q-block for x = 0, else key block), request
    int64_t row0;        // first row of the block in the tensor (before paging)
    int32_t j;           // key block index in the request (x > 0)
    int32_t n;           // rows of the block
};

// Units: the q-blocks' column slabs of Q first (ysq per q-block), then the key
// blocks' slabs of K and V (yskv per key block).  A q-block holds the query rows
// at positions [max(P, bs i), min(Lk, bs i + bs)); a key block the keys
// [bs j, min(Lk, bs j + bs)).
__device__ __forceinline__ PoolUnit pool_unit(const PoolArgs& a, int32_t u, int32_t nq, int32_t ysq,
                                              int32_t yskv) {
    PoolUnit p;
    if (u < nq * ysq) {
        p.x = 0;
        p.t = u / ysq;
        p.y = u % ysq;
        p.b = a.blk_req_q[p.t];
        const ReqSpan r = req_span(a.cu_q, a.cu_k, p.b);
        const int32_t i = r.i0 + p.t - a.cu_qblocks[p.b];
        const int32_t lo = max(r.p, i * kBlock);
        p.j = i;
        p.row0 = a.cu_q[p.b] + static_cast<int64_t>(lo - r.p);
        p.n = min(r.lk, i * kBlock + kBlock) - lo;
        return p;
    }
    u -= nq * ysq;
    p.t = u / yskv;
    p.y = u % yskv;
    p.x = max(a.first, 1);
    while (p.x < a.last - 1 && p.y >= a.slabs[p.x]) {
        p.y -= a.slabs[p.x];
        ++p.x;
    }
    p.b = a.blk_req[p.t];
    p.j = p.t - a.cu_blocks[p.b];
    p.row0 = a.cu_k[p.b] + static_cast<int64_t>(p.j) * kBlock;
    p.n = min(kBlock, a.cu_k[p.b + 1] - a.cu_k[p.b] - p.j * kBlock);
    return p;
}

__device__ __forceinline__ void named_sync_pool() {
    asm volatile("bar.sync 1, %0;" ::"n"(kPoolConsumers) : "memory");
}
}  // namespace

template <bool kE4M3>
struct PoolVec;
template <>
struct PoolVec<false> {  // 8 bf16 per 16 bytes
    static constexpr int N = 8;
    __device__ static void unpack(float* x, uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
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
    __device__ static void unpack(float* x, uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFF), __NV_E4M3);
            __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(
                static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3);
            float2 a = __half22float2(*reinterpret_cast<__half2*>(&lo));
            float2 b = __half22float2(*reinterpret_cast<__half2*>(&hi));
            x[4 * i] = a.x;
            x[4 * i + 1] = a.y;
            x[4 * i + 2] = b.x;
            x[4 * i + 3] = b.y;
        }
    }
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

size_t pool_smem_bytes(bool e4m3) {
    const int n = e4m3 ? 16 : 8;
    return 1024 + static_cast<size_t>(kPoolStages) * kPoolStageBytes +
           sizeof(float) * 3 * 128 * (n + 1) + sizeof(PoolSmem);
}

template <bool kE4M3>
__global__ void __launch_bounds__(kPoolThreads, 1)
    pool_kernel(const __grid_constant__ PoolArgs a, const __grid_constant__ CUtensorMap tq,
                const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
    using V = PoolVec<kE4M3>;
    constexpr int N = V::N;
    constexpr int kEsz = kE4M3 ? 1 : 2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~uintptr_t(1023));
    float(*red)[128][N + 1] =
        reinterpret_cast<float(*)[128][N + 1]>(stages + kPoolStages * kPoolStageBytes);
    PoolSmem* ps = reinterpret_cast<PoolSmem*>(stages + kPoolStages * kPoolStageBytes +
                                               sizeof(float) * 3 * 128 * (N + 1));
    volatile int32_t* abort = &ps->abort;
    WsHeader* hdr = a.hdr;
    if (!hdr->valid) return;
    const int32_t ysq = a.first == 0 ? a.slabs[0] : 0;
    int32_t yskv = 0;
    for (int x = max(a.first, 1); x < a.last; ++x) yskv += a.slabs[x];
    const int32_t nq = hdr->total_qblocks;
    const int32_t units = nq * ysq + hdr->total_blocks * yskv;
    const int32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int st = 0; st < kPoolStages; ++st) {
            mbar_init(&ps->full[st], 1);
            mbar_init(&ps->empty[st], kPoolConsumers / 32);
        }
        ps->abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kPoolConsumers / 32) {
        // ---- producer ---------------------------------------------------------
        if (lane == 0) {
            const CUtensorMap* maps[3] = {&tq, &tk, &tv};
            int32_t cnt = 0;
            bool ok = true;
            for (int32_t u = blockIdx.x; ok && u < units; u += gridDim.x) {
                const PoolUnit p = pool_unit(a, u, nq, ysq, yskv);
                int64_t row0 = p.row0;
                if (a.paged[p.x]) {
                    int32_t page = a.block_table[static_cast<int64_t>(p.b) * a.max_blocks_per_seq + p.j];
                    if (page < 0 || page >= a.num_pages) {
                        set_error(hdr, FP2_ERR_BAD_INDEX, p.t);
                        page = 0;
                    }
                    row0 = static_cast<int64_t>(page) * kBlock;
                }
                const uint32_t bytes = static_cast<uint32_t>(a.hb[p.x]) * kHeadDim * kEsz * kPoolStageRows;
                const int32_t nsub = (p.n + kPoolStageRows - 1) / kPoolStageRows;
                for (int32_t sub = 0; sub < nsub; ++sub, ++cnt) {
                    const int32_t st = cnt % kPoolStages;
                    if (!(ok = mbar_wait(&ps->empty[st], ((cnt / kPoolStages) & 1) ^ 1, hdr, abort,
                                         700000 + sub)))
                        break;
                    mbar_arrive_expect_tx(&ps->full[st], bytes);
                    tma_load_3d(stages + st * kPoolStageBytes, maps[p.x], &ps->full[st], 0,
                                p.y * a.hb[p.x], static_cast<int32_t>(row0 + sub * kPoolStageRows));
                }
            }
            // the issued copies land before the CTA exits (the consumers may have
            // stopped waiting after an abort)
            for (int32_t c = max(0, cnt - kPoolStages); c < cnt; ++c)
                mbar_wait_drain(&ps->full[c % kPoolStages], (c / kPoolStages) & 1);
        }
    } else {
        // ---- consumers: thread (row group rg, 16-byte column lane tc) -----------
        const int32_t tc = tid & 127;
        const int32_t rg = tid >> 7;
        int32_t cnt = 0;
        bool ok = true;
        for (int32_t u = blockIdx.x; u < units; u += gridDim.x) {
            const PoolUnit p = pool_unit(a, u, nq, ysq, yskv);
            const int32_t x = p.x;
            const int32_t row_bytes = a.hb[x] * kHeadDim * kEsz;   // one row of the slab
            const int32_t ncols = a.heads[x] * kHeadDim;
            const int32_t col = p.y * a.hb[x] * kHeadDim + tc * N;
            const bool active = tc * 16 < row_bytes && col < ncols;
            // key units with a variance output also sum (x - shift)^2, the shift
            // being the block's first row (no cancellation for a large mean)
            const bool var_unit = x == 1 && a.kvar != nullptr;
            float acc[N];
            float sh[N];
            float sq = 0.f;
#pragma unroll
            for (int e = 0; e < N; ++e) acc[e] = sh[e] = 0.f;
            const int32_t nsub = (p.n + kPoolStageRows - 1) / kPoolStageRows;
            for (int32_t sub = 0; sub < nsub; ++sub, ++cnt) {
                const int32_t st = cnt % kPoolStages;
                // after a failed wait nothing more is read, but every consumer
                // still passes the same named barriers
                if (ok) ok = mbar_wait(&ps->full[st], (cnt / kPoolStages) & 1, hdr, abort, 710000 + sub);
                if (ok && active) {
                    const uint8_t* base = stages + st * kPoolStageBytes + tc * 16;
                    const int32_t nr = min(kPoolStageRows, p.n - sub * kPoolStageRows);
                    if (!var_unit) {
#pragma unroll 4
                        for (int32_t rr = rg; rr < nr; rr += 4)
                            V::add(acc, *reinterpret_cast<const uint4*>(base + rr * row_bytes));
                    } else {
                        if (sub == 0) V::unpack(sh, *reinterpret_cast<const uint4*>(base));
#pragma unroll 2
                        for (int32_t rr = rg; rr < nr; rr += 4) {
                            float xv[N];
                            V::unpack(xv, *reinterpret_cast<const uint4*>(base + rr * row_bytes));
#pragma unroll
                            for (int e = 0; e < N; ++e) {
                                acc[e] += xv[e];
                                const float dv = xv[e] - sh[e];
                                sq = fmaf(dv, dv, sq);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ps->empty[st]);
            }
            if (rg > 0) {
#pragma unroll
                for (int e = 0; e < N; ++e) red[rg - 1][tc][e] = acc[e];
                red[rg - 1][tc][N] = sq;
            }
            named_sync_pool();
            if (rg == 0 && var_unit) {
                // mean key variance of every head of the slab: per lane, the sum over
                // its columns of E[(x - s)^2] - (mean - s)^2; then the lanes of a head
                // (warp-aligned groups of 128 / N) add up, and the first one writes
                float lv = 0.f;
                if (active && ok) {
#pragma unroll
                    for (int g = 0; g < 3; ++g) sq += red[g][tc][N];
                    float m2 = 0.f;
#pragma unroll
                    for (int e = 0; e < N; ++e) {
                        float tot = acc[e];
#pragma unroll
                        for (int g = 0; g < 3; ++g) tot += red[g][tc][e];
                        const float dm = tot / static_cast<float>(p.n) - sh[e];
                        m2 = fmaf(dm, dm, m2);
                    }
                    lv = sq / static_cast<float>(p.n) - m2;
                }
#pragma unroll
                for (int o = 1; o < kHeadDim / N; o <<= 1) lv += __shfl_xor_sync(0xffffffffu, lv, o);
                if (active && ok && (tc % (kHeadDim / N)) == 0) {
                    const int32_t h = col / kHeadDim;
                    const float s = a.scale[x] ? a.scale[x][h] : 1.f;
                    a.kvar[static_cast<int64_t>(p.t) * a.heads[x] + h] = fmaxf(lv, 0.f) * s * s / kHeadDim;
                }
            }
            if (rg == 0 && active && ok) {
#pragma unroll
                for (int g = 0; g < 3; ++g)
#pragma unroll
                    for (int e = 0; e < N; ++e) acc[e] += red[g][tc][e];
                const int32_t h = col / kHeadDim;
                const float sc = (a.scale[x] ? a.scale[x][h] : 1.f) / static_cast<float>(p.n);
#pragma unroll
                for (int e = 0; e < N; ++e) acc[e] *= sc;
                const int32_t t = p.t;
                if (a.out[x]) {
                    float* out = a.out[x] + static_cast<int64_t>(t) * ncols + col;
#pragma unroll
                    for (int e = 0; e < N; e += 4)
                        *reinterpret_cast<float4*>(out + e) =
                            make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
                }
                if (x < 2) {
                    // hi + lo bf16 parts for the score MMAs: hi = bf16(m), lo = bf16(m - hi)
                    int64_t row;
                    if (x == 0) {
                        const int32_t g = h / a.G, hh = h % a.G;
                        row = (static_cast<int64_t>(g) * a.max_blocks + t) * a.G + hh;
                    } else {
                        row = static_cast<int64_t>(h) * a.max_blocks + t;
                    }
                    const int64_t plane =
                        static_cast<int64_t>(a.heads[x]) * a.max_blocks * kHeadDim;
                    uint16_t* hi = a.split[x] + row * kHeadDim + (col % kHeadDim);
                    uint16_t* lo = hi + plane;
                    uint32_t ph[N / 2], pl[N / 2];
#pragma unroll
                    for (int e = 0; e < N; e += 2) {
                        const uint32_t hp = pack_bf16(acc[e], acc[e + 1]);
                        const float h0 = __uint_as_float(hp << 16), h1 = __uint_as_float(hp & 0xFFFF0000u);
                        ph[e / 2] = hp;
                        pl[e / 2] = pack_bf16(acc[e] - h0, acc[e + 1] - h1);
                    }
#pragma unroll
                    for (int e = 0; e < N / 2; e += 4) {
                        *reinterpret_cast<uint4*>(hi + 2 * e) = make_uint4(ph[e], ph[e + 1], ph[e + 2], ph[e + 3]);
                        *reinterpret_cast<uint4*>(lo + 2 * e) = make_uint4(pl[e], pl[e + 1], pl[e + 2], pl[e + 3]);
                    }
                }
            }
            named_sync_pool();  // red is reused by the next unit
        }
    }
}

// ---------------------------------------------------------------------------
// scores, threshold, union, compaction (tcgen05)
//
// One CTA = one KV head g x one tile of qt = floor(128 / G) q-blocks of one
// request: 128 rows (q-block, query head) of qbar against all causal key
// blocks, 128 key blocks per chunk.  s = tau * qbar . kbar is computed on the
// tensor cores as hi.hi + hi.lo + lo.hi with bf16 hi/lo parts of the fp32
// means (relative error about 2^-16, the fp32 accumulation in TMEM).
//   pass 1: row max m over j <= i
//   pass 2: the same scores again; keep bit = exp(s - m) >= alpha (or j == i);
//           OR over the G rows of each q-block; ascending compaction.
// warps 0-3: epilogue (row r = TMEM lane r); warp 4: TMA loads and MMA issue.
// ---------------------------------------------------------------------------
namespace {
constexpr int kTileQ = 32768;   // one 128 x 128 bf16 operand (two 64-column chunks)

struct ScoreSmem {
    uint64_t q_full;
    uint64_t kv_full[2];
    uint64_t kv_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    int32_t abort;
    uint32_t keep[128][4];
};

__device__ __forceinline__ uint64_t score_desc(uint32_t base, int k) {
    return sdesc_sw128(base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
}

__device__ __forceinline__ void named_sync_epi() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}
}  // namespace

__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ ScoreArgs a, const __grid_constant__ CUtensorMap tqh,
                 const __grid_constant__ CUtensorMap tql, const __grid_constant__ CUtensorMap tkh,
                 const __grid_constant__ CUtensorMap tkl) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* qh = sm;
    uint8_t* ql = sm + kTileQ;
    uint8_t* kh = sm + 2 * kTileQ;      // 2 stages
    uint8_t* kl = sm + 4 * kTileQ;      // 2 stages
    ScoreSmem* ss = reinterpret_cast<ScoreSmem*>(sm + 6 * kTileQ);
    volatile int32_t* abort = &ss->abort;
    WsHeader* hdr = a.hdr;
    if (!hdr->valid) return;
    const int32_t total_tiles = a.cu_tiles[a.batch];
    if (static_cast<int32_t>(blockIdx.y) >= total_tiles) return;
    // grid (KV head, tile): CTAs start in launch order, so with heads fastest
    // the late (long-row) tiles of every head start first
    const int32_t tile = total_tiles - 1 - blockIdx.y;
    int32_t lo = 0, hi = a.batch - 1;                   // request owning this tile
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (a.cu_tiles[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int32_t b = lo;
    const int32_t g = blockIdx.x;
    const int32_t G = a.G;
    const int32_t cb = a.cu_blocks[b];                  // first key block of the request
    const int32_t cq = a.cu_qblocks[b];                 // first q-block of the request
    const int32_t nbq = a.cu_qblocks[b + 1] - cq;
    const int32_t l0 = (tile - a.cu_tiles[b]) * a.qt;   // the tile's first q-block (in the request)
    const int32_t nq = min(a.qt, nbq - l0);
    const int32_t i0 = req_span(a.cu_q, a.cu_k, b).i0 + l0;  // its absolute block index
    const int32_t nrows = nq * G;
    const int32_t nchunk = (i0 + nq - 1) / 128 + 1;
    const int32_t steps = 2 * nchunk;
    const int32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 4) {
        tmem_alloc(&ss->tmem_base, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&ss->q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ss->kv_full[s], 1);
            mbar_init(&ss->kv_empty[s], 1);
            mbar_init(&ss->acc_full[s], 1);
            mbar_init(&ss->acc_empty[s], 128);
        }
        ss->abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ss->tmem_base;

    if (warp == 4) {
        if (lane == 0) {
            const int32_t qrow = (g * static_cast<int32_t>(a.max_blocks) + cq + l0) * G;
            const int32_t krow = g * static_cast<int32_t>(a.max_blocks) + cb;
            mbar_arrive_expect_tx(&ss->q_full, 2 * kTileQ);
            for (int ch = 0; ch < 2; ++ch) {
                tma_load_2d(qh + ch * 16384, &tqh, &ss->q_full, ch * 64, qrow);
                tma_load_2d(ql + ch * 16384, &tql, &ss->q_full, ch * 64, qrow);
            }
            int32_t nload = 0;  // K chunk loads issued
            auto load = [&](int32_t idx) -> bool {
                const int32_t s = idx & 1;
                if (!mbar_wait(&ss->kv_empty[s], ((idx >> 1) & 1) ^ 1, hdr, abort, 600000 + idx))
                    return false;
                const int32_t row = krow + (idx % nchunk) * 128;
                mbar_arrive_expect_tx(&ss->kv_full[s], 2 * kTileQ);
                for (int ch = 0; ch < 2; ++ch) {
                    tma_load_2d(kh + s * kTileQ + ch * 16384, &tkh, &ss->kv_full[s], ch * 64, row);
                    tma_load_2d(kl + s * kTileQ + ch * 16384, &tkl, &ss->kv_full[s], ch * 64, row);
                }
                ++nload;
                return true;
            };
            bool ok = load(0) && mbar_wait(&ss->q_full, 0, hdr, abort, 610000);
            const uint32_t idesc = idesc_make(kFmtBF16, 0, 128);
            for (int32_t idx = 0; ok && idx < steps; ++idx) {
                const int32_t s = idx & 1;
                if (idx + 1 < steps && !(ok = load(idx + 1))) break;
                if (!(ok = mbar_wait(&ss->kv_full[s], (idx >> 1) & 1, hdr, abort, 620000 + idx) &&
                           mbar_wait(&ss->acc_empty[s], ((idx >> 1) & 1) ^ 1, hdr, abort, 630000 + idx)))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + s * 128;
                const uint32_t ah = smem_u32(qh), al = smem_u32(ql);
                const uint32_t bh = smem_u32(kh + s * kTileQ), bl = smem_u32(kl + s * kTileQ);
#pragma unroll
                for (int k = 0; k < 8; ++k) mma_bf16_ss(d, score_desc(ah, k), score_desc(bh, k), idesc, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k) mma_bf16_ss(d, score_desc(ah, k), score_desc(bl, k), idesc, 1);
#pragma unroll
                for (int k = 0; k < 8; ++k) mma_bf16_ss(d, score_desc(al, k), score_desc(bh, k), idesc, 1);
                mma_commit(&ss->acc_full[s]);
                mma_commit(&ss->kv_empty[s]);
            }
            // all loads consumed before the CTA exits; after an abort, at least landed
            for (int32_t idx = max(0, steps - 2); ok && idx < steps; ++idx)
                ok = mbar_wait(&ss->kv_empty[idx & 1], (idx >> 1) & 1, hdr, abort, 640000 + idx);
            if (!ok) {
                for (int32_t idx = max(0, nload - 2); idx < nload; ++idx)
                    mbar_wait_drain(&ss->kv_full[idx & 1], (idx >> 1) & 1);
                mbar_wait_drain(&ss->q_full, 0);
            }
        }
    } else {
        // ---- epilogue: row r of the tile ---------------------------------------
        // keep bit for key block j <= i: s - m >= ln(alpha), tested on the raw
        // accumulator as acc >= (m + ln(alpha)) / tau (tau > 0).  The G rows of a
        // q-block are G consecutive lanes when G divides 32 (warp shuffles OR
        // them); otherwise they meet in shared memory.
        const int32_t r = tid;
        const bool valid = r < nrows;
        const int32_t ii = valid ? r / G : 0;
        const int32_t hh = valid ? r % G : 0;
        const int32_t i = i0 + ii;
        const int32_t h = g * G + hh;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const bool lanes_group = (32 % G) == 0;
        float m = -INFINITY;
        float thr_raw = 0.f;
        int32_t cnt = 0;  // kept blocks of this q-block (group leader lane / owner thread)
        const bool leader = lanes_group ? (valid && hh == 0) : (r < nq);
        const int32_t lead_i = lanes_group ? i : i0 + r;
        const int64_t own_row = static_cast<int64_t>(cq + l0 + (lead_i - i0)) * a.hkv + g;
        bool ok = true;
        for (int32_t idx = 0; idx < steps; ++idx) {
            const int32_t s = idx & 1;
            const int32_t c = idx % nchunk;
            const bool pass2 = idx >= nchunk;
            ok = __all_sync(0xffffffffu, mbar_wait(&ss->acc_full[s], (idx >> 1) & 1, hdr, abort,
                                                   650000 + idx)) && ok;
            tc_fence_after();
            uint32_t v[128];
            const uint32_t addr = tmem + lane_off + s * 128;
            tmem_ld32(addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
            tmem_ld32(addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
            tmem_ld32(addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&v[64]));
            tmem_ld32(addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&v[96]));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&ss->acc_empty[s]);
            const int32_t j0 = c * 128;
            const bool full = j0 + 127 <= i;  // every column of the chunk is causal for this row
            if (!pass2) {
                float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (full) {
#pragma unroll
                    for (int e = 0; e < 128; ++e) mp[e & 3] = fmaxf(mp[e & 3], __uint_as_float(v[e]));
                } else {
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        if (j0 + e <= i) mp[e & 3] = fmaxf(mp[e & 3], __uint_as_float(v[e]));
                }
                m = fmaxf(m, fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])));
                if (idx == nchunk - 1) {
                    m *= a.tau;                       // row max of s
                    thr_raw = (m + a.ln_alpha) / a.tau;
                }
                continue;
            }
            uint32_t bits[4] = {0u, 0u, 0u, 0u};
            if (valid) {
                if (a.keep_all) {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int32_t lim = i - (j0 + 32 * w);   // keep j <= i
                        bits[w] = lim >= 31 ? 0xffffffffu : (lim < 0 ? 0u : ((2u << lim) - 1u));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        bits[e >> 5] |= (__uint_as_float(v[e]) >= thr_raw) ? (1u << (e & 31)) : 0u;
                    if (!full) {
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            const int32_t lim = i - (j0 + 32 * w);
                            bits[w] &= lim >= 31 ? 0xffffffffu : (lim < 0 ? 0u : ((2u << lim) - 1u));
                        }
                    }
                    if (i >= j0 && i < j0 + 128) bits[(i - j0) >> 5] |= 1u << ((i - j0) & 31);  // diagonal
                }
                if (a.score_dbg) {
                    float* dbg = a.score_dbg + (static_cast<int64_t>(cq + l0 + ii) * a.hq + h) * a.nb_max;
#pragma unroll
                    for (int e = 0; e < 128; ++e)
                        if (j0 + e <= i) dbg[j0 + e] = __uint_as_float(v[e]) * a.tau - m;
                }
            }
            uint32_t u[4];
            if (lanes_group) {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    u[w] = bits[w];
                    for (int o = 1; o < G; o <<= 1) u[w] |= __shfl_xor_sync(0xffffffffu, u[w], o);
                }
            } else {
#pragma unroll
                for (int w = 0; w < 4; ++w) ss->keep[r][w] = bits[w];
                named_sync_epi();
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    u[w] = 0;
                    if (r < nq)
                        for (int32_t q = 0; q < G; ++q) u[w] |= ss->keep[r * G + q][w];
                }
                named_sync_epi();
            }
            if (ok && leader) {
                int32_t* dst = a.kept_idx + own_row * a.nb_max;
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t x = u[w];
                    while (x) {
                        const int bit = __ffs(x) - 1;
                        x &= x - 1;
                        dst[cnt++] = j0 + w * 32 + bit;
                    }
                }
            }
        }
        if (ok && leader) a.kept_cnt[own_row] = cnt;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

size_t score_smem_bytes() { return 1024 + 6 * kTileQ + sizeof(ScoreSmem); }

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

template __global__ void pool_kernel<false>(const __grid_constant__ PoolArgs,
                                            const __grid_constant__ CUtensorMap,
                                            const __grid_constant__ CUtensorMap,
                                            const __grid_constant__ CUtensorMap);
template __global__ void pool_kernel<true>(const __grid_constant__ PoolArgs,
                                           const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap,
                                           const __grid_constant__ CUtensorMap);

}  // namespace fp2

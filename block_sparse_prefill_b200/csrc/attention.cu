// attention.cu -- sparse flash attention over the kept key blocks with the mean
// correction of the pruned blocks, for sm_100a (tcgen05 MMA, TMEM accumulators,
// TMA tile loads).
//
// What it computes (the method of the FlashPrefill V2 write-ups: lode.cx,
// "How It Works" -- attend only the blocks that pass the max-relative threshold
// and add a mean correction term for the pruned ones; aimodeling.com, "From
// Prototype to Production" -- FP8, paged KV cache, continuous batching): for
// row r of q-block i and query head h (KV head g = h / G),
//   o_r = [sum_{kept c <= r} e^{l_c} v_c + sum_{pruned j<i} 128 e^{lbar_j} vbar_j]
//       / [sum_{kept c <= r} e^{l_c}     + sum_{pruned j<i} 128 e^{lbar_j}]
// with l_c = tau q_r . k_c and lbar_j = tau q_r . kbar_j (pruned blocks are full).
//
// Structure (one CTA = one q-block x two query heads of one KV head, so every
// K/V tile fetched into shared memory serves both heads):
//   warps 0-3  softmax of Q tile 0 (one thread per row, rows = TMEM lanes)
//   warps 4-7  softmax of Q tile 1
//   warp  8    TMA producer: Q tiles, then K/V (or mean-K/mean-V) tiles into a
//              ring of shared-memory slots, following the kept list and, in
//              paged mode, the block table
//   warp  9    TMEM owner and MMA issuer: S_t = Q_t K^T (both operands in shared
//              memory), O_t += P_t V (P_t from TMEM, V from shared memory)
// TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,384) O_1 [384,512); P_t is
// written over the first columns of S_t.  The running max is only raised when
// it grows by more than a threshold (log2 units), so O is rarely rescaled.
// Tile order: diagonal block first (it fixes the causal mask and usually the
// row max), then the other kept blocks from nearest to farthest, then the
// correction tiles: 128 consecutive block means each, with the kept ones (and
// those >= i) masked out.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace fp2 {

namespace {

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;

template <bool kE4M3>
struct Cfg {
    static constexpr int kEsz = kE4M3 ? 1 : 2;
    static constexpr int kTileBytes = 128 * 128 * kEsz;     // one 128 x 128 operand tile
    static constexpr int kSlots = kE4M3 ? 8 : 4;            // K/V ring slots
    static constexpr int kChunks = kE4M3 ? 1 : 2;           // 128-byte-wide column chunks per row
    static constexpr int kKSteps = kE4M3 ? 4 : 8;           // MMA K steps per 128
    static constexpr uint32_t kFmt = kE4M3 ? kFmtE4M3 : kFmtBF16;
    static constexpr uint32_t kIdescQK = idesc_make(kFmt, 0, 128);
    static constexpr uint32_t kIdescPV = idesc_make(kFmt, 1, 128);
    // P = 2^(x - m + kPOffset); the running max m is raised only when a row max
    // exceeds it by more than kRescale, so P <= 2^(kPOffset + kRescale).
    // e4m3: P scaled by 2^8 keeps small weights out of the subnormal range
    // (the scale cancels in O / l) with P <= 2^8.75 < 448, the e4m3 maximum.
    // bf16: no offset, and O is rescaled only for jumps above 2^8.
    static constexpr float kPOffset = kE4M3 ? 8.f : 0.f;
    static constexpr float kRescale = kE4M3 ? 0.75f : 8.f;
};

struct Bars {
    uint64_t q_full;
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done[2];
    uint64_t kv_full[8];
    uint64_t kv_empty[8];
    uint64_t v_tail;      // V rows past the request end zeroed (partial diagonal block)
};

struct SmemMisc {
    Bars bars;
    uint32_t tmem_base;
    int32_t abort;
    int32_t cnt;      // kept blocks
    int32_t ncorr;    // correction tiles
};

template <bool kE4M3>
__host__ __device__ constexpr size_t tiles_bytes() {
    return static_cast<size_t>(2 + Cfg<kE4M3>::kSlots) * Cfg<kE4M3>::kTileBytes;
}

__host__ __device__ inline size_t lists_bytes(int32_t nb_max) {
    // kept list + pruned bitmask + correction tile list
    return sizeof(int32_t) * (nb_max + (nb_max + 31) / 32 + (nb_max + 127) / 128 + 4);
}

// Descriptor of K-major operand step k (Q or K tile at `base`).
template <bool kE4M3>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int k) {
    const uint32_t addr = kE4M3 ? base + k * 32 : base + (k >> 2) * 16384 + (k & 3) * 32;
    return sdesc_sw128(addr, 16, 1024);
}

// Descriptor of the MN-major V tile, keys [k*K, (k+1)*K).
template <bool kE4M3>
__device__ __forceinline__ uint64_t vmajor_desc(uint32_t base, int k) {
    const uint32_t addr = base + k * (kE4M3 ? 4096 : 2048);
    return sdesc_sw128(addr, 16384, 1024);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr,
                                          volatile int32_t* abort, int32_t where) {
    const bool ok = mbar_wait(bar, parity, hdr, abort, where);
    return __all_sync(0xffffffffu, ok);
}

}  // namespace

template <bool kE4M3>
__global__ void __launch_bounds__(kThreads, 1)
    attention_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap tq,
                     const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                     const __grid_constant__ CUtensorMap tkb,
                     const __grid_constant__ CUtensorMap tvb) {
    using C = Cfg<kE4M3>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* q_s = smem;                                  // 2 tiles
    uint8_t* kv_s = smem + 2 * C::kTileBytes;             // kSlots tiles
    SmemMisc* misc = reinterpret_cast<SmemMisc*>(smem + tiles_bytes<kE4M3>());
    int32_t* klist = reinterpret_cast<int32_t*>(misc + 1);
    uint32_t* pruned = reinterpret_cast<uint32_t*>(klist + a.nb_cap);
    int32_t* ctiles = reinterpret_cast<int32_t*>(pruned + (a.nb_cap + 31) / 32);
    Bars& bars = misc->bars;
    volatile int32_t* abort = &misc->abort;

    // ---- work item ---------------------------------------------------------
    WsHeader* hdr = a.hdr;
    if (!hdr->valid) return;
    const int32_t total_blocks = hdr->total_blocks;
    const int32_t per_blk = a.hkv * a.pairs;
    const int32_t t_rev = blockIdx.x / per_blk;
    if (t_rev >= total_blocks) return;
    const int32_t t = total_blocks - 1 - t_rev;  // late q-blocks (long kept lists) first
    const int32_t rem = blockIdx.x % per_blk;
    const int32_t g = rem / a.pairs;
    const int32_t hp = rem % a.pairs;
    const int32_t h0 = g * a.G + 2 * hp;
    const int32_t ntiles = min(2, a.G - 2 * hp);
    const int32_t b = a.blk_req[t];
    const int32_t cb = a.cu_blocks[b];
    const int32_t i = t - cb;
    const int32_t L = a.cu[b + 1] - a.cu[b];
    const int32_t nrows = min(kBlock, L - i * kBlock);
    const int32_t qrow0 = a.cu[b] + i * kBlock;

    const int32_t tid = threadIdx.x;
    const int32_t warp = tid >> 5;
    const int32_t lane = tid & 31;

    // ---- set-up ------------------------------------------------------------
    if (warp == kMmaWarp) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars.q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars.s_full[s], 1);
            mbar_init(&bars.p_full[s], 128);
            mbar_init(&bars.o_done[s], 1);
        }
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.kv_empty[s], 1);
        }
        mbar_init(&bars.v_tail, 1);
        misc->abort = 0;
        fence_mbar_init();
    }
    // kept list of (q-block t, KV head g)
    const int64_t lrow = static_cast<int64_t>(t) * a.hkv + g;
    int32_t cnt = a.kept_cnt[lrow];
    const bool cnt_ok = cnt >= 1 && cnt <= i + 1;
    if (!cnt_ok) cnt = 1;
    const int32_t* src = a.kept_idx + lrow * a.nb_max;
    for (int32_t e = tid; e < cnt; e += kThreads) klist[e] = cnt_ok ? src[e] : i;
    const int32_t nwords = (i + 31) / 32;  // bits for key blocks j < i
    for (int32_t w = tid; w < nwords; w += kThreads) {
        const int32_t lo = w * 32;
        const int32_t nbits = min(32, i - lo);
        pruned[w] = (nbits == 32) ? 0xffffffffu : ((1u << nbits) - 1u);
    }
    __syncthreads();
    if (tid == 0) {
        bool ok = cnt_ok && klist[cnt - 1] == i;
        for (int32_t e = 1; ok && e < cnt; ++e) ok = klist[e] > klist[e - 1] && klist[e - 1] >= 0;
        if (!ok) {
            set_error(hdr, FP2_ERR_BAD_INDEX, t);
            klist[0] = i;
            cnt = 1;
        }
        misc->cnt = cnt;
    }
    __syncthreads();
    cnt = misc->cnt;
    if (a.correction) {
        for (int32_t e = tid; e < cnt - 1; e += kThreads) {
            const int32_t j = klist[e];
            atomicAnd(&pruned[j >> 5], ~(1u << (j & 31)));
        }
    }
    __syncthreads();
    if (tid == 0) {
        int32_t nc = 0;
        if (a.correction) {
            for (int32_t ct = 0; ct * 128 < i; ++ct) {
                uint32_t any = 0;
                for (int32_t w = ct * 4; w < min(ct * 4 + 4, nwords); ++w) any |= pruned[w];
                if (any) ctiles[nc++] = ct;
            }
        }
        misc->ncorr = nc;
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const int32_t ncorr = misc->ncorr;
    const int32_t ntot = cnt + ncorr;

    // ---- roles -------------------------------------------------------------
    if (warp == kProducerWarp) {
        // lane 0 issues every TMA; the whole warp zeroes the V rows past the
        // request end of a partial diagonal block (a paged pool may hold
        // anything there, and zero attention weights times NaN is NaN)
        const bool leader = lane == 0;
        if (leader) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            mbar_arrive_expect_tx(&bars.q_full, ntiles * C::kTileBytes);
            for (int qt = 0; qt < ntiles; ++qt)
                for (int ch = 0; ch < C::kChunks; ++ch)
                    tma_load_3d(q_s + qt * C::kTileBytes + ch * 16384, &tq, &bars.q_full, ch * 64,
                                h0 + qt, qrow0);
        }
        int32_t issued = 0;
        for (int32_t n = 0; n < ntot && !*abort; ++n) {
            const CUtensorMap* mk;
            const CUtensorMap* mv;
            int32_t row = 0;
            if (n < cnt) {
                const int32_t j = klist[cnt - 1 - n];
                mk = &tk;
                mv = &tv;
                if (a.block_table) {
                    int32_t page = a.block_table[static_cast<int64_t>(b) * a.max_blocks_per_seq + j];
                    if (page < 0 || page >= a.num_pages) {
                        if (leader) set_error(hdr, FP2_ERR_BAD_INDEX, t);
                        page = 0;
                    }
                    row = page * kBlock;
                } else {
                    row = a.cu[b] + j * kBlock;
                }
            } else {
                mk = &tkb;
                mv = &tvb;
                row = cb + ctiles[n - cnt] * 128;
            }
            bool ok = true;
            for (int kv = 0; kv < 2 && ok; ++kv) {
                const int32_t idx = 2 * n + kv;
                const int32_t s = idx % C::kSlots;
                if (leader) {
                    ok = mbar_wait(&bars.kv_empty[s], ((idx / C::kSlots) & 1) ^ 1, hdr, abort,
                                   100000 + idx);
                    if (ok) {
                        mbar_arrive_expect_tx(&bars.kv_full[s], C::kTileBytes);
                        for (int ch = 0; ch < C::kChunks; ++ch)
                            tma_load_3d(kv_s + s * C::kTileBytes + ch * 16384, kv ? mv : mk,
                                        &bars.kv_full[s], ch * 64, g, row);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                ++issued;
                if (kv == 1 && n == 0 && nrows < kBlock) {
                    ok = warp_wait(&bars.kv_full[s], (idx / C::kSlots) & 1, hdr, abort, 150000);
                    if (!ok) break;
                    uint8_t* vt = kv_s + s * C::kTileBytes;
                    const int32_t nz = (kBlock - nrows) * 8;  // 16-byte units per chunk
                    for (int ch = 0; ch < C::kChunks; ++ch)
                        for (int32_t e = lane; e < nz; e += 32)
                            *reinterpret_cast<uint4*>(vt + ch * 16384 + nrows * 128 + e * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (leader) mbar_arrive(&bars.v_tail);
                }
            }
            if (!ok) break;
        }
        // drain: every issued tile has been consumed and released
        if (leader) {
            for (int32_t idx = max(0, issued - C::kSlots); idx < issued; ++idx) {
                const int32_t s = idx % C::kSlots;
                if (!mbar_wait(&bars.kv_empty[s], (idx / C::kSlots) & 1, hdr, abort, 200000 + idx))
                    break;
            }
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            const uint32_t q_addr = smem_u32(q_s);
            const uint32_t kv_addr = smem_u32(kv_s);
            bool ok = mbar_wait(&bars.q_full, 0, hdr, abort, 300000);
            tc_fence_after();
            for (int32_t n = 0; ok && n < ntot; ++n) {
                const int32_t ik = 2 * n, iv = 2 * n + 1;
                const int32_t sk = ik % C::kSlots, sv = iv % C::kSlots;
                if (!(ok = mbar_wait(&bars.kv_full[sk], (ik / C::kSlots) & 1, hdr, abort, 310000 + n)))
                    break;
                tc_fence_after();
                for (int qt = 0; qt < ntiles && ok; ++qt) {
                    if (n > 0) {
                        if (!(ok = mbar_wait(&bars.o_done[qt], (n - 1) & 1, hdr, abort, 320000 + n)))
                            break;
                        tc_fence_after();
                    }
                    const uint32_t d_s = tmem + qt * 128;
                    const uint32_t qb = q_addr + qt * C::kTileBytes;
                    const uint32_t kb = kv_addr + sk * C::kTileBytes;
#pragma unroll
                    for (int k = 0; k < C::kKSteps; ++k) {
                        if (kE4M3)
                            mma_f8_ss(d_s, kmajor_desc<kE4M3>(qb, k), kmajor_desc<kE4M3>(kb, k),
                                      C::kIdescQK, k > 0);
                        else
                            mma_bf16_ss(d_s, kmajor_desc<kE4M3>(qb, k), kmajor_desc<kE4M3>(kb, k),
                                        C::kIdescQK, k > 0);
                    }
                    mma_commit(&bars.s_full[qt]);
                }
                if (!ok) break;
                mma_commit(&bars.kv_empty[sk]);
                if (!(ok = mbar_wait(&bars.kv_full[sv], (iv / C::kSlots) & 1, hdr, abort, 330000 + n)))
                    break;
                if (n == 0 && nrows < kBlock &&
                    !(ok = mbar_wait(&bars.v_tail, 0, hdr, abort, 335000)))
                    break;
                tc_fence_after();
                for (int qt = 0; qt < ntiles && ok; ++qt) {
                    if (!(ok = mbar_wait(&bars.p_full[qt], n & 1, hdr, abort, 340000 + n))) break;
                    tc_fence_after();
                    const uint32_t d_o = tmem + 256 + qt * 128;
                    const uint32_t p_t = tmem + qt * 128;
                    const uint32_t vb = kv_addr + sv * C::kTileBytes;
#pragma unroll
                    for (int k = 0; k < C::kKSteps; ++k) {
                        if (kE4M3)
                            mma_f8_ts(d_o, p_t + 8 * k, vmajor_desc<kE4M3>(vb, k), C::kIdescPV,
                                      (n > 0 || k > 0) ? 1u : 0u);
                        else
                            mma_bf16_ts(d_o, p_t + 8 * k, vmajor_desc<kE4M3>(vb, k), C::kIdescPV,
                                        (n > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit(&bars.o_done[qt]);
                }
                if (!ok) break;
                mma_commit(&bars.kv_empty[sv]);
            }
        }
    } else if (warp / 4 < ntiles) {
        // ---- softmax + epilogue of Q tile qt ---------------------------------
        const int qt = warp / 4;
        const int32_t r = tid & 127;
        const int32_t h = h0 + qt;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + qt * 128;
        const uint32_t o_addr = tmem + lane_off + 256 + qt * 128;
        float qk = a.scale_log2;
        if (kE4M3) qk *= a.q_scale[h] * a.k_scale[g];
        float m_ref = -INFINITY;
        float l = 0.f;      // row sum of the weights the PV MMA uses (O normaliser)
        float l_lse = 0.f;  // row sum before P is rounded to the MMA precision (LSE)
        bool ok = true;
        for (int32_t n = 0; n < ntot; ++n) {
            if (!(ok = warp_wait(&bars.s_full[qt], n & 1, hdr, abort, 400000 + n))) break;
            tc_fence_after();
            // logits of this tile in log2 units, masked entries -inf:
            //   diagonal block (n == 0): keys c <= r
            //   kept block: every key
            //   correction tile: pruned block means only, plus log2(128) for the 128 rows each stands for
            const int kind = (n == 0) ? 0 : (n < cnt ? 1 : 2);
            const int32_t w0 = (kind == 2) ? ctiles[n - cnt] * 4 : 0;
            auto logit = [&](uint32_t raw, int c, uint32_t bits) -> float {
                const float sx = __uint_as_float(raw);
                if (kind == 0) return (c <= r) ? sx * qk : -INFINITY;
                if (kind == 1) return sx * qk;
                return ((bits >> (c & 31)) & 1u) ? fmaf(sx, qk, 7.f) : -INFINITY;
            };
            // pass 1: row max
            float mx = -INFINITY;
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 64) {
                uint32_t sv[64];
                tmem_ld32(s_addr + c0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(s_addr + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_wait_ld();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int cw = (c0 >> 5) + half;
                    const uint32_t bits = (kind == 2 && w0 + cw < nwords) ? pruned[w0 + cw] : 0u;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        mx = fmaxf(mx, logit(sv[half * 32 + c], c0 + half * 32 + c, bits));
                }
            }
            const float m_new = fmaxf(m_ref, mx);
            const bool need = m_new > m_ref + C::kRescale;
            if (__any_sync(0xffffffffu, need)) {
                const float f = need ? ex2(m_ref - m_new) : 1.f;
                if (n > 0) {
                    if (!(ok = warp_wait(&bars.o_done[qt], (n - 1) & 1, hdr, abort, 410000 + n))) break;
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < 128; c0 += 32) {
                        uint32_t ov[32];
                        tmem_ld32(o_addr + c0, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * f);
                        tmem_st32(o_addr + c0, ov);
                    }
                    tmem_wait_st();
                }
                if (need) {
                    l *= f;
                    l_lse *= f;
                    m_ref = m_new;
                }
            }
            const float m_use = ((m_ref == -INFINITY) ? 0.f : m_ref) - C::kPOffset;
            // pass 2: P = exp2(x - m) in the MMA precision, written over the
            // already-consumed leading columns of S
            float rs = 0.f, rs_q = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 64) {
                uint32_t sv[64];
                tmem_ld32(s_addr + c0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_ld32(s_addr + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                tmem_wait_ld();
                float p[64];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int cw = (c0 >> 5) + half;
                    const uint32_t bits = (kind == 2 && w0 + cw < nwords) ? pruned[w0 + cw] : 0u;
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const int cc = half * 32 + c;
                        p[cc] = ex2(logit(sv[cc], c0 + cc, bits) - m_use);
                        rs += p[cc];
                    }
                }
                if (kE4M3) {
                    // the row sum takes the quantised weights the PV MMA sees, so
                    // numerator and denominator use the same P
                    uint32_t pk[16];
                    __half2 hs = __float2half2_rn(0.f);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        pk[c] = pack_e4m3x4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
                        hs = __hadd2(hs, e4m3x4_sum2(pk[c]));
                    }
                    const float2 hf = __half22float2(hs);
                    rs_q += hf.x + hf.y;
                    tmem_st16(s_addr + c0 / 4, pk);
                } else {
                    uint32_t pk[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
                    tmem_st32(s_addr + c0 / 2, pk);
                }
            }
            l += kE4M3 ? rs_q : rs;
            l_lse += rs;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars.p_full[qt]);
        }
        // ---- epilogue: O / l -> bf16 ----------------------------------------
        if (ok && ntot > 0 && warp_wait(&bars.o_done[qt], (ntot - 1) & 1, hdr, abort, 420000)) {
            tc_fence_after();
            float inv = 1.f / l;
            if (kE4M3) inv *= a.v_scale[g];
            uint16_t* orow = static_cast<uint16_t*>(a.out) +
                             (static_cast<int64_t>(qrow0 + r) * a.hq + h) * kHeadDim;
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(o_addr + c0, ov);
                tmem_wait_ld();
                if (r < nrows) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        pk[c] = pack_bf16(__uint_as_float(ov[2 * c]) * inv,
                                          __uint_as_float(ov[2 * c + 1]) * inv);
                    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
            }
            if (a.lse && r < nrows) {
                const float m_use = ((m_ref == -INFINITY) ? 0.f : m_ref) - C::kPOffset;
                a.lse[static_cast<int64_t>(qrow0 + r) * a.hq + h] =
                    (m_use + __log2f(l_lse)) * 0.69314718055994530942f;
            }
        }
    }

    // ---- teardown ----------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

size_t attn_smem_bytes(bool e4m3, int32_t nb_cap) {
    const size_t tiles = e4m3 ? tiles_bytes<true>() : tiles_bytes<false>();
    return 1024 + tiles + sizeof(SmemMisc) + lists_bytes(nb_cap);
}

cudaError_t launch_attention(bool e4m3, const AttnArgs& a, const CUtensorMap& tq,
                             const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkb,
                             const CUtensorMap& tvb, int64_t max_blocks, cudaStream_t stream) {
    const size_t smem = attn_smem_bytes(e4m3, a.nb_cap);
    const int64_t grid = max_blocks * a.hkv * a.pairs;
    if (grid <= 0) return cudaSuccess;
    cudaError_t err;
    if (e4m3) {
        err = cudaFuncSetAttribute(attention_kernel<true>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (err != cudaSuccess) return err;
        attention_kernel<true><<<dim3(static_cast<unsigned>(grid)), kThreads, smem, stream>>>(
            a, tq, tk, tv, tkb, tvb);
    } else {
        err = cudaFuncSetAttribute(attention_kernel<false>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (err != cudaSuccess) return err;
        attention_kernel<false><<<dim3(static_cast<unsigned>(grid)), kThreads, smem, stream>>>(
            a, tq, tk, tv, tkb, tvb);
    }
    return cudaGetLastError();
}

}  // namespace fp2

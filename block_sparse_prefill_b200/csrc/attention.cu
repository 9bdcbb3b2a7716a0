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
//   warpgroup 0 (warps 0-3)  softmax of Q tile 0 (one thread per row = TMEM lane)
//   warpgroup 1 (warps 4-7)  softmax of Q tile 1
//   warpgroup 2: warp 8      TMA producer: Q tiles, then K/V (or mean-K/mean-V)
//                            tiles into a ring of shared-memory slots, following
//                            the kept list and, in paged mode, the block table
//                warp 9      TMEM owner and MMA issuer
//                warps 10-11 idle (they only donate registers)
// The softmax warpgroups raise their register budget (setmaxnreg) so that a
// whole 128-column row of S stays in registers; warpgroup 2 lowers its own.
//
// TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,384) O_1 [384,512); P_t is
// written over the first columns of S_t and read by the PV MMA from TMEM.
// MMA issue order per kept tile n (tcgen05.mma from one thread run in issue
// order, so S_t(n+1) may be issued right after PV_t(n), which still reads P_t
// from the same columns):
//   PV_0(n), S_0(n+1), PV_1(n), S_1(n+1)
// so the softmax of one tile overlaps the other tile's two MMAs.
// The running max is only raised when a row max exceeds it by more than a
// threshold (log2 units), so O is rarely rescaled.
// Tile order: diagonal block first (it fixes the causal mask and usually the
// row max), then the other kept blocks from nearest to farthest, then the
// correction tiles: 128 consecutive block means each, with the kept ones (and
// those >= i) masked out.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace fp2 {

namespace {

constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
// Registers per thread after the split.  setmaxnreg only redistributes the
// registers the CTA was launched with (384 threads x 168 = 64512), so
// 256 x kSoftmaxRegs + 128 x kOtherRegs must not exceed that: 53248 + 11264.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 208;
constexpr int kOtherRegs = 88;
static_assert(256 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

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

template <int kRegs>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegs));
}
template <int kRegs>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegs));
}

// S = Q_t K^T for one Q tile (kKSteps MMAs over d).
template <bool kE4M3>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {
    using C = Cfg<kE4M3>;
#pragma unroll
    for (int k = 0; k < C::kKSteps; ++k) {
        if (kE4M3)
            mma_f8_ss(d_tmem, kmajor_desc<true>(q_addr, k), kmajor_desc<true>(k_addr, k), C::kIdescQK,
                      k > 0);
        else
            mma_bf16_ss(d_tmem, kmajor_desc<false>(q_addr, k), kmajor_desc<false>(k_addr, k),
                        C::kIdescQK, k > 0);
    }
}

// O += P V for one Q tile (P from TMEM, kKSteps MMAs over the 128 keys).
template <bool kE4M3>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_addr,
                                         bool first) {
    using C = Cfg<kE4M3>;
#pragma unroll
    for (int k = 0; k < C::kKSteps; ++k) {
        const uint32_t acc = (!first || k > 0) ? 1u : 0u;
        if (kE4M3)
            mma_f8_ts(o_tmem, p_tmem + 8 * k, vmajor_desc<true>(v_addr, k), C::kIdescPV, acc);
        else
            mma_bf16_ts(o_tmem, p_tmem + 8 * k, vmajor_desc<false>(v_addr, k), C::kIdescPV, acc);
    }
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
    if (warp >= 8) {
      regs_dec<kOtherRegs>();
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
            // tile n: K in ring entry 2n, V in ring entry 2n + 1
            auto slot = [](int32_t idx) { return idx % C::kSlots; };
            auto phase = [](int32_t idx) { return static_cast<uint32_t>((idx / C::kSlots) & 1); };
            bool ok = mbar_wait(&bars.q_full, 0, hdr, abort, 300000) &&
                      mbar_wait(&bars.kv_full[slot(0)], phase(0), hdr, abort, 301000);
            if (ok) {
                tc_fence_after();
                for (int qt = 0; qt < ntiles; ++qt) {
                    issue_qk<kE4M3>(tmem + qt * 128, q_addr + qt * C::kTileBytes,
                                    kv_addr + slot(0) * C::kTileBytes);
                    mma_commit(&bars.s_full[qt]);
                }
                mma_commit(&bars.kv_empty[slot(0)]);
            }
            for (int32_t n = 0; ok && n < ntot; ++n) {
                const int32_t iv = 2 * n + 1, ik = 2 * n + 2;
                const bool next = n + 1 < ntot;
                if (!(ok = mbar_wait(&bars.kv_full[slot(iv)], phase(iv), hdr, abort, 330000 + n)))
                    break;
                if (n == 0 && nrows < kBlock &&
                    !(ok = mbar_wait(&bars.v_tail, 0, hdr, abort, 335000)))
                    break;
                for (int qt = 0; qt < ntiles && ok; ++qt) {
                    if (!(ok = mbar_wait(&bars.p_full[qt], n & 1, hdr, abort, 340000 + n))) break;
                    tc_fence_after();
                    issue_pv<kE4M3>(tmem + 256 + qt * 128, tmem + qt * 128,
                                    kv_addr + slot(iv) * C::kTileBytes, n == 0);
                    mma_commit(&bars.o_done[qt]);
                    if (next) {
                        if (qt == 0 && !(ok = mbar_wait(&bars.kv_full[slot(ik)], phase(ik), hdr,
                                                        abort, 310000 + n)))
                            break;
                        tc_fence_after();
                        issue_qk<kE4M3>(tmem + qt * 128, q_addr + qt * C::kTileBytes,
                                        kv_addr + slot(ik) * C::kTileBytes);
                        mma_commit(&bars.s_full[qt]);
                    }
                }
                if (!ok) break;
                if (next) mma_commit(&bars.kv_empty[slot(ik)]);
                mma_commit(&bars.kv_empty[slot(iv)]);
            }
        }
      }
    } else if (regs_inc<kSoftmaxRegs>(), warp / 4 < ntiles) {
        // ---- softmax + epilogue of Q tile qt ---------------------------------
        const int qt = warp / 4;
        const int32_t r = tid & 127;
        const int32_t h = h0 + qt;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + qt * 128;
        const uint32_t o_addr = tmem + lane_off + 256 + qt * 128;
        float qk = a.scale_log2;
        if (kE4M3) qk *= a.q_scale[h] * a.k_scale[g];
        // correction tiles: +log2(128) after scaling == +7/qk before it
        const float corr_bias = 7.f / qk;
        float m_ref = -INFINITY;
        float l = 0.f;      // row sum of the weights the PV MMA uses (O normaliser)
        float l_lse = 0.f;  // row sum before P is rounded to the MMA precision (LSE)
        bool ok = true;
        for (int32_t n = 0; n < ntot; ++n) {
            if (!(ok = warp_wait(&bars.s_full[qt], n & 1, hdr, abort, 400000 + n))) break;
            tc_fence_after();
            uint32_t sv[128];
            tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
            tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
            tmem_wait_ld();
            // masks (warp-uniform branch per tile kind):
            //   diagonal block (n == 0): keys c <= r
            //   kept block: every key
            //   correction tile: pruned block means only, weighted by 128
            if (n == 0) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c > r) sv[c] = __float_as_uint(-INFINITY);
            } else if (n >= cnt) {
                const int32_t w0 = ctiles[n - cnt] * 4;
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const uint32_t bits = (w0 + wi < nwords) ? pruned[w0 + wi] : 0u;
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        sv[wi * 32 + c] =
                            ((bits >> c) & 1u)
                                ? __float_as_uint(__uint_as_float(sv[wi * 32 + c]) + corr_bias)
                                : __float_as_uint(-INFINITY);
                }
            }
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sv[c]));
            const float m_new = fmaxf(m_ref, mx * qk);
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
            // P = exp2(s * qk - m + offset) in the MMA precision, written over S
            const float neg = C::kPOffset - ((m_ref == -INFINITY) ? 0.f : m_ref);
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                const float p = ex2(fmaf(__uint_as_float(sv[c]), qk, neg));
                sv[c] = __float_as_uint(p);
                rs += p;
            }
            l_lse += rs;
            if (kE4M3) {
                // the O normaliser sums the quantised weights the PV MMA sees
                __half2 hs = __float2half2_rn(0.f);
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const uint32_t pk =
                        pack_e4m3x4(__uint_as_float(sv[4 * c]), __uint_as_float(sv[4 * c + 1]),
                                    __uint_as_float(sv[4 * c + 2]), __uint_as_float(sv[4 * c + 3]));
                    hs = __hadd2(hs, e4m3x4_sum2(pk));
                    sv[c] = pk;
                }
                const float2 hf = __half22float2(hs);
                l += hf.x + hf.y;
                tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            } else {
                l += rs;
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    sv[c] = pack_bf16(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]));
                tmem_st32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                tmem_st32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            }
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
    // the setmaxnreg split assumes the kernel was built with kLaunchRegs per
    // thread; with fewer, the softmax warps' register request could never be met
    cudaFuncAttributes fa;
    cudaError_t err = e4m3 ? cudaFuncGetAttributes(&fa, attention_kernel<true>)
                           : cudaFuncGetAttributes(&fa, attention_kernel<false>);
    if (err != cudaSuccess) return err;
    if (fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
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

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
// With correction 2 each pruned block's lbar_j also gets (tau^2 / 2) |q_r|^2 kvar_j,
// kvar_j its key variance averaged over the dimensions.  Chunked prefill: the
// q-blocks keep the request's absolute grid, so only the Q tile's row offset and
// the rows the epilogue stores change.
//
// Structure: persistent, one CTA per SM.  A work item is one q-block x two query
// heads of one KV head, so every K/V tile fetched into shared memory serves both
// heads; the CTA takes items from a counter in the workspace, in the order the
// setup kernel wrote: most tiles first.
//   warpgroup 0 (warps 0-3)  softmax of Q tile 0 (one thread per row = TMEM lane)
//   warpgroup 1 (warps 4-7)  softmax of Q tile 1
//   warpgroup 2: warp 8      TMA producer: Q tiles, then K/V (or mean-K/mean-V)
//                            tiles into a ring of shared-memory slots, at the rows
//                            the scheduler prepared
//                warp 9      TMEM owner and MMA issuer
//                warp 10     scheduler: takes work items from a global counter and
//                            prepares them in shared memory: the kept list as K/V
//                            rows (pages of the pool, through the block table, in
//                            paged mode), the pruned blocks, the correction tiles
//                warp 11     idle (it only donates registers)
// The softmax warpgroups raise their register budget (setmaxnreg) so that a
// whole 128-column row of S stays in registers; warpgroup 2 lowers its own.
//
// TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,384) O_1 [384,512); P_t is
// written over the first columns of S_t and read by the PV MMA from TMEM.
// MMA issue order per kept tile n (tcgen05.mma from one thread run in issue
// order, so S_t(n+1) may be issued right after PV_t(n), which still reads P_t
// from the same columns):
//   PV_0(n), S_0(n+1), PV_1(n), S_1(n+1)
// so the softmax of one tile overlaps the other tile's two MMAs.  Three commits
// per step (each costs tensor-pipe time): S_0 ready, S_1 ready, and one event
// that frees the step's K/V ring entries.
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
constexpr int kSchedWarp = 10;
constexpr uint32_t kTmemCols = 512;
// Registers per thread after the split.  setmaxnreg only redistributes the
// registers the CTA was launched with (384 threads x 168 = 64512), so
// 256 x kSoftmaxRegs + 128 x kOtherRegs must not exceed that: 55296 + 9216.
// With 216 the softmax keeps a whole row of S without spilling (208 spilled);
// the producer, issuer and scheduler fit in 72.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
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
    uint64_t q_empty;     // the last S MMAs of a work item have read Q (committed right
                          // after them, so the next item's Q loads during the item's
                          // last tile step)
    uint64_t q_read;      // correction 2: the softmax warps have read |q_r|^2 off the Q
                          // tile (one arrival per softmax warp and item)
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_done[2];   // the last PV of Q tile t in a work item has finished
    uint64_t kv_full[8];
    uint64_t ev[8];       // slot-release events: the issuer commits one after the S MMAs
                          // of an item's first step and one at the end of every step; a
                          // commit tracks every earlier MMA, so event E + j of an item
                          // whose first event is E frees its ring entries base .. base + 2j
                          // (all of them for j = ntot).  A ring of kSlots barriers: no
                          // event can run kSlots ahead of the producer's wait for it.
    uint64_t v_tail[2];   // per metadata buffer: V rows past the request end zeroed
                          // (partial diagonal block); per buffer so that a waiter can
                          // never be two phases behind
    uint64_t meta_full[2];
    uint64_t meta_empty[2];
    uint64_t never;       // completed by nothing (the timeout test hook waits on it)
};

struct SmemMisc {
    Bars bars;
    uint32_t tmem_base;
    int32_t abort;
    int32_t rel_ev[8];    // event that frees each ring slot's current entry (producer only)
};

// One work item (a q-block x up to two query heads of one KV head), prepared
// by the scheduler warp into one of two shared-memory buffers.  The kept list
// (as the first K/V row of each kept block, ascending), the pruned-block bitmask
// and the correction tile list follow the header.
struct ItemMeta {
    int32_t stop;     // 1: no work left
    int32_t t, b, i, g, h0, ntiles;
    int32_t nkeys;    // keys of the diagonal block (< 128: the V rows past them are zeroed)
    int32_t r_lo, r_hi;  // rows [r_lo, r_hi) of the Q tile are query rows (stored)
    int32_t qrow0;    // row of q / out of the tile's row 0 (rows outside [r_lo, r_hi)
                      // belong to another request, or lie before row 0: never stored)
    int32_t cb, cnt, ncorr, nwords;
    int32_t pad[1];
};

template <bool kE4M3>
__host__ __device__ constexpr size_t tiles_bytes() {
    return static_cast<size_t>(2 + Cfg<kE4M3>::kSlots) * Cfg<kE4M3>::kTileBytes;
}

// End of the operand tiles and SmemMisc, rounded up to 16 bytes: where the two
// metadata buffers begin.
template <bool kE4M3>
__host__ __device__ constexpr size_t misc_end() {
    return (tiles_bytes<kE4M3>() + sizeof(SmemMisc) + 15) & ~size_t(15);
}

// One metadata buffer: header, kept list, pruned bitmask, correction tile list
// and (correction 2) the variance coefficient of every column of the correction
// tiles (16-byte aligned, after the lists).
__host__ __device__ inline size_t meta_lists_bytes(int32_t nb_cap) {
    const size_t b = sizeof(ItemMeta) +
                     sizeof(int32_t) * (nb_cap + (nb_cap + 31) / 32 + (nb_cap + 127) / 128 + 4);
    return (b + 15) & ~size_t(15);
}
__host__ __device__ inline size_t meta_bytes(int32_t nb_cap, bool var) {
    return meta_lists_bytes(nb_cap) + (var ? sizeof(float) * 128 * ((nb_cap + 127) / 128) : 0);
}

// Byte offset of K-major operand step k inside a tile (Q or K).
template <bool kE4M3>
__device__ __forceinline__ constexpr uint32_t kmajor_off(int k) {
    return kE4M3 ? k * 32 : (k >> 2) * 16384 + (k & 3) * 32;
}

// The value itself, opaque to the compiler: keeps a descriptor from being
// hoisted (with its per-step variants) out of the issuer's loops, which under
// the issuer's register budget would spill.
__device__ __forceinline__ uint64_t opaque64(uint64_t x) {
    asm volatile("mov.b64 %0, %0;" : "+l"(x));
    return x;
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
    // step k's descriptors = step 0's + (offset >> 4) in the start-address field
    // (no carry out of it: shared-memory addresses are below 256 KB)
    const uint64_t qa = opaque64(sdesc_sw128(q_addr, 16, 1024));
    const uint64_t kb = sdesc_sw128(k_addr, 16, 1024);
#pragma unroll
    for (int k = 0; k < C::kKSteps; ++k) {
        const uint64_t off = kmajor_off<kE4M3>(k) >> 4;
        if (kE4M3)
            mma_f8_ss(d_tmem, qa + off, kb + off, C::kIdescQK, k > 0);
        else
            mma_bf16_ss(d_tmem, qa + off, kb + off, C::kIdescQK, k > 0);
    }
}

// O += P V for one Q tile (P from TMEM, kKSteps MMAs over the 128 keys).
template <bool kE4M3>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_addr,
                                         bool first) {
    using C = Cfg<kE4M3>;
    const uint64_t vb = sdesc_sw128(v_addr, 16384, 1024);
#pragma unroll
    for (int k = 0; k < C::kKSteps; ++k) {
        const uint32_t acc = (!first || k > 0) ? 1u : 0u;
        const uint64_t off = (k * (kE4M3 ? 4096u : 2048u)) >> 4;  // keys [k*K, (k+1)*K)
        if (kE4M3)
            mma_f8_ts(o_tmem, p_tmem + 8 * k, vb + off, C::kIdescPV, acc);
        else
            mma_bf16_ts(o_tmem, p_tmem + 8 * k, vb + off, C::kIdescPV, acc);
    }
}

}  // namespace

// kVar: correction 2 (the variance term), a separate instantiation so that the
// other corrections keep their own register allocation.
template <bool kE4M3, bool kVar>
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
    // metadata buffers start 16-byte aligned (correction 2 reads them as float4)
    uint8_t* meta_base = smem + misc_end<kE4M3>();
    constexpr bool var = kVar;
    const size_t meta_stride = meta_bytes(a.nb_cap, var);
    Bars& bars = misc->bars;
    volatile int32_t* abort = &misc->abort;
    WsHeader* hdr = a.hdr;
    if (!hdr->valid) return;

    const int32_t tid = threadIdx.x;
    const int32_t warp = tid >> 5;
    const int32_t lane = tid & 31;

    auto meta = [&](int32_t buf) { return reinterpret_cast<ItemMeta*>(meta_base + buf * meta_stride); };
    auto klist_of = [](ItemMeta* m) { return reinterpret_cast<int32_t*>(m + 1); };
    auto pruned_of = [&](ItemMeta* m) { return reinterpret_cast<uint32_t*>(klist_of(m) + a.nb_cap); };
    auto ctiles_of = [&](ItemMeta* m) {
        return reinterpret_cast<int32_t*>(pruned_of(m) + (a.nb_cap + 31) / 32);
    };
    auto cvals_of = [&](ItemMeta* m) {
        return reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(m) + meta_lists_bytes(a.nb_cap));
    };

    // ---- set-up ------------------------------------------------------------
    if (warp == kMmaWarp) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bars.q_full, 1);
        mbar_init(&bars.q_empty, 1);
        mbar_init(&bars.q_read, 8);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars.s_full[s], 1);
            mbar_init(&bars.p_full[s], 128);
            mbar_init(&bars.o_done[s], 1);
            mbar_init(&bars.meta_full[s], 1);
            mbar_init(&bars.meta_empty[s], 10);  // producer, MMA issuer, 8 softmax warps
        }
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(&bars.kv_full[s], 1);
            mbar_init(&bars.ev[s], 1);
        }
        mbar_init(&bars.never, 1);
        mbar_init(&bars.v_tail[0], 1);
        mbar_init(&bars.v_tail[1], 1);
        misc->abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp >= 8) {
      regs_dec<kOtherRegs>();
      if (warp == kSchedWarp) {
        // ---- scheduler: next work item -> metadata buffer ----------------
        const int32_t n_items = hdr->total_qblocks * a.hkv * a.pairs;
        for (int32_t k = 0;; ++k) {
            const int32_t buf = k & 1;
            if (!warp_wait(&bars.meta_empty[buf], ((k >> 1) & 1) ^ 1, hdr, abort, 500000 + k)) break;
            ItemMeta* m = meta(buf);
            int32_t item = 0;
            if (lane == 0) item = atomicAdd(&hdr->work_next, 1);
            item = __shfl_sync(0xffffffffu, item, 0);
            if (item >= n_items) {
                if (lane == 0) {
                    m->stop = 1;
                    mbar_arrive(&bars.meta_full[buf]);
                }
                break;
            }
            const int32_t code = a.order[item / a.pairs];   // t * hkv + g, heaviest first
            const int32_t t = code / a.hkv;
            const int32_t g = code % a.hkv;
            const int32_t hp = item % a.pairs;
            const int32_t b = a.blk_req_q[t];
            const int32_t cb = a.cu_blocks[b];
            const ReqSpan span = req_span(a.cu_q, a.cu_k, b);
            const int32_t i = span.i0 + t - a.cu_qblocks[b];   // absolute block index
            int32_t* klist = klist_of(m);
            uint32_t* pruned = pruned_of(m);
            int32_t* ctiles = ctiles_of(m);
            // kept list of (q-block t, KV head g), checked: ascending, in [0, i], ends at i
            const int64_t lrow = static_cast<int64_t>(t) * a.hkv + g;
            int32_t cnt = a.kept_cnt[lrow];
            bool good = cnt >= 1 && cnt <= i + 1;
            const int32_t* src = a.kept_idx + lrow * a.nb_max;
            if (good)
                for (int32_t e = lane; e < cnt; e += 32) klist[e] = src[e];
            __syncwarp();
            if (good) {
                bool bad = false;
                for (int32_t e = lane; e < cnt; e += 32)
                    bad |= klist[e] < 0 || klist[e] > i || (e > 0 && klist[e] <= klist[e - 1]);
                good = !__any_sync(0xffffffffu, bad) && klist[cnt - 1] == i;
            }
            if (!good) {
                if (lane == 0) set_error(hdr, FP2_ERR_BAD_INDEX, t);
                cnt = 1;
                __syncwarp();
                if (lane == 0) klist[0] = i;
            }
            // pruned blocks j < i (bit set) and the correction tiles holding any
            const int32_t nwords = (i + 31) / 32;
            for (int32_t w = lane; w < nwords; w += 32) {
                const int32_t nbits = min(32, i - w * 32);
                pruned[w] = (nbits == 32) ? 0xffffffffu : ((1u << nbits) - 1u);
            }
            __syncwarp();
            for (int32_t e = lane; e < cnt - 1; e += 32) {
                const int32_t j = klist[e];
                atomicAnd(&pruned[j >> 5], ~(1u << (j & 31)));
            }
            __syncwarp();
            int32_t nc = 0;
            if (a.correction) {
                const int32_t nct = (i + 127) / 128;
                for (int32_t c0 = 0; c0 < nct; c0 += 32) {
                    const int32_t ct = c0 + lane;
                    uint32_t any = 0;
                    if (ct < nct)
                        for (int32_t w = ct * 4; w < min(ct * 4 + 4, nwords); ++w) any |= pruned[w];
                    const uint32_t mask = __ballot_sync(0xffffffffu, any != 0);
                    if (any) ctiles[nc + __popc(mask & ((1u << lane) - 1u))] = ct;
                    nc += __popc(mask);
                }
            }
            if (var) {
                // correction 2: tau^2 / 2 log2(e) kvar_j of every column of the
                // correction tiles (0 where the column is masked)
                float* cv = cvals_of(m);
                for (int32_t e = 0; e < nc; ++e) {
                    const int32_t j0 = ctiles[e] * 128;
                    for (int32_t c = lane; c < 128; c += 32) {
                        const int32_t j = j0 + c;
                        const bool pr = j < i && ((pruned[j >> 5] >> (j & 31)) & 1u);
                        cv[e * 128 + c] =
                            pr ? a.var_coef * a.k_var[static_cast<int64_t>(cb + j) * a.hkv + g] : 0.f;
                    }
                }
            }
            // kept blocks -> the first K/V row of each (a page of the pool, or the
            // request's rows), so the producer's per-tile work is one shared-memory read
            for (int32_t e = lane; e < cnt; e += 32) {
                const int32_t j = klist[e];
                int32_t row;
                if (a.block_table) {
                    int32_t page = a.block_table[static_cast<int64_t>(b) * a.max_blocks_per_seq + j];
                    if (page < 0 || page >= a.num_pages) {
                        set_error(hdr, FP2_ERR_BAD_INDEX, t);
                        page = 0;
                    }
                    row = page * kBlock;
                } else {
                    row = a.cu_k[b] + j * kBlock;
                }
                klist[e] = row;
            }
            __syncwarp();
            if (lane == 0) {
                m->stop = 0;
                m->t = t;
                m->b = b;
                m->i = i;
                m->g = g;
                m->h0 = g * a.G + 2 * hp;
                m->ntiles = min(2, a.G - 2 * hp);
                m->nkeys = min(kBlock, span.lk - i * kBlock);
                m->r_lo = max(0, span.p - i * kBlock);
                m->r_hi = m->nkeys;
                m->qrow0 = a.cu_q[b] + i * kBlock - span.p;
                m->cb = cb;
                m->cnt = cnt;
                m->ncorr = nc;
                m->nwords = nwords;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.meta_full[buf]);
        }
      } else if (warp == kProducerWarp) {
        // ---- TMA producer ----------------------------------------------------
        // lane 0 issues every TMA; the whole warp zeroes the V rows past the
        // request end of a partial diagonal block (a paged pool may hold
        // anything there, and zero attention weights times NaN is NaN)
        const bool leader = lane == 0;
        if (leader) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
        }
        int32_t issued = 0;   // K/V ring entries issued so far
        int32_t nq = 0;       // Q loads issued so far
        int32_t ev_item = 0;  // first release event of the current item
        for (int32_t k = 0; !*abort; ++k) {
            const int32_t buf = k & 1;
            if (!warp_wait(&bars.meta_full[buf], (k >> 1) & 1, hdr, abort, 510000 + k)) break;
            ItemMeta* m = meta(buf);
            if (m->stop) break;
            const int32_t ntiles = m->ntiles, cnt = m->cnt, ntot = m->cnt + m->ncorr;
            const int32_t nrows = m->nkeys, g = m->g, cb = m->cb;
            const int32_t* klist = klist_of(m);
            const int32_t* ctiles = ctiles_of(m);
            const int32_t item_base = issued;
            bool ok = true;
            for (int32_t n = 0; ok && n < ntot; ++n) {
                if (n == 1 || (n == 0 && ntot == 1)) {
                    // Q after the first K/V pair: those loads are already in flight
                    // while the previous item's last MMAs still read the Q buffer
                    if (leader) {
                        if (k > 0) ok = mbar_wait(&bars.q_empty, (k - 1) & 1, hdr, abort, 520000 + k);
                        if (ok && var && k > 0)
                            ok = mbar_wait(&bars.q_read, (k - 1) & 1, hdr, abort, 525000 + k);
                        if (ok) {
                            ++nq;
                            mbar_arrive_expect_tx(&bars.q_full, ntiles * C::kTileBytes);
                            for (int qt = 0; qt < ntiles; ++qt)
                                for (int ch = 0; ch < C::kChunks; ++ch)
                                    tma_load_3d(q_s + qt * C::kTileBytes + ch * 16384, &tq,
                                                &bars.q_full, ch * 64, m->h0 + qt, m->qrow0);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) break;
                }
                const CUtensorMap* mk;
                const CUtensorMap* mv;
                int32_t row = 0;
                if (n < cnt) {
                    row = klist[cnt - 1 - n];  // nearest kept block first (the diagonal)
                    mk = &tk;
                    mv = &tv;
                } else {
                    mk = &tkb;
                    mv = &tvb;
                    row = cb + ctiles[n - cnt] * 128;
                }
                for (int kv = 0; kv < 2 && ok; ++kv) {
                    const int32_t idx = issued;
                    const int32_t s = idx % C::kSlots;
                    if (leader) {
                        if (idx >= C::kSlots) {
                            const int32_t e = misc->rel_ev[s];
                            ok = mbar_wait(&bars.ev[e % C::kSlots], static_cast<uint32_t>((e / C::kSlots) & 1),
                                           hdr, abort, 100000 + n);
                        }
                        if (ok) {
                            // entry idx is freed by event ev_item + ceil((idx - base) / 2)
                            misc->rel_ev[s] = ev_item + (idx - item_base + 1) / 2;
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
                        if (leader) mbar_arrive(&bars.v_tail[buf]);
                    }
                }
            }
            __syncwarp();
            if (leader) mbar_arrive(&bars.meta_empty[buf]);
            if (!ok) break;
            ev_item += ntot + 1;
        }
        // drain: every issued tile has been consumed and released (the last item's
        // last event); after an abort, at least every issued copy has landed
        if (leader) {
            bool drained = true;
            if (ev_item > 0)
                drained = mbar_wait(&bars.ev[(ev_item - 1) % C::kSlots],
                                    static_cast<uint32_t>(((ev_item - 1) / C::kSlots) & 1), hdr, abort, 200000);
            if (!drained) {
                for (int32_t idx = max(0, issued - C::kSlots); idx < issued; ++idx)
                    mbar_wait_drain(&bars.kv_full[idx % C::kSlots], (idx / C::kSlots) & 1);
                if (nq > 0) mbar_wait_drain(&bars.q_full, (nq - 1) & 1);
            }
        }
      } else if (warp == kMmaWarp) {
        // ---- MMA issuer ------------------------------------------------------
        if (lane == 0) {
            const uint32_t q_addr = smem_u32(q_s);
            const uint32_t kv_addr = smem_u32(kv_s);
            auto slot = [](int32_t idx) { return idx % C::kSlots; };
            auto phase = [](int32_t idx) { return static_cast<uint32_t>((idx / C::kSlots) & 1); };
            int32_t base = 0;          // ring entry of the current item's first K tile
            int32_t ev_item = 0;       // first release event of the current item
            int32_t it[2] = {0, 0};    // PV iterations issued per Q tile
            int32_t vt[2] = {0, 0};    // partial items seen per metadata buffer
            bool ok = true;
            for (int32_t k = 0; ok; ++k) {
                const int32_t buf = k & 1;
                if (!(ok = mbar_wait(&bars.meta_full[buf], (k >> 1) & 1, hdr, abort, 530000 + k))) break;
                ItemMeta* m = meta(buf);
                if (m->stop) break;
                const int32_t ntiles = m->ntiles, ntot = m->cnt + m->ncorr;
                const bool partial = m->nkeys < kBlock;
                if (a.test_wait_timeout && k == 0 &&
                    !(ok = mbar_wait(&bars.never, 0, hdr, abort, 900000)))
                    break;
                ok = mbar_wait(&bars.q_full, k & 1, hdr, abort, 300000) &&
                     mbar_wait(&bars.kv_full[slot(base)], phase(base), hdr, abort, 301000);
                if (!ok) break;
                tc_fence_after();
                for (int qt = 0; qt < ntiles; ++qt) {
                    issue_qk<kE4M3>(tmem + qt * 128, q_addr + qt * C::kTileBytes,
                                    kv_addr + slot(base) * C::kTileBytes);
                    mma_commit(&bars.s_full[qt]);
                }
                mma_commit(&bars.ev[ev_item % C::kSlots]);  // frees K_0
                if (ntot == 1) mma_commit(&bars.q_empty);
                for (int32_t n = 0; ok && n < ntot; ++n) {
                    const int32_t iv = base + 2 * n + 1, ik = base + 2 * n + 2;
                    const bool next = n + 1 < ntot;
                    if (!(ok = mbar_wait(&bars.kv_full[slot(iv)], phase(iv), hdr, abort, 330000 + n)))
                        break;
                    if (n == 0 && partial) {
                        if (!(ok = mbar_wait(&bars.v_tail[buf], vt[buf] & 1, hdr, abort, 335000))) break;
                        ++vt[buf];
                    }
                    for (int qt = 0; qt < ntiles && ok; ++qt) {
                        if (!(ok = mbar_wait(&bars.p_full[qt], it[qt] & 1, hdr, abort, 340000 + n))) break;
                        ++it[qt];
                        tc_fence_after();
                        issue_pv<kE4M3>(tmem + 256 + qt * 128, tmem + qt * 128,
                                        kv_addr + slot(iv) * C::kTileBytes, n == 0);
                        // O_t is complete after the item's last PV.  Within the
                        // item no O-done signal is needed: S_t(n+1) is issued after
                        // PV_t(n), and a commit tracks every earlier MMA, so the
                        // softmax's S-ready wait also covers PV_t(n).  (Each commit
                        // costs tensor-pipe time.)
                        if (!next) mma_commit(&bars.o_done[qt]);
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
                    if (n + 2 == ntot) mma_commit(&bars.q_empty);  // S_t(ntot-1) were the last
                    mma_commit(&bars.ev[(ev_item + n + 1) % C::kSlots]);  // frees V_n, K_(n+1)
                }
                base += 2 * ntot;
                ev_item += ntot + 1;
                mbar_arrive(&bars.meta_empty[buf]);
            }
        }
      }
    } else {
        regs_inc<kSoftmaxRegs>();
        // ---- softmax + epilogue of Q tile qt ---------------------------------
        const int qt = warp / 4;
        const int32_t r = tid & 127;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + qt * 128;
        const uint32_t o_addr = tmem + lane_off + 256 + qt * 128;
        int32_t it = 0;     // tile steps of this Q tile so far (s_full phases)
        int32_t items = 0;  // work items of this Q tile so far (o_done phases)
        bool ok = true;
        for (int32_t k = 0; ok; ++k) {
            const int32_t buf = k & 1;
            if (!(ok = warp_wait(&bars.meta_full[buf], (k >> 1) & 1, hdr, abort, 540000 + k))) break;
            ItemMeta* m = meta(buf);
            if (m->stop) break;
            if (qt >= m->ntiles) {
                __syncwarp();
                if (lane == 0) {
                    if (var) mbar_arrive(&bars.q_read);
                    mbar_arrive(&bars.meta_empty[buf]);
                }
                continue;
            }
            const int32_t cnt = m->cnt, ntot = m->cnt + m->ncorr, nwords = m->nwords;
            float qk = a.scale_log2;
            // e4m3: a zero scale (an all-zero head) makes every logit 0; the floor keeps
            // masked (-inf) scores at -inf instead of -inf * 0 = NaN
            if (kE4M3) qk = fmaxf(qk * a.q_scale[m->h0 + qt] * a.k_scale[m->g], 1.17549435e-38f);
            // correction 2: w = |q_r|^2 (dequantised), read off the Q tile, whose 16-byte
            // units of row r sit in the 128-byte swizzle order (the sum does not care)
            float w = 0.f;
            if (var) {
                if (!(ok = warp_wait(&bars.q_full, k & 1, hdr, abort, 405000))) break;
                const uint8_t* qrow = q_s + qt * C::kTileBytes + r * 128;
#pragma unroll
                for (int ch = 0; ch < C::kChunks; ++ch)
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint4 x4 = *reinterpret_cast<const uint4*>(qrow + ch * 16384 + u * 16);
                        const uint32_t wd[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            if (kE4M3) {
                                const float2 lo = __half22float2(e4m3x2_to_half2(wd[e] & 0xFFFFu));
                                const float2 hi = __half22float2(e4m3x2_to_half2(wd[e] >> 16));
                                w = fmaf(lo.x, lo.x, fmaf(lo.y, lo.y, fmaf(hi.x, hi.x, fmaf(hi.y, hi.y, w))));
                            } else {
                                const float a0 = __uint_as_float(wd[e] << 16);
                                const float a1 = __uint_as_float(wd[e] & 0xFFFF0000u);
                                w = fmaf(a0, a0, fmaf(a1, a1, w));
                            }
                        }
                    }
                if (kE4M3) {
                    const float qs = a.q_scale[m->h0 + qt];
                    w *= qs * qs;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars.q_read);
            }
            float m_ref = -INFINITY;
            float l = 0.f;      // row sum of the weights the PV MMA uses (O normaliser)
            float l_lse = 0.f;  // row sum before P is rounded to the MMA precision (LSE)
            for (int32_t n = 0; n < ntot; ++n) {
                if (!(ok = warp_wait(&bars.s_full[qt], it & 1, hdr, abort, 400000 + n))) break;
                tc_fence_after();
                uint32_t sv[128];
                tmem_ld128(s_addr, sv);
                tmem_wait_ld();
                // masks (warp-uniform branch per tile kind):
                //   diagonal block (n == 0): keys c <= r
                //   kept block: every key
                //   correction tile: pruned block means only, weighted by 128
                if (n == 0 && kE4M3) {
                    // warp w % 4 holds rows [32 (w % 4), 32 (w % 4) + 32): only that
                    // column block needs a per-element test; the blocks right of it are
                    // masked whole, those left of it not at all (uniform branches).
                    // Measured at 128K: e4m3 1.8% faster than the per-element form
                    // below, bf16 1% slower, so bf16 keeps that one.
                    const int wq = warp & 3;
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        if (cb == wq) {
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (32 * cb + c > r) sv[32 * cb + c] = __float_as_uint(-INFINITY);
                        } else if (cb > wq) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) sv[32 * cb + c] = __float_as_uint(-INFINITY);
                        }
                    }
                } else if (n == 0) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c > r) sv[c] = __float_as_uint(-INFINITY);
                } else if (n >= cnt) {
                    // (lists re-read from the metadata buffer: fewer live registers)
                    const uint32_t* pruned = pruned_of(m);
                    const int32_t w0 = ctiles_of(m)[n - cnt] * 4;
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi) {
                        const uint32_t bits = (w0 + wi < nwords) ? pruned[w0 + wi] : 0u;
                        // (the same word for the whole warp: most words of a correction
                        // tile are all pruned, and those need no per-column test)
                        if (bits != 0xffffffffu) {
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                if (!((bits >> c) & 1u)) sv[wi * 32 + c] = __float_as_uint(-INFINITY);
                        }
                    }
                }
                // a correction column stands for the 128 keys of a pruned block: its
                // weight is 128 e^{lbar}, i.e. +log2(128) on the scaled logit
                const float bias = (n >= cnt) ? 7.f : 0.f;
                // correction 2: the scaled logit of a correction column gets + w coef_j,
                // i.e. the raw score gets + (w / qk) coef_j (one packed FMA per pair)
                const float sc = qk;
                if (var && n >= cnt) {
                    const float4* cv = reinterpret_cast<const float4*>(cvals_of(m) + (n - cnt) * 128);
                    const float wq = w / qk;
#pragma unroll
                    for (int c4 = 0; c4 < 32; ++c4) {
                        const float4 cc = cv[c4];
                        const float2 lo = ffma2(make_float2(wq, wq), make_float2(cc.x, cc.y),
                                                make_float2(__uint_as_float(sv[4 * c4]), __uint_as_float(sv[4 * c4 + 1])));
                        const float2 hi = ffma2(make_float2(wq, wq), make_float2(cc.z, cc.w),
                                                make_float2(__uint_as_float(sv[4 * c4 + 2]), __uint_as_float(sv[4 * c4 + 3])));
                        sv[4 * c4] = __float_as_uint(lo.x);
                        sv[4 * c4 + 1] = __float_as_uint(lo.y);
                        sv[4 * c4 + 2] = __float_as_uint(hi.x);
                        sv[4 * c4 + 3] = __float_as_uint(hi.y);
                    }
                }
                // row max over 4 independent 3-input max chains
                float mxp[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) mxp[j] = -INFINITY;
#pragma unroll
                for (int c = 0; c < 128; c += 2)
                    mxp[(c >> 1) & 3] =
                        fmax3(mxp[(c >> 1) & 3], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
                const float mx = fmax3(mxp[0], mxp[1], fmaxf(mxp[2], mxp[3]));
                const float m_new = fmaxf(m_ref, fmaf(mx, sc, bias));
                const bool need = m_new > m_ref + C::kRescale;
                if (__any_sync(0xffffffffu, need)) {
                    const float f = need ? ex2(m_ref - m_new) : 1.f;
                    if (n > 0) {
                        // PV_t(n-1) has finished: S_t(n) was issued after it
#pragma unroll
                        for (int c0 = 0; c0 < 128; c0 += 32) {
                            uint32_t ov[32];
                            tmem_ld32(o_addr + c0, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                ov[c] = __float_as_uint(__uint_as_float(ov[c]) * f);
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
                const float neg = C::kPOffset + bias - ((m_ref == -INFINITY) ? 0.f : m_ref);
                // exp2 of packed pairs (MUFU), in two halves of 64 keys: the first
                // half's P goes to TMEM (asynchronously) while the second half is computed
                float2 rsp[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) rsp[j] = make_float2(0.f, 0.f);
                __half2 hs[4];  // e4m3: sums of the quantised weights
#pragma unroll
                for (int j = 0; j < 4; ++j) hs[j] = __float2half2_rn(0.f);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                    for (int c = 64 * hf; c < 64 * hf + 64; c += 2) {
                        float2 x = ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                         make_float2(sc, sc), make_float2(neg, neg));
                        x.x = ex2(x.x);
                        x.y = ex2(x.y);
                        sv[c] = __float_as_uint(x.x);
                        sv[c + 1] = __float_as_uint(x.y);
                        rsp[(c >> 1) & 3] = fadd2(rsp[(c >> 1) & 3], x);
                    }
                    if (kE4M3) {
                        // the O normaliser sums the quantised weights the PV MMA sees
#pragma unroll
                        for (int c = 16 * hf; c < 16 * hf + 16; ++c) {
                            const uint32_t pk = pack_e4m3x4(
                                __uint_as_float(sv[4 * c]), __uint_as_float(sv[4 * c + 1]),
                                __uint_as_float(sv[4 * c + 2]), __uint_as_float(sv[4 * c + 3]));
                            hs[c & 3] = __hadd2(hs[c & 3], e4m3x4_sum2(pk));
                            sv[c] = pk;
                        }
                        tmem_st16(s_addr + 16 * hf, &sv[16 * hf]);
                    } else {
#pragma unroll
                        for (int c = 32 * hf; c < 32 * hf + 32; ++c)
                            sv[c] = pack_bf16(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]));
                        tmem_st32(s_addr + 32 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * hf]));
                    }
                }
                const float2 rs2 = fadd2(fadd2(rsp[0], rsp[1]), fadd2(rsp[2], rsp[3]));
                const float rs = rs2.x + rs2.y;
                l_lse += rs;
                if (kE4M3) {
                    const float2 h01 = __half22float2(hs[0]), h23 = __half22float2(hs[1]);
                    const float2 h45 = __half22float2(hs[2]), h67 = __half22float2(hs[3]);
                    l += ((h01.x + h01.y) + (h23.x + h23.y)) + ((h45.x + h45.y) + (h67.x + h67.y));
                } else {
                    l += rs;
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars.p_full[qt]);
                ++it;
            }
            // ---- epilogue: O / l -> bf16 ------------------------------------
            if (ok && ntot > 0 && (ok = warp_wait(&bars.o_done[qt], (items++) & 1, hdr, abort, 420000))) {
                const int32_t g = m->g, h = m->h0 + qt, r_lo = m->r_lo, r_hi = m->r_hi, qrow0 = m->qrow0;
                const bool store = r >= r_lo && r < r_hi;
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
                    if (store) {
                        uint32_t pk[16];
#pragma unroll
                        for (int c = 0; c < 16; ++c)
                            pk[c] = pack_bf16(__uint_as_float(ov[2 * c]) * inv,
                                              __uint_as_float(ov[2 * c + 1]) * inv);
                        // each thread writes its own row: with 32-byte stores a warp's
                        // store covers whole sectors of 32 rows, half as many requests
                        // as with 16-byte ones (the epilogue is bound by those requests)
                        if (a.out_align32) {
                            st_global_v8(orow + c0, pk);
                            st_global_v8(orow + c0 + 16, pk + 8);
                        } else {
                            uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                        }
                    }
                }
                if (a.lse && store) {
                    const float m_use = ((m_ref == -INFINITY) ? 0.f : m_ref) - C::kPOffset;
                    a.lse[static_cast<int64_t>(qrow0 + r) * a.hq + h] =
                        (m_use + __log2f(l_lse)) * 0.69314718055994530942f;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.meta_empty[buf]);
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

size_t attn_smem_bytes(bool e4m3, int32_t nb_cap, bool var) {
    const size_t tiles = e4m3 ? tiles_bytes<true>() : tiles_bytes<false>();
    return 1024 + (e4m3 ? misc_end<true>() : misc_end<false>()) + 2 * meta_bytes(nb_cap, var);
}

template <bool kE4M3, bool kVar>
cudaError_t launch_one(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const CUtensorMap& tkb, const CUtensorMap& tvb,
                       unsigned grid, size_t smem, cudaStream_t stream) {
    // the setmaxnreg split assumes the kernel was built with kLaunchRegs per
    // thread; with fewer, the softmax warps' register request could never be met
    cudaFuncAttributes fa;
    cudaError_t err = cudaFuncGetAttributes(&fa, attention_kernel<kE4M3, kVar>);
    if (err != cudaSuccess) return err;
    if (fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
    err = cudaFuncSetAttribute(attention_kernel<kE4M3, kVar>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem));
    if (err != cudaSuccess) return err;
    attention_kernel<kE4M3, kVar><<<grid, kThreads, smem, stream>>>(a, tq, tk, tv, tkb, tvb);
    return cudaGetLastError();
}

cudaError_t launch_attention(bool e4m3, const AttnArgs& a, const CUtensorMap& tq,
                             const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tkb,
                             const CUtensorMap& tvb, int64_t max_blocks, cudaStream_t stream) {
    const bool var = a.correction == 2;
    const size_t smem = attn_smem_bytes(e4m3, a.nb_cap, var);
    const int64_t items = max_blocks * a.hkv * a.pairs;
    if (items <= 0) return cudaSuccess;
    // persistent: one CTA per SM, work items taken from a counter in the workspace
    int dev = 0, sms = 0;
    cudaError_t err;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return err;
    const unsigned grid = static_cast<unsigned>(items < sms ? items : sms);
    if (e4m3)
        return var ? launch_one<true, true>(a, tq, tk, tv, tkb, tvb, grid, smem, stream)
                   : launch_one<true, false>(a, tq, tk, tv, tkb, tvb, grid, smem, stream);
    return var ? launch_one<false, true>(a, tq, tk, tv, tkb, tvb, grid, smem, stream)
               : launch_one<false, false>(a, tq, tk, tv, tkb, tvb, grid, smem, stream);
}

}  // namespace fp2

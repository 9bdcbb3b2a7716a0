// common.cuh -- definitions shared by the kernels and the host entry points:
// workspace layout, device error flag, bounded mbarrier waits.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/fp2.h"
#include "sm100.cuh"

namespace fp2 {

constexpr int kHeadDim = 128;
constexpr int kBlock = 128;

// Workspace header (first 256 bytes of the caller's workspace).
struct WsHeader {
    int32_t status;         // first device-side fp2_status recorded (0 = none)
    int32_t detail;         // detail of that error (offending index, ...)
    int32_t valid;          // 1 when the last setup pass accepted cu_seqlens
    int32_t total_blocks;   // key blocks: sum_b ceil(Lk_b / block_size) of the last setup pass
    int32_t work_next;      // next work item of the persistent attention kernel
    int32_t total_qblocks;  // q-blocks: sum_b (ceil(Lk_b / bs) - floor(P_b / bs)), P_b = Lk_b - Lq_b
};

// Requests and their blocks.  Request b has Lk keys; its queries are its last
// Lq <= Lk tokens, at positions P = Lk - Lq .. Lk - 1 (plain prefill: Lq = Lk,
// P = 0).  Key blocks j = 0 .. ceil(Lk / bs) - 1 cover positions [bs j, bs j + bs);
// q-blocks keep the same absolute grid, so the request's q-blocks are the
// blocks i = floor(P / bs) .. ceil(Lk / bs) - 1 (none when Lq = 0), the first
// one partial at its start when P is not a multiple of bs.
struct ReqSpan {
    int32_t lk;   // keys
    int32_t p;    // position of the first query row
    int32_t i0;   // absolute index of the request's first q-block
};

__host__ __device__ inline ReqSpan req_span(const int32_t* cu_q, const int32_t* cu_k, int32_t b) {
    ReqSpan r;
    r.lk = cu_k[b + 1] - cu_k[b];
    const int32_t lq = cu_q[b + 1] - cu_q[b];
    r.p = r.lk - lq;
    r.i0 = lq > 0 ? r.p / kBlock : (r.lk + kBlock - 1) / kBlock;
    return r;
}

// Byte offsets of the workspace regions (all 256-byte aligned).
struct WsLayout {
    size_t cu_blocks;   // int32 [batch + 1]: key blocks before request b
    size_t cu_qblocks;  // int32 [batch + 1]: q-blocks before request b
    size_t cu_tiles;    // int32 [batch + 1] (estimator q-tiles)
    size_t blk_req;     // int32 [max_blocks]: request of every key block
    size_t blk_req_q;   // int32 [max_blocks]: request of every q-block
    size_t order;       // int32 [max_blocks * hkv]: the attention kernel's work order
    size_t qsplit;      // bf16 [2][Hkv][max_blocks * G][d]: q-block means as hi + lo parts,
                        // rows of one KV head's query heads grouped (row = block * G + head)
    size_t ksplit;      // bf16 [2][Hkv][max_blocks][d]: key-block means as hi + lo parts
    size_t kbar_lp;     // bf16 / e4m3 [max_blocks, Hkv, d] (operands of the correction MMA)
    size_t vbar_lp;     // bf16 / e4m3 [max_blocks, Hkv, d]
    size_t total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// `estimator` = false leaves out the split-mean regions (qsplit, ksplit), which
// only the estimator uses: the layout of the attention call's own scratch.
__host__ __device__ inline WsLayout ws_layout(int32_t batch, int64_t max_blocks, int32_t hq,
                                              int32_t hkv, int32_t esize, bool estimator = true) {
    WsLayout w;
    size_t off = 256;
    w.cu_blocks = off;
    off = align256(off + sizeof(int32_t) * (batch + 1));
    w.cu_qblocks = off;
    off = align256(off + sizeof(int32_t) * (batch + 1));
    w.cu_tiles = off;
    off = align256(off + sizeof(int32_t) * (batch + 1));
    w.blk_req = off;
    off = align256(off + sizeof(int32_t) * max_blocks);
    w.blk_req_q = off;
    off = align256(off + sizeof(int32_t) * max_blocks);
    w.order = off;
    off = align256(off + sizeof(int32_t) * max_blocks * hkv);
    w.qsplit = off;
    if (estimator) off = align256(off + 2 * sizeof(uint16_t) * max_blocks * hq * kHeadDim);
    w.ksplit = off;
    if (estimator) off = align256(off + 2 * sizeof(uint16_t) * max_blocks * hkv * kHeadDim);
    w.kbar_lp = off;
    off = align256(off + size_t(esize) * max_blocks * hkv * kHeadDim);
    w.vbar_lp = off;
    off = align256(off + size_t(esize) * max_blocks * hkv * kHeadDim);
    w.total = off;
    return w;
}

// Records the first device-side error; later ones are dropped.
__device__ __forceinline__ void set_error(WsHeader* hdr, int32_t code, int32_t detail) {
    if (atomicCAS(&hdr->status, 0, code) == 0) atomicExch(&hdr->detail, detail);
}

// Bounded wait on an mbarrier phase.  Returns false (after recording
// FP2_ERR_TIMEOUT) when the phase has not completed within ~2^31 cycles
// (about a second), or when `abort` is already set by another role.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr,
                                          volatile int32_t* abort, int32_t where) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    uint32_t spins = 0;
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((++spins & 255u) == 0) {
            if (*abort) return false;
            if (clock64() - start > (1ll << 31)) {
                set_error(hdr, FP2_ERR_TIMEOUT, where);
                *abort = 1;
                return false;
            }
        }
    }
}

// Bounded wait that ignores the abort flag: a role that stops early still waits
// (at most ~2^31 cycles) for the TMA copies it issued to land before the CTA exits.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const long long start = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - start > (1ll << 31)) return false;
    return true;
}

}  // namespace fp2

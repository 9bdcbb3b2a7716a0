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
    int32_t status;        // first device-side fp2_status recorded (0 = none)
    int32_t detail;        // detail of that error (offending index, ...)
    int32_t valid;         // 1 when the last setup pass accepted cu_seqlens
    int32_t total_blocks;  // sum_b ceil(L_b / block_size) of the last setup pass
    int32_t work_next;     // next work item of the persistent attention kernel
};

// Byte offsets of the workspace regions (all 256-byte aligned).
struct WsLayout {
    size_t cu_blocks;   // int32 [batch + 1]
    size_t cu_tiles;    // int32 [batch + 1] (estimator q-tiles)
    size_t blk_req;     // int32 [max_blocks]
    size_t order;       // int32 [max_blocks]: global blocks by block index in the request, descending
    size_t qsplit;      // bf16 [2][Hkv][max_blocks * G][d]: q-block means as hi + lo parts,
                        // rows of one KV head's query heads grouped (row = block * G + head)
    size_t ksplit;      // bf16 [2][Hkv][max_blocks][d]: key-block means as hi + lo parts
    size_t kbar_lp;     // bf16 / e4m3 [max_blocks, Hkv, d] (operands of the correction MMA)
    size_t vbar_lp;     // bf16 / e4m3 [max_blocks, Hkv, d]
    size_t total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(int32_t batch, int64_t max_blocks, int32_t hq,
                                              int32_t hkv, int32_t esize) {
    WsLayout w;
    size_t off = 256;
    w.cu_blocks = off;
    off = align256(off + sizeof(int32_t) * (batch + 1));
    w.cu_tiles = off;
    off = align256(off + sizeof(int32_t) * (batch + 1));
    w.blk_req = off;
    off = align256(off + sizeof(int32_t) * max_blocks);
    w.order = off;
    off = align256(off + sizeof(int32_t) * max_blocks);
    w.qsplit = off;
    off = align256(off + 2 * sizeof(uint16_t) * max_blocks * hq * kHeadDim);
    w.ksplit = off;
    off = align256(off + 2 * sizeof(uint16_t) * max_blocks * hkv * kHeadDim);
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

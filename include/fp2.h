/*
 * fp2.h -- C ABI of the B200 (sm_100a) block-sparse prefill attention library.
 *
 * The method (write-ups of "FlashPrefill V2: Block-Sparse Prefill Attention for
 * Long-Context LLM Serving"):
 *   - lode.cx, "How It Works": a block-level sample of attention scores, its
 *     maximum, and a threshold relative to that maximum pick the attended
 *     blocks; a mean correction term compensates the pruned mass;
 *   - aipulsen.com: scores are estimated at the block level;
 *   - aimodeling.com, "From Prototype to Production": max-based dynamic
 *     thresholding, the mean correction term, FP8, paged KV cache and
 *     continuous batching;
 *   - stuffinsider.com, "Technical Details": queries and keys are cut into
 *     blocks; prefill only.
 * The write-ups fix these steps only in words.  The exact readings used here:
 *   blocks   block_size rows from the first token of each request; causal
 *            (token r sees keys c <= r of its own request);
 *   estimate qbar/kbar/vbar = per-block means of the (dequantised) rows;
 *            s[h,i,j] = sm_scale * qbar[h,i] . kbar[h/G, j] for j <= i;
 *   keep     m = max_j s; head h keeps j iff s - m >= ln(alpha); a KV head keeps
 *            the union over its G query heads plus the diagonal block;
 *            alpha <= 0 keeps every causal block;
 *   attend   softmax attention over kept blocks; with correction, each pruned
 *            block j < i adds n_j * exp(sm_scale q.kbar_j) * vbar_j to the
 *            numerator and n_j * exp(sm_scale q.kbar_j) to the denominator.
 *
 * Layouts (all row-major, token-major "THD"):
 *   q        [total_tokens, Hq, head_dim]          bf16 or e4m3
 *   k, v     [total_tokens, Hkv, head_dim]         contiguous mode
 *   k_pool   [num_pages * block_size, Hkv, head_dim] paged mode; page p holds
 *            rows p*block_size .. p*block_size + block_size - 1
 *   out      [total_tokens, Hq, head_dim]          bf16
 *   lse      [total_tokens, Hq]                    fp32 natural-log sum-exp
 *   cu_seqlens [batch + 1] int32, cu_seqlens[0] = 0, non-decreasing,
 *            cu_seqlens[batch] = total_tokens; request b is rows
 *            cu_seqlens[b] .. cu_seqlens[b+1]-1 of q (and of k/v when contiguous);
 *            a request may be empty.  With total_tokens == 0 a call only
 *            checks cu_seqlens (q, k, v and out may then be NULL).
 *   block_table [batch, max_blocks_per_seq] int32: page of logical block j of
 *            request b (paged mode).
 *   Blocks of all requests are numbered globally in request order:
 *   block id of (b, j) = sum_{b' < b} ceil(L_b' / block_size) + j.
 *
 * Ownership: every pointer passed to a compute call is a DEVICE pointer owned
 * by the caller, except the fp2_params / fp2_blockmeta structs themselves,
 * which are read on the host during the call.  The library allocates no memory
 * and keeps no global state; scratch memory is the caller's workspace (the one
 * exception, fp2_sparse_prefill_noalloc, uses a static device array instead).
 * Alignment: q, k, v (or the pools), out, k_mean and v_mean start on 16-byte
 * boundaries (TMA operands and 16-byte accesses), lse on 4 bytes, the workspace
 * on 256 bytes; otherwise the call returns FP2_ERR_INVALID_ARG (FP2_ERR_WORKSPACE
 * for the workspace) without enqueuing anything.  An out that starts on a 32-byte
 * boundary is written with 32-byte stores, which makes the attention calls a few
 * percent faster; the bytes written are the same either way.
 *
 * Errors: argument errors are returned synchronously and nothing is enqueued.
 * A failed launch returns FP2_ERR_CUDA.  Errors found on the device (a bad
 * cu_seqlens, a page index outside the pool, a wait that ran out of time) are
 * recorded in a flag inside the workspace; the kernels then skip the bad
 * access and the call's results are undefined.  fp2_get_error() reads and
 * clears that flag.
 *
 * All compute calls are asynchronous on `stream` (a cudaStream_t, NULL = the
 * legacy default stream).  Calls sharing one workspace must be ordered on the
 * device (same stream, or synchronised streams).
 */
#ifndef FP2_H
#define FP2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp2_status {
    FP2_OK = 0,
    FP2_ERR_INVALID_ARG = 1,   /* bad argument; nothing was enqueued */
    FP2_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim != 128) */
    FP2_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small */
    FP2_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
    FP2_ERR_TIMEOUT = 5,       /* device: a pipeline wait exceeded its limit */
    FP2_ERR_BAD_INDEX = 6      /* device: bad cu_seqlens or page index */
} fp2_status;

typedef enum fp2_dtype {
    FP2_BF16 = 0,              /* q/k/v bf16 */
    FP2_E4M3 = 1               /* q/k/v float8 e4m3 codes with per-head scales */
} fp2_dtype;

/* Problem parameters (read on the host). */
typedef struct fp2_params {
    int32_t num_q_heads;       /* Hq >= 1 */
    int32_t num_kv_heads;      /* Hkv >= 1, Hq % Hkv == 0 (G = Hq / Hkv query heads per KV head) */
    int32_t head_dim;          /* must be 128 */
    int32_t block_size;        /* must be 128; also the KV page size */
    float alpha;               /* threshold; <= 0 keeps every causal block; must be <= 1 */
    float sm_scale;            /* softmax scale tau; 0 selects 1/sqrt(head_dim) */
    int32_t correction;        /* 0: drop pruned blocks; 1: mean correction; 2: mean correction
                                  with the variance term (see fp2_sparse_prefill) */
    int32_t dtype;             /* fp2_dtype */
    const float* q_scale;      /* e4m3 only: device [Hq] dequantisation scales, finite and
                                  >= 0 (an all-zero head may have scale 0) */
    const float* k_scale;      /* e4m3 only: device [Hkv] */
    const float* v_scale;      /* e4m3 only: device [Hkv] */
} fp2_params;

/* Block metadata written by the estimator and read by the attention calls.
 * All arrays are device memory owned by the caller. */
typedef struct fp2_blockmeta {
    int32_t* kept_cnt;         /* [max_blocks, Hkv]: number of kept key blocks */
    int32_t* kept_idx;         /* [max_blocks, Hkv, nb_max]: kept key blocks of every
                                  q-block, ascending, diagonal block last */
    float* k_mean;             /* [max_blocks, Hkv, head_dim] fp32 dequantised block means */
    float* v_mean;             /* [max_blocks, Hkv, head_dim] fp32; needed when correction != 0 */
    float* score_dbg;          /* optional (NULL): [max_blocks, Hq, nb_max] s - m, fp32;
                                  entries j > i are left untouched */
    int32_t nb_max;            /* row stride of kept_idx / score_dbg, >= ceil(max_seqlen / block_size) */
    int32_t max_blocks;        /* capacity in blocks, >= sum_b ceil(L_b / block_size) */
    float* k_var;              /* optional (NULL): [max_blocks, Hkv] fp32, the key variance of
                                  every block averaged over the head dimensions (dequantised);
                                  written by the estimator when non-NULL, needed when
                                  correction == 2 */
} fp2_blockmeta;

/* Upper bound of sum_b ceil(L_b / block_size) for any batch of `batch` requests
 * holding `total_tokens` tokens: total_tokens / block_size + batch. */
int64_t fp2_max_blocks(int32_t batch, int64_t total_tokens, int32_t block_size);

/* Workspace bytes needed by every call below for this problem size (an upper
 * bound independent of the lengths inside cu_seqlens).  Returns 0 for invalid
 * arguments. */
size_t fp2_workspace_bytes(const fp2_params* params, int32_t batch, int64_t total_tokens,
                           int32_t max_seqlen);

/* Clears the workspace's device error flag (enqueued on `stream`).  Call once
 * on a new workspace before its first use. */
fp2_status fp2_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* fp2_estimate -- the block-score estimator and the max-relative threshold.
 * Defined by: lode.cx, "How It Works" (a small sample of attention scores,
 * its maximum, and the blocks above a threshold relative to that maximum);
 * aipulsen.com (scores estimated at the block level); aimodeling.com, "From
 * Prototype to Production" (max-based dynamic thresholding).  The sample is
 * read here as the block-mean score (exact mean of the block pair's token
 * logits), the threshold as exp(s - m) >= alpha (see the readings above).
 * Computes block means, block scores, per-head row maximum, alpha threshold,
 * GQA union, forced diagonal and the ascending kept lists.  Writes
 * meta->kept_cnt, kept_idx, k_mean, v_mean (v_mean only when non-NULL) and
 * score_dbg (when non-NULL).
 *   q            [total_tokens, Hq, d]
 *   k, v         contiguous [total_tokens, Hkv, d] when block_table == NULL,
 *                else page pools [num_pages * block_size, Hkv, d]
 *   block_table  NULL (contiguous) or [batch, max_blocks_per_seq] page indices
 *   num_pages    pages in the pools (paged mode; ignored otherwise); num_pages *
 *                block_size < 2^31, else FP2_ERR_UNSUPPORTED
 * Errors: bad arguments or sizes are returned before anything is enqueued; a
 * bad cu_seqlens or a page index outside the pool is flagged on the device. */
fp2_status fp2_estimate(const fp2_params* params, const void* q, const void* k, const void* v,
                        const int32_t* cu_seqlens, int32_t batch, int64_t total_tokens,
                        int32_t max_seqlen, const int32_t* block_table,
                        int32_t max_blocks_per_seq, int32_t num_pages, fp2_blockmeta* meta,
                        void* workspace, size_t ws_bytes, void* stream);

/* fp2_sparse_prefill -- sparse attention over the kept blocks with the mean
 * correction, contiguous K/V.
 * Defined by: lode.cx, "How It Works" (attend only what passes the threshold;
 * a mean correction term compensates what pruning removes) and the operator
 * list after it (PackGQA: the query heads of a KV head share its K/V tiles;
 * FP8); aimodeling.com, "From Prototype to Production" (the mean correction
 * suppresses the approximation error; FP8 inference); stuffinsider.com,
 * "Technical Details" (query and key blocks; prefill, all queries in one pass).
 * Attends over the kept blocks of `meta` (from fp2_estimate on the same
 * inputs, or any caller-made lists that are ascending, in [0, i] and end with
 * the diagonal block i), plus the mean correction when params->correction != 0
 * (then meta->k_mean and v_mean must hold the block means).  Writes out (bf16)
 * and, when non-NULL, lse.  `meta` is only read.
 * correction == 2 adds to every pruned block's corrected logit the second-order
 * term (sm_scale^2 / 2) |q_r|^2 kvar_j, kvar_j = meta->k_var (the block's key
 * variance averaged over the dimensions): by Jensen's inequality the plain mean
 * correction undercounts a block's mass by about e^{var/2} of its logits, and
 * this term restores it when the keys' variance is spread evenly over the
 * dimensions.  It is an extension of the write-ups' mean correction (lode.cx,
 * "How It Works"; aimodeling.com: the correction suppresses the approximation
 * error), not a step they state.  Its length limit is lower: the attention
 * stages one variance per pruned block, so ceil(max_seqlen / block_size) may be
 * at most FP2_MAX_SEQ_BLOCKS_VAR_BF16 (2048 blocks, 262144 tokens) for bf16 or
 * FP2_MAX_SEQ_BLOCKS_VAR_E4M3 (4096 blocks, 524288 tokens) for e4m3.
 * Length limit of the attention calls (this one, fp2_prefill_paged and
 * fp2_sparse_prefill_noalloc): a work item keeps its kept-block list in shared
 * memory, so ceil(max_seqlen / block_size) may be at most FP2_MAX_SEQ_BLOCKS_BF16
 * (4129 blocks, 528512 tokens) for bf16 and FP2_MAX_SEQ_BLOCKS_E4M3 (8071
 * blocks, 1033088 tokens) for e4m3; longer returns FP2_ERR_UNSUPPORTED.
 * Errors: bad arguments or sizes are returned before anything is enqueued; a
 * kept list that breaks the rules above is flagged on the device
 * (FP2_ERR_BAD_INDEX) and replaced by the diagonal block alone. */
#define FP2_MAX_SEQ_BLOCKS_BF16 4129
#define FP2_MAX_SEQ_BLOCKS_E4M3 8071
#define FP2_MAX_SEQ_BLOCKS_VAR_BF16 2048
#define FP2_MAX_SEQ_BLOCKS_VAR_E4M3 4096
fp2_status fp2_sparse_prefill(const fp2_params* params, const void* q, const void* k,
                              const void* v, const int32_t* cu_seqlens, int32_t batch,
                              int64_t total_tokens, int32_t max_seqlen,
                              const fp2_blockmeta* meta, void* out, float* lse, void* workspace,
                              size_t ws_bytes, void* stream);

/* fp2_prefill_paged -- fp2_sparse_prefill on a paged KV cache.
 * Defined by: aimodeling.com, "From Prototype to Production" (native support
 * of a paged KV cache and continuous batching, as an attention backend of a
 * serving framework); lode.cx, after the operator list (paged KV cache and
 * continuous batching).
 * Same computation and arguments as fp2_sparse_prefill, with the K/V tiles of
 * logical block j of request b read from page block_table[b][j] of the pools
 * k_pool / v_pool [num_pages * block_size, Hkv, d].  `meta` comes from
 * fp2_estimate on the same pools and block table (or from the caller) and is
 * only read.  num_pages * block_size < 2^31, else FP2_ERR_UNSUPPORTED.  A page
 * index outside [0, num_pages) is flagged on the device (FP2_ERR_BAD_INDEX) and
 * page 0 is read in its place. */
fp2_status fp2_prefill_paged(const fp2_params* params, const void* q, const void* k_pool,
                             const void* v_pool, const int32_t* cu_seqlens, int32_t batch,
                             int64_t total_tokens, int32_t max_seqlen, const int32_t* block_table,
                             int32_t max_blocks_per_seq, int32_t num_pages,
                             const fp2_blockmeta* meta, void* out, float* lse, void* workspace,
                             size_t ws_bytes, void* stream);

/* fp2_estimate_chunked / fp2_prefill_chunked -- chunked prefill on a KV cache
 * that already holds a prefix of each request.
 * Defined by: aimodeling.com, "From Prototype to Production" (paged KV cache and
 * continuous batching in a serving framework's attention backend); the
 * write-ups do not treat chunks, so the plainest extension is taken.  Request
 * b has Lk_b keys (cu_seqlens_k) and computes only its last Lq_b <= Lk_b query
 * rows (cu_seqlens_q), at positions P_b = Lk_b - Lq_b .. Lk_b - 1: query row t
 * of the chunk sees keys c <= P_b + t.  Key blocks are as in plain prefill.
 * q-blocks keep the request's absolute grid of block_size positions, so the
 * request has q-blocks i = floor(P_b / bs) .. ceil(Lk_b / bs) - 1 (none when
 * Lq_b = 0), the first one holding the query rows from P_b on; qbar of a
 * q-block is the mean of the query rows it holds.  With cu_seqlens_q ==
 * cu_seqlens_k these are fp2_estimate and fp2_sparse_prefill / fp2_prefill_paged.
 *   q            [total_q, Hq, d] (the chunk rows); out [total_q, Hq, d]; lse [total_q, Hq]
 *   k, v         contiguous [total_k, Hkv, d] (all keys) when block_table == NULL,
 *                else page pools as in fp2_prefill_paged
 *   meta         kept_cnt / kept_idx rows: q-blocks, numbered globally in request
 *                order (request b's q-blocks follow those of the requests before
 *                it); their entries are key-block indices j <= i of the request.
 *                k_mean / v_mean rows: key blocks (sum_b ceil(Lk_b / bs) of them),
 *                so max_blocks >= fp2_max_blocks(batch, total_k, bs)
 *   max_seqlen_k >= every Lk_b; the workspace from
 *                fp2_workspace_bytes(params, batch, total_k, max_seqlen_k)
 * Errors as for the plain calls; Lq_b > Lk_b is flagged on the device. */
fp2_status fp2_estimate_chunked(const fp2_params* params, const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                                int32_t batch, int64_t total_q, int64_t total_k,
                                int32_t max_seqlen_k, const int32_t* block_table,
                                int32_t max_blocks_per_seq, int32_t num_pages,
                                fp2_blockmeta* meta, void* workspace, size_t ws_bytes,
                                void* stream);
fp2_status fp2_prefill_chunked(const fp2_params* params, const void* q, const void* k, const void* v,
                               const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                               int32_t batch, int64_t total_q, int64_t total_k,
                               int32_t max_seqlen_k, const int32_t* block_table,
                               int32_t max_blocks_per_seq, int32_t num_pages,
                               const fp2_blockmeta* meta, void* out, float* lse, void* workspace,
                               size_t ws_bytes, void* stream);

/* Synchronises `stream`, returns the first device-side error recorded in the
 * workspace since the last call (FP2_OK if none) and clears it. */
fp2_status fp2_get_error(void* workspace, void* stream);

/* Static description of a status code. */
const char* fp2_status_string(fp2_status status);

/* Size of the device scratch array behind fp2_sparse_prefill_noalloc (8 MiB). */
#define FP2_NOALLOC_SCRATCH_BYTES (8u << 20)

/* Allocation-free form of fp2_sparse_prefill.  The FlashPrefill V2 write-ups
 * have no counterpart of this call; it exists for callers that cannot allocate
 * device memory at the point where they run attention: a plugin or operator
 * inside a host framework that owns every device allocation (and forbids
 * allocating behind its back), code whose memory budget is fixed up front, or
 * latency-critical code that must avoid cudaMalloc's implicit device
 * synchronisation.  Such callers pass no workspace.  Instead the library uses
 * one file-scope device array of FP2_NOALLOC_SCRATCH_BYTES, which every GPU
 * that loads the library holds until the process exits.
 *   - Arguments, layouts and results are those of fp2_sparse_prefill.
 *   - Returns FP2_ERR_WORKSPACE, without enqueuing anything, when the problem
 *     needs more scratch than FP2_NOALLOC_SCRATCH_BYTES (about 4.2 MB for a
 *     131072-token request with 8 KV heads).
 *   - device_status: optional caller-owned DEVICE int32; when non-NULL it
 *     receives (asynchronously, on `stream`) the device-side fp2_status of
 *     this call (0 = none), since there is no workspace to query with
 *     fp2_get_error.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress), so make that first call before any CUDA stream
 *     capture on that device.
 *   - All calls share the one array, and the array keeps the last call's
 *     contents: calls that overlap on the GPU (different streams, or
 *     different host threads, without ordering) race on it.
 *   - It calls no cudaMalloc/cudaFree or allocating library routine. */
fp2_status fp2_sparse_prefill_noalloc(const fp2_params* params, const void* q, const void* k,
                                      const void* v, const int32_t* cu_seqlens, int32_t batch,
                                      int64_t total_tokens, int32_t max_seqlen,
                                      const fp2_blockmeta* meta, void* out, float* lse,
                                      int32_t* device_status, void* stream);

/* Library version (major * 10000 + minor * 100 + patch). */
int32_t fp2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP2_H */

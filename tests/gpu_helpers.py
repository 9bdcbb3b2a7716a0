"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_prefill_b200 as fp2
from oracle.oracle import Oracle, chunk_starts, near_threshold

BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
E4M3_MAX_ABS = 6e-2
# e4m3 mean-abs: not fixed by the stated tolerances; taken with the bf16 bounds' ratio
# (mean-abs = max-abs / 10), which catches a systematic bias of the e4m3 correction
# operands (block means rounded to e4m3) that the max-abs bound alone would let through
E4M3_MEAN_ABS = 6e-3

_ORC = None


def oracle() -> Oracle:
    global _ORC
    if _ORC is None:
        _ORC = Oracle()
    return _ORC


def params_for(wl, alpha=None, correction=True, dev="cuda"):
    p = fp2.Params(num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads,
                   alpha=wl.alpha if alpha is None else alpha, correction=correction,
                   dtype=fp2.FP2_E4M3 if wl.dtype == "e4m3" else fp2.FP2_BF16)
    if wl.dtype == "e4m3":
        p.q_scale = torch.from_numpy(wl.q_scale).to(dev)
        p.k_scale = torch.from_numpy(wl.k_scale).to(dev)
        p.v_scale = torch.from_numpy(wl.v_scale).to(dev)
    return p


def run_gpu(wl, alpha=None, correction=True, paged=False, scores=False, lse=True, dev="cuda", kept=None,
            out_shift=0):
    """Estimator + attention on the GPU.  Returns numpy arrays.  With ``kept``
    (dict of kept_cnt / kept_idx numpy arrays, e.g. the oracle's) the attention
    runs on those lists instead of the estimator's (the block means still come
    from the estimator).  ``out_shift`` places the output ``out_shift`` bf16
    elements past the start of its allocation (8: 16-byte but not 32-byte aligned)."""
    params = params_for(wl, alpha, correction, dev)
    T, B = wl.total_tokens, wl.batch
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    q = wl.q.to(dev)
    meta = fp2.BlockMeta.empty(params, B, T, wl.max_seqlen, dev, scores=scores)
    ws = fp2.Workspace(params, B, T, wl.max_seqlen, dev)
    n_out = T * wl.num_q_heads * 128
    out_buf = torch.full((n_out + 16,), float("nan"), dtype=torch.bfloat16, device=dev)
    out = out_buf[out_shift:out_shift + n_out].view(T, wl.num_q_heads, 128)
    assert out_shift != 8 or out.data_ptr() % 32 == 16
    lse_t = torch.full((T, wl.num_q_heads), float("nan"), dtype=torch.float32, device=dev) if lse else None
    def given_mask():
        if kept is not None:
            n = kept["kept_cnt"].shape[0]
            meta.kept_cnt[:n].copy_(torch.from_numpy(np.ascontiguousarray(kept["kept_cnt"], np.int32)))
            ki = np.ascontiguousarray(kept["kept_idx"], np.int32)
            meta.kept_idx[:n, :, :ki.shape[2]].copy_(torch.from_numpy(ki))

    if paged:
        bt = torch.from_numpy(wl.block_table).to(dev)
        kp, vp = wl.k_pool.to(dev), wl.v_pool.to(dev)
        fp2.estimate(params, q, kp, vp, cu, wl.max_seqlen, meta, ws, block_table=bt, num_pages=wl.num_pages)
        given_mask()
        fp2.prefill_paged(params, q, kp, vp, cu, wl.max_seqlen, bt, wl.num_pages, meta, out, ws, lse=lse_t)
    else:
        k, v = wl.k.to(dev), wl.v.to(dev)
        fp2.estimate(params, q, k, v, cu, wl.max_seqlen, meta, ws)
        given_mask()
        fp2.sparse_prefill(params, q, k, v, cu, wl.max_seqlen, meta, out, ws, lse=lse_t)
    torch.cuda.synchronize()
    err = fp2.get_error(ws)
    assert err == 0, f"device error flag {fp2.status_string(err)}"
    nblk = oracle().total_blocks(wl.cu_seqlens, 128)
    res = {
        "kept_cnt": meta.kept_cnt[:nblk].cpu().numpy(),
        "kept_idx": meta.kept_idx[:nblk].cpu().numpy(),
        "k_mean": meta.k_mean[:nblk].cpu().numpy(),
        "v_mean": meta.v_mean[:nblk].cpu().numpy(),
        "k_var": meta.k_var[:nblk].cpu().numpy() if meta.k_var is not None else None,
        "o": out.float().cpu().numpy(),
        "lse": lse_t.cpu().numpy() if lse else None,
        "score_dbg": meta.score_dbg[:nblk].cpu().numpy() if scores else None,
    }
    return res


def mask_sets(cnt, idx):
    return [[set(idx[t, g, :cnt[t, g]].tolist()) for g in range(cnt.shape[1])] for t in range(cnt.shape[0])]


# near-threshold statistics of every mask comparison in this session, printed
# by conftest.py's terminal summary: (test, near, excused, outside, compared)
MASK_STATS = []


def local_block_index(cu_seqlens, bs=128):
    """Index inside its request of every global q-block (requests in order)."""
    lens = np.diff(np.asarray(cu_seqlens, np.int64))
    return np.concatenate([np.arange((int(L) + bs - 1) // bs) for L in lens] or [np.zeros(0, np.int64)])


def compare_masks(gpu, est, alpha, Hkv, cu_seqlens, label="", block_index=None):
    """Kept lists must match except at near-threshold blocks.

    Returns dict(outside, excused, near, compared): kept-list entries that differ
    outside the near-threshold band, differing entries the band excuses, blocks
    inside the band (any head of the group), and blocks compared (union of both
    lists).  Also checks that every GPU list is ascending, in [0, i] and ends
    with the diagonal block i, and records the counts in MASK_STATS."""
    near = near_threshold(est["s"], est["m"], Hkv, alpha, None)
    gs = mask_sets(gpu["kept_cnt"], gpu["kept_idx"])
    os_ = mask_sets(est["kept_cnt"], est["kept_idx"])
    ii = local_block_index(cu_seqlens) if block_index is None else np.asarray(block_index)
    assert len(ii) == len(gs), "q-block count differs from cu_seqlens"
    outside, excused, total = 0, 0, 0
    for t in range(len(gs)):
        for g in range(Hkv):
            diff = gs[t][g] ^ os_[t][g]
            total += len(gs[t][g] | os_[t][g])
            for j in diff:
                if near[t, g, j]:
                    excused += 1
                else:
                    outside += 1
            c = int(gpu["kept_cnt"][t, g])
            lst = gpu["kept_idx"][t, g, :c]
            assert 1 <= c <= ii[t] + 1, f"q-block {t} head {g}: {c} kept blocks"
            assert (np.diff(lst) > 0).all() and lst[0] >= 0, f"q-block {t} head {g}: list not ascending"
            assert lst[-1] == ii[t], f"q-block {t} head {g}: list ends at {lst[-1]}, not the diagonal {ii[t]}"
    res = {"outside": outside, "excused": excused, "near": int(near.sum()), "compared": total}
    MASK_STATS.append((label, res))
    return res


def check_mask_counts(res):
    """No difference outside the band, and the band excuses at most
    max(2, 0.1% of the compared blocks): the GPU's score error is far inside
    the 1e-3 band, so excused differences must stay rare."""
    assert res["outside"] == 0, (f"{res['outside']} kept-list entries differ outside the near-threshold band "
                                 f"({res['near']} near, {res['compared']} compared)")
    assert res["excused"] <= max(2, res["compared"] // 1000), (
        f"{res['excused']} kept-list differences inside the near-threshold band "
        f"({res['near']} near, {res['compared']} compared)")


# output errors of every parity check in this session, printed by conftest.py's
# terminal summary: (test, max-abs, mean-abs)
OUT_STATS = []


def record_output_errors(label, mx, mn):
    OUT_STATS.append((label, mx, mn))


def out_errors(gpu_o, ref_o, rows=None):
    a, b = gpu_o, ref_o
    if rows is not None:
        a, b = a[rows], b[rows]
    m = ~np.isnan(b)
    e = np.abs(a[m] - b[m])
    return float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0


def sample_blocks(nblk, n, seed, include=()):
    rng = np.random.default_rng(seed)
    pick = set(int(x) for x in include if 0 <= x < nblk)
    extra = rng.choice(nblk, size=min(n, nblk), replace=False)
    for x in extra:
        if len(pick) >= n:
            break
        pick.add(int(x))
    return np.array(sorted(pick), dtype=np.int64)


def sample_blocks_per_request(cu_seqlens, n, seed, bs=128):
    """Global q-blocks: up to ``n`` seeded ones per request, its first and last included."""
    rng = np.random.default_rng(seed)
    lens = np.diff(np.asarray(cu_seqlens, np.int64))
    sel, base = [], 0
    for L in lens:
        nb = (int(L) + bs - 1) // bs
        if nb:
            pick = {0, nb - 1}
            for x in rng.permutation(nb):
                if len(pick) >= min(n, nb):
                    break
                pick.add(int(x))
            sel.extend(base + p for p in sorted(pick))
        base += nb
    return np.array(sel, dtype=np.int64)


def rows_of_blocks(cu_seqlens, sel, bs=128):
    """Token rows of the given global q-blocks."""
    lens = np.diff(cu_seqlens)
    starts = []
    t = 0
    for b, L in enumerate(lens):
        for j in range((int(L) + bs - 1) // bs):
            starts.append((int(cu_seqlens[b]) + j * bs, min(bs, int(L) - j * bs)))
            t += 1
    rows = []
    for s in sel:
        r0, n = starts[int(s)]
        rows.extend(range(r0, r0 + n))
    return np.array(rows, dtype=np.int64)


def tau(wl):
    return 1.0 / math.sqrt(wl.head_dim)


# ---------------------------------------------------------------------------
# chunked prefill (queries are the last rows of each request)
# ---------------------------------------------------------------------------
def chunk_block_index(wl, bs=128):
    """Absolute block index i of every q-block of a chunked workload, in the global
    q-block order: request b's q-blocks are i = floor(P_b / bs) .. ceil(Lk_b / bs) - 1."""
    p0 = chunk_starts(wl.cu_seqlens_q, wl.cu_seqlens)
    out = []
    for P, lq, lk in zip(p0, wl.query_lens, wl.seqlens):
        if lq > 0:
            out.extend(range(int(P) // bs, (int(lk) + bs - 1) // bs))
    return np.array(out, dtype=np.int64)


def chunk_rows_of_blocks(wl, sel, bs=128):
    """Rows of the chunk's q tensor held by the given global q-blocks."""
    p0 = chunk_starts(wl.cu_seqlens_q, wl.cu_seqlens)
    cuq = wl.cu_seqlens_q
    spans = []
    for b, (P, lq, lk) in enumerate(zip(p0, wl.query_lens, wl.seqlens)):
        if lq == 0:
            continue
        for i in range(int(P) // bs, (int(lk) + bs - 1) // bs):
            lo, hi = max(int(P), i * bs), min(int(lk), i * bs + bs)
            spans.append((int(cuq[b]) + lo - int(P), hi - lo))
    rows = []
    for s_ in sel:
        r0, n = spans[int(s_)]
        rows.extend(range(r0, r0 + n))
    return np.array(rows, dtype=np.int64)


def run_gpu_chunked(wl, alpha=None, correction=True, paged=False, lse=True, dev="cuda", kept=None):
    """fp2_estimate_chunked + fp2_prefill_chunked on a chunked workload (contiguous K/V
    or the page pools).  Returns numpy arrays; kept lists per q-block, means per key block."""
    params = params_for(wl, alpha, correction, dev)
    B, Tq, Tk = wl.batch, wl.total_queries, wl.total_tokens
    cu_q = torch.from_numpy(wl.cu_seqlens_q).to(dev)
    cu_k = torch.from_numpy(wl.cu_seqlens).to(dev)
    q = wl.q.to(dev)
    meta = fp2.BlockMeta.empty(params, B, Tk, wl.max_seqlen, dev)
    ws = fp2.Workspace(params, B, Tk, wl.max_seqlen, dev)
    out = torch.full((Tq, wl.num_q_heads, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    lse_t = torch.full((Tq, wl.num_q_heads), float("nan"), dtype=torch.float32, device=dev) if lse else None
    if paged:
        bt = torch.from_numpy(wl.block_table).to(dev)
        k, v, npg = wl.k_pool.to(dev), wl.v_pool.to(dev), wl.num_pages
    else:
        bt, k, v, npg = None, wl.k.to(dev), wl.v.to(dev), 0
    fp2.estimate_chunked(params, q, k, v, cu_q, cu_k, Tk, wl.max_seqlen, meta, ws, block_table=bt, num_pages=npg)
    if kept is not None:
        n = kept["kept_cnt"].shape[0]
        meta.kept_cnt[:n].copy_(torch.from_numpy(np.ascontiguousarray(kept["kept_cnt"], np.int32)))
        ki = np.ascontiguousarray(kept["kept_idx"], np.int32)
        meta.kept_idx[:n, :, :ki.shape[2]].copy_(torch.from_numpy(ki))
    fp2.prefill_chunked(params, q, k, v, cu_q, cu_k, Tk, wl.max_seqlen, meta, out, ws, lse=lse_t,
                        block_table=bt, num_pages=npg)
    torch.cuda.synchronize()
    err = fp2.get_error(ws)
    assert err == 0, f"device error flag {fp2.status_string(err)}"
    nq = len(chunk_block_index(wl))
    nk = oracle().total_blocks(wl.cu_seqlens, 128)
    return {
        "kept_cnt": meta.kept_cnt[:nq].cpu().numpy(),
        "kept_idx": meta.kept_idx[:nq].cpu().numpy(),
        "k_mean": meta.k_mean[:nk].cpu().numpy(),
        "o": out.float().cpu().numpy(),
        "lse": lse_t.cpu().numpy() if lse else None,
    }

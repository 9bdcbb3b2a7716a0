"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_prefill_b200 as fp2
from oracle.oracle import Oracle, near_threshold

BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
E4M3_MAX_ABS = 6e-2

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


def run_gpu(wl, alpha=None, correction=True, paged=False, scores=False, lse=True, dev="cuda"):
    """Estimator + attention on the GPU.  Returns numpy arrays."""
    params = params_for(wl, alpha, correction, dev)
    T, B = wl.total_tokens, wl.batch
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    q = wl.q.to(dev)
    meta = fp2.BlockMeta.empty(params, B, T, wl.max_seqlen, dev, scores=scores)
    ws = fp2.Workspace(params, B, T, wl.max_seqlen, dev)
    out = torch.full((T, wl.num_q_heads, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    lse_t = torch.full((T, wl.num_q_heads), float("nan"), dtype=torch.float32, device=dev) if lse else None
    if paged:
        bt = torch.from_numpy(wl.block_table).to(dev)
        fp2.prefill_paged(params, q, wl.k_pool.to(dev), wl.v_pool.to(dev), cu, wl.max_seqlen, bt,
                          wl.num_pages, meta, out, ws, lse=lse_t)
    else:
        k, v = wl.k.to(dev), wl.v.to(dev)
        fp2.estimate(params, q, k, v, cu, wl.max_seqlen, meta, ws)
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
        "o": out.float().cpu().numpy(),
        "lse": lse_t.cpu().numpy() if lse else None,
        "score_dbg": meta.score_dbg[:nblk].cpu().numpy() if scores else None,
    }
    return res


def mask_sets(cnt, idx):
    return [[set(idx[t, g, :cnt[t, g]].tolist()) for g in range(cnt.shape[1])] for t in range(cnt.shape[0])]


def compare_masks(gpu, est, alpha, Hkv):
    """Kept lists must match except at near-threshold blocks.  Returns
    (mismatches outside the band, near-threshold blocks, blocks compared)."""
    near = near_threshold(est["s"], est["m"], Hkv, alpha, None)
    gs = mask_sets(gpu["kept_cnt"], gpu["kept_idx"])
    os_ = mask_sets(est["kept_cnt"], est["kept_idx"])
    bad, nnear, total = 0, int(near.sum()), 0
    for t in range(len(gs)):
        for g in range(Hkv):
            diff = gs[t][g] ^ os_[t][g]
            total += len(gs[t][g] | os_[t][g])
            for j in diff:
                if not near[t, g, j]:
                    bad += 1
    # lists are ascending with the diagonal last
    for t in range(len(gs)):
        for g in range(Hkv):
            c = gpu["kept_cnt"][t, g]
            lst = gpu["kept_idx"][t, g, :c]
            assert c >= 1 and (np.diff(lst) > 0).all()
    return bad, nnear, total


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

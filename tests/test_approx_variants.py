"""Approximation quality of the mean correction and two variants of it (CPU, oracle).

Not a parity test.  The method approximates dense causal attention, and this
measures how far its output lands from dense attention.  The input is the seeded
Llama-3-8B-shaped workload of the 128K benchmark, generated at 8192 tokens
(alpha = 0.05).  The error is taken over every row of six seeded q-blocks and
all 32 query heads.  Corrections:
  none      pruned blocks dropped;
  mean      the mean correction, which the GPU kernels implement;
  variance  the mean correction plus half the within-block logit variance,
            taken per dimension of the keys (oracle correction mode 2);
  pooled    the mean correction with the q-block's mean query (mode 3);
  isotropic the variance term with the key variance averaged over the
            dimensions (mode 4): one scalar per row times one per block;
  hybrid8   the variance term with the 8 channels of largest total key
            variance per KV head kept exactly and the rest averaged (mode 2
            on variances whose other channels are replaced by their mean);
  strided   the mean correction, with kept lists estimated from every 8th
            query row of each block instead of all 128 (the estimator would
            read an eighth of Q).
By Jensen's inequality the mean correction undercounts a pruned block's mass by
about exp(var / 2), which the variance term restores.  The test requires
variance < mean < none and prints the errors (run with -s).  Set
FP2_APPROX_SEQLEN=32768 to run the same study at 32K, and FP2_APPROX_ALPHA to change
alpha.  FP2_APPROX_OUTLIERS="n,gain[,both]" scales n seeded key channels (and the
same query channels with ",both") by gain: outlier channels, as in trained models,
make the key variance anisotropic.
"""
import math
import os

import numpy as np
import torch

from oracle.oracle import Oracle
from workloads import make_config

SEQLEN = int(os.environ.get("FP2_APPROX_SEQLEN", "8192"))
ALPHA = float(os.environ.get("FP2_APPROX_ALPHA", "0.05"))
# "n,gain[,both]": multiply n seeded key channels (and the same query channels with
# "both") by gain, for key variance that is not isotropic
OUTLIERS = os.environ.get("FP2_APPROX_OUTLIERS", "")


def _dense_rows(q, k, v, rows, hq, hkv, tau):
    """Dense causal attention (torch fp64) of the given rows of a single request,
    128 rows at a time."""
    g = hq // hkv
    end_all = int(rows.max()) + 1
    kt_all = torch.from_numpy(k[:end_all]).double().repeat_interleave(g, dim=1).transpose(0, 1)  # [Hq, end, d]
    vt_all = torch.from_numpy(v[:end_all]).double().repeat_interleave(g, dim=1).transpose(0, 1)
    out = []
    for s in range(0, len(rows), 128):
        rr = rows[s:s + 128]
        end = int(rr.max()) + 1
        qt = torch.from_numpy(q[rr]).double().transpose(0, 1)                                    # [Hq, R, d]
        logits = (qt @ kt_all[:, :end].transpose(1, 2)) * tau
        mask = torch.arange(end)[None, :] <= torch.from_numpy(rr)[:, None]
        w = torch.softmax(logits.masked_fill(~mask[None], -math.inf), dim=-1)
        out.append((w @ vt_all[:, :end]).transpose(0, 1).numpy())
    return np.concatenate(out)


def test_correction_variants_against_dense():
    wl = make_config(2, seqlen=SEQLEN, alpha=ALPHA)
    orc = Oracle()
    q, k, v = wl.float_inputs()
    if OUTLIERS:
        parts = OUTLIERS.split(",")
        ch = np.random.default_rng(3).choice(wl.head_dim, int(parts[0]), replace=False)
        k = k.copy()
        k[:, :, ch] *= float(parts[1])
        if len(parts) > 2 and parts[2] == "both":
            q = q.copy()
            q[:, :, ch] *= float(parts[1])
    cu = wl.cu_seqlens
    tau = 1.0 / math.sqrt(wl.head_dim)
    qb = orc.block_means(q, cu, 128)
    kb = orc.block_means(k, cu, 128)
    vb = orc.block_means(v, cu, 128)
    kv = orc.block_vars(k, cu, 128, kb)
    est = orc.estimate(qb, kb, cu, 128, alpha=wl.alpha, tau=tau)
    nb = qb.shape[0]
    sel = np.sort(np.random.default_rng(5).choice(np.arange(8, nb), 6, replace=False))
    rows = np.concatenate([np.arange(i * 128, min(wl.total_tokens, (i + 1) * 128)) for i in sel])
    ref = _dense_rows(q, k, v, rows, wl.num_q_heads, wl.num_kv_heads, tau)
    ref_norm = np.linalg.norm(ref)
    err = {}
    # hybrid: per KV head, the 8 channels of largest total variance exact, the rest averaged
    top = np.argsort(-kv.sum(axis=0), axis=1)[:, :8]                  # [Hkv, 8]
    exact = np.zeros(kv.shape[1:], bool)
    exact[np.arange(kv.shape[1])[:, None], top] = True
    rest_mean = (kv * ~exact).sum(axis=2, keepdims=True) / (~exact).sum(axis=1)[None, :, None]
    kv_hybrid = np.where(exact[None], kv, rest_mean)
    for name, mode, kvar in (("none", 0, kv), ("mean", 1, kv), ("variance", 2, kv), ("pooled", 3, kv),
                             ("isotropic", 4, kv), ("hybrid8", 2, kv_hybrid)):
        r = orc.attend(q, k, v, cu, 128, tau, est["kept_cnt"], est["kept_idx"], correction=mode, kbar=kb,
                       vbar=vb, kvar=kvar, qbar=qb, sel=sel)
        err[name] = float(np.linalg.norm(r["o"][rows] - ref) / ref_norm)
    # strided estimate: query means over rows 0, 8, 16, ... of each block; in the
    # subsampled sequence a block is 128 / 8 rows
    stride = 8
    q_sub = np.ascontiguousarray(q[::stride])
    qb_sub = orc.block_means(q_sub, np.array([0, q_sub.shape[0]], np.int32), 128 // stride)
    assert qb_sub.shape == qb.shape
    est_s = orc.estimate(qb_sub, kb, cu, 128, alpha=wl.alpha, tau=tau, nb_max=est["nb_max"])
    r = orc.attend(q, k, v, cu, 128, tau, est_s["kept_cnt"], est_s["kept_idx"], correction=1, kbar=kb, vbar=vb,
                   sel=sel)
    err["strided"] = float(np.linalg.norm(r["o"][rows] - ref) / ref_norm)
    same = np.mean([set(est["kept_idx"][t, g, :est["kept_cnt"][t, g]].tolist())
                    == set(est_s["kept_idx"][t, g, :est_s["kept_cnt"][t, g]].tolist())
                    for t in range(nb) for g in range(wl.num_kv_heads)])
    density = est["kept_cnt"].sum() / (wl.num_kv_heads * nb * (nb + 1) / 2)
    print(f"\n{SEQLEN} tokens, alpha {wl.alpha}, outliers '{OUTLIERS}', kept density {density:.4f}, "
          f"q-blocks {sel.tolist()}: "
          + ", ".join(f"{k_} rel-L2 {v_:.4f}" for k_, v_ in err.items())
          + f"; strided: kept lists equal to the full estimate's {same:.3f}, kept density "
          f"{est_s['kept_cnt'].sum() / (wl.num_kv_heads * nb * (nb + 1) / 2):.4f}")
    assert err["variance"] < err["mean"] < err["none"], err
    assert err["isotropic"] < err["mean"], err
    assert err["strided"] < err["none"], err

"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each ``pin_*`` takes an ``oracle.oracle.Oracle`` and raises ``AssertionError``
on a mismatch.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on builds with one planted mistake and
requires that every mistake trips at least one pin.

What pins what (definitions D0-D4 in the oracle header):
  dense_sdpa        D3 core, D0 causality, LSE: alpha <= 0 equals
                    torch's scaled_dot_product_attention (fp64, GQA expanded)
  means_numpy       D1 block means (partial tail block) against numpy.mean
  bilinearity       D1 score = mean of the brute-force token logit block
  threshold_golden  D2 on hand-derived cases (tests/golden/threshold_cases.json)
  diagonal_kept     D2 forced diagonal
  nesting           D2 monotone in alpha
  weights_sum       D3 normalised weights (with correction) sum to one
  exact_correction  D3 correction is exact when K/V rows are constant per block
  gqa_packing       D2/D3 head -> group map: packed heads = each head alone
  ragged            D0 ragged batch (an empty request included) = each request alone
  e4m3_scales       D4 dequantisation: codes x power-of-two scale = scaled values
  chunk_dense_sdpa  D0 chunked form (the last Lq of Lk tokens), alpha <= 0: torch SDPA
                    with an explicit bottom-right causal mask
  chunk_equals_full D0 chunked form: a block-aligned chunk = the full prefill's rows
  chunk_bilinearity D0/D1 chunked form: a partial first q-block's score = mean logit
  chunk_exact_correction  D3 on chunks, the cached prefix's pruned blocks included
  variance_term     D3 variant 2: half the within-block logit variance (numpy) on
                    blocks with an exactly diagonal key covariance; block variances
  isotropic_variance_term  D3 variant 4 on Hadamard blocks (isotropic covariance)
  pooled_reduces_to_rows  D3 variant 3 = row-wise correction for block-constant q

``pin_near_threshold`` takes the mask comparison's band function
(``oracle.oracle.near_threshold``) instead of an oracle build: hand-derived
near / not-near flags (tests/golden/near_threshold_cases.json) on both sides of
the band, with |threshold| below and above one, and a GQA union where one head
of a group is near.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TAU = 1.0 / math.sqrt(128.0)


def _rand_inputs(seqlens, hq, hkv, d=128, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    T = int(sum(seqlens))
    q = (rng.standard_normal((T, hq, d)) * scale).astype(np.float32)
    k = (rng.standard_normal((T, hkv, d)) * scale).astype(np.float32)
    v = rng.standard_normal((T, hkv, d)).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    return q, k, v, cu


def _sdpa(q, k, v, cu, hq, hkv):
    """Dense causal attention per request with torch (fp64), GQA expanded."""
    g = hq // hkv
    outs, lses = [], []
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        qt = torch.from_numpy(q[s:e]).double().permute(1, 0, 2)
        kt = torch.from_numpy(k[s:e]).double().repeat_interleave(g, dim=1).permute(1, 0, 2)
        vt = torch.from_numpy(v[s:e]).double().repeat_interleave(g, dim=1).permute(1, 0, 2)
        o = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], is_causal=True,
                                                             scale=TAU)[0]
        logits = (qt @ kt.transpose(1, 2)) * TAU
        mask = torch.ones(e - s, e - s, dtype=torch.bool).tril()
        lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
        outs.append(o.permute(1, 0, 2).numpy())
        lses.append(lse.permute(1, 0).numpy())
    return np.concatenate(outs), np.concatenate(lses)


def _means(orc, q, k, v, cu, bs=128):
    return orc.block_means(q, cu, bs), orc.block_means(k, cu, bs), orc.block_means(v, cu, bs)


def pin_dense_sdpa(orc):
    lens = [1, 127, 129, 200, 383, 512]
    hq, hkv = 4, 2
    q, k, v, cu = _rand_inputs(lens, hq, hkv, seed=11)
    qb, kb, vb = _means(orc, q, k, v, cu)
    est = orc.estimate(qb, kb, cu, 128, alpha=0.0, tau=TAU)
    ref_o, ref_lse = _sdpa(q, k, v, cu, hq, hkv)
    for corr in (False, True):
        r = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=corr,
                       kbar=kb, vbar=vb)
        assert np.abs(r["o"] - ref_o).max() < 1e-12, "alpha<=0 output differs from dense SDPA"
        assert np.abs(r["lse"] - ref_lse).max() < 1e-12, "LSE differs from torch.logsumexp"


def pin_means_numpy(orc):
    lens = [1, 200, 383]
    q, k, v, cu = _rand_inputs(lens, 2, 1, seed=12)
    kb = orc.block_means(k, cu, 128)
    t = 0
    for b, L in enumerate(lens):
        for j in range((L + 127) // 128):
            rows = k[cu[b] + j * 128: cu[b] + min(L, (j + 1) * 128)].astype(np.float64)
            assert np.abs(kb[t] - rows.mean(axis=0)).max() < 1e-14, "block mean differs from numpy.mean"
            t += 1
    assert t == kb.shape[0]
    # scales multiply the stored values
    sc = np.array([0.25, 3.0])
    qb = orc.block_means(q, cu, 128, scale=sc)
    qb1 = orc.block_means(q, cu, 128)
    assert np.abs(qb - qb1 * sc[None, :, None]).max() < 1e-13


def pin_bilinearity(orc):
    lens = [383, 256]
    hq, hkv = 4, 2
    q, k, v, cu = _rand_inputs(lens, hq, hkv, seed=13)
    qb, kb, vb = _means(orc, q, k, v, cu)
    est = orc.estimate(qb, kb, cu, 128, alpha=0.1, tau=TAU, want_scores=True)
    s = est["s"]
    t0 = 0
    for b, L in enumerate(lens):
        nb = (L + 127) // 128
        qq = torch.from_numpy(q[cu[b]:cu[b + 1]]).double()
        kk = torch.from_numpy(k[cu[b]:cu[b + 1]]).double()
        for h in range(hq):
            g = h // (hq // hkv)
            logits = (qq[:, h, :] @ kk[:, g, :].T * TAU).numpy()
            for i in range(nb):
                for j in range(i + 1):
                    blk = logits[i * 128:min(L, (i + 1) * 128), j * 128:min(L, (j + 1) * 128)]
                    assert abs(s[t0 + i, h, j] - blk.mean()) < 1e-12, "score is not the mean block logit"
        t0 += nb


def _golden_case(c):
    L, hq, hkv = c["L"], c["Hq"], c["Hkv"]
    d = 128
    q = np.zeros((L, hq, d), np.float32)
    for h, ax in enumerate(c["qaxis"]):
        q[:, h, ax] = 8.0
    k = np.zeros((L, hkv, d), np.float32)
    for ax, coefs in c["coef"].items():
        for j, cval in enumerate(coefs):
            k[j * 128:min(L, (j + 1) * 128), :, int(ax)] = cval
    v = np.zeros((L, hkv, d), np.float32)
    cu = np.array([0, L], np.int32)
    return q, k, v, cu


def pin_threshold_golden(orc):
    with open(os.path.join(GOLDEN, "threshold_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v, cu = _golden_case(c)
        qb, kb, _ = _means(orc, q, k, v, cu)
        est = orc.estimate(qb, kb, cu, 128, alpha=c["alpha"], tau=TAU, want_scores=True)
        nb = len(c["kept"])
        for i in range(nb):
            for g in range(c["Hkv"]):
                got = list(est["kept_idx"][i, g, :est["kept_cnt"][i, g]])
                assert got == c["kept"][i][g], f"{c['name']}: q-block {i} kept {got}, expected {c['kept'][i][g]}"
        if "s_last_row" in c:
            assert np.abs(est["s"][nb - 1, 0, :nb] - np.array(c["s_last_row"])).max() < 1e-7


def _structured(seqlens, hq=4, hkv=2, seed=21, lam=7.5):
    from workloads import make_workload
    return make_workload(seqlens, hq, hkv, alpha=0.1, seed=seed, n_retrieval=2, lam=lam)


def pin_diagonal_kept(orc):
    wl = _structured([1000, 640])
    q, k, v = wl.float_inputs()
    cu = wl.cu_seqlens
    qb, kb, _ = _means(orc, q, k, v, cu)
    for a in (0.5, 1.0):
        est = orc.estimate(qb, kb, cu, 128, alpha=a, tau=TAU)
        t = 0
        for L in wl.seqlens:
            for i in range((L + 127) // 128):
                for g in range(wl.num_kv_heads):
                    c = est["kept_cnt"][t, g]
                    assert c >= 1 and est["kept_idx"][t, g, c - 1] == i, "diagonal block not kept"
                t += 1


def pin_nesting(orc):
    wl = _structured([2048])
    q, k, v = wl.float_inputs()
    cu = wl.cu_seqlens
    qb, kb, _ = _means(orc, q, k, v, cu)
    prev = None
    for a in (0.02, 0.05, 0.1, 0.2, 0.5):
        est = orc.estimate(qb, kb, cu, 128, alpha=a, tau=TAU)
        sets = [[set(est["kept_idx"][i, g, :est["kept_cnt"][i, g]]) for g in range(2)] for i in range(16)]
        if prev is not None:
            for i in range(16):
                for g in range(2):
                    assert sets[i][g] <= prev[i][g], "kept set grew when alpha grew"
        prev = sets


def pin_weights_sum(orc):
    wl = _structured([1024])
    q, k, v = wl.float_inputs()
    cu = wl.cu_seqlens
    qb, kb, vb = _means(orc, q, k, v, cu)
    est = orc.estimate(qb, kb, cu, 128, alpha=0.3, tau=TAU)
    assert (est["kept_cnt"][1:] < np.arange(2, 9)[:, None]).any(), "case prunes nothing"
    r = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=True, kbar=kb,
                   vbar=vb, want_wsum=True)
    assert np.abs(r["wsum"] - 1.0).max() < 1e-12, "softmax weights do not sum to one"


def pin_exact_correction(orc):
    """K and V rows constant inside every block: replacing a pruned block by n_j
    copies of its mean key/value is then exact, so the corrected sparse output
    equals dense attention for any alpha."""
    lens = [1024, 700]
    hq, hkv = 4, 2
    rng = np.random.default_rng(31)
    T = sum(lens)
    # a shared query direction spreads the block scores so that alpha prunes
    q = (rng.standard_normal((T, hq, 128)) + rng.standard_normal((1, hq, 128))).astype(np.float32)
    k = np.zeros((T, hkv, 128), np.float32)
    v = np.zeros((T, hkv, 128), np.float32)
    cu = np.array([0, lens[0], T], np.int32)
    for b, L in enumerate(lens):
        for j in range((L + 127) // 128):
            s, e = cu[b] + j * 128, cu[b] + min(L, (j + 1) * 128)
            k[s:e] = (rng.standard_normal((hkv, 128)) * 1.5).astype(np.float32)
            v[s:e] = rng.standard_normal((hkv, 128)).astype(np.float32)
    qb, kb, vb = _means(orc, q, k, v, cu)
    ref_o, ref_lse = _sdpa(q, k, v, cu, hq, hkv)
    for a in (0.3, 0.9):
        est = orc.estimate(qb, kb, cu, 128, alpha=a, tau=TAU)
        full = np.array([min(i, 7) + 1 for i in range(8)] + [i + 1 for i in range(6)])
        assert (est["kept_cnt"].min(axis=1) < full).any(), "case prunes nothing"
        r = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=True, kbar=kb, vbar=vb)
        assert np.abs(r["o"] - ref_o).max() < 1e-11, "mean correction is not exact on block-constant K/V"
        assert np.abs(r["lse"] - ref_lse).max() < 1e-11
        r0 = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=False)
        assert np.abs(r0["o"] - ref_o).max() > 1e-3, "pruning had no effect"


def pin_gqa_packing(orc):
    wl = _structured([900], hq=4, hkv=2, seed=41)
    q, k, v = wl.float_inputs()
    cu = wl.cu_seqlens
    qb, kb, vb = _means(orc, q, k, v, cu)
    est = orc.estimate(qb, kb, cu, 128, alpha=0.2, tau=TAU)
    packed = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=True, kbar=kb, vbar=vb)
    for h in range(4):
        g = h // 2
        one = orc.attend(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1], cu, 128, TAU,
                         est["kept_cnt"][:, g:g + 1], est["kept_idx"][:, g:g + 1], correction=True,
                         kbar=kb[:, g:g + 1], vbar=vb[:, g:g + 1])
        assert np.abs(one["o"][:, 0] - packed["o"][:, h]).max() == 0.0, "packed head differs from head alone"
    # the group list is the union of the per-head lists
    for h in range(4):
        g = h // 2
        alone = orc.estimate(qb[:, h:h + 1], kb[:, g:g + 1], cu, 128, alpha=0.2, tau=TAU)
        for i in range(qb.shape[0]):
            sh = set(alone["kept_idx"][i, 0, :alone["kept_cnt"][i, 0]])
            sg = set(est["kept_idx"][i, g, :est["kept_cnt"][i, g]])
            assert sh <= sg, "group list misses a head's block"


def pin_ragged(orc):
    lens = [300, 0, 1, 520]                          # an empty request among them
    wl = _structured(lens, seed=51)
    q, k, v = wl.float_inputs()
    cu = wl.cu_seqlens
    qb, kb, vb = _means(orc, q, k, v, cu)
    est = orc.estimate(qb, kb, cu, 128, alpha=0.2, tau=TAU)
    full = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=True, kbar=kb, vbar=vb)
    t0 = 0
    for b, L in enumerate(lens):
        s, e = int(cu[b]), int(cu[b + 1])
        cu1 = np.array([0, L], np.int32)
        qb1, kb1, vb1 = _means(orc, q[s:e], k[s:e], v[s:e], cu1)
        e1 = orc.estimate(qb1, kb1, cu1, 128, alpha=0.2, tau=TAU, nb_max=est["nb_max"])
        nb = (L + 127) // 128
        assert e1["kept_cnt"].shape[0] == nb
        assert (e1["kept_cnt"] == est["kept_cnt"][t0:t0 + nb]).all()
        r1 = orc.attend(q[s:e], k[s:e], v[s:e], cu1, 128, TAU, e1["kept_cnt"], e1["kept_idx"], correction=True,
                        kbar=kb1, vbar=vb1)
        assert r1["o"].shape[0] == L
        assert np.array_equal(r1["o"], full["o"][s:e]), "request in a batch differs from request alone"
        t0 += nb
    assert t0 == est["kept_cnt"].shape[0]


def pin_e4m3_scales(orc):
    lens = [500]
    hq, hkv = 4, 2
    rng = np.random.default_rng(61)
    codes = [torch.from_numpy(rng.standard_normal((500, h, 128)).astype(np.float32) * 40).to(torch.float8_e4m3fn).float().numpy()
             for h in (hq, hkv, hkv)]
    q8, k8, v8 = codes
    cu = np.array([0, 500], np.int32)
    qs = np.array([2.0 ** -6, 2.0 ** -5, 2.0 ** -7, 2.0 ** -6])
    ks = np.array([2.0 ** -5, 2.0 ** -6])
    vs = np.array([2.0 ** -4, 2.0 ** -3])
    qsc, ksc, vsc = (q8 * qs[None, :, None]).astype(np.float32), (k8 * ks[None, :, None]).astype(np.float32), \
        (v8 * vs[None, :, None]).astype(np.float32)
    qb = orc.block_means(q8, cu, 128, qs)
    kb = orc.block_means(k8, cu, 128, ks)
    vb = orc.block_means(v8, cu, 128, vs)
    est = orc.estimate(qb, kb, cu, 128, alpha=0.3, tau=TAU)
    a = orc.attend(q8, k8, v8, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=True, kbar=kb, vbar=vb,
                   q_scale=qs, k_scale=ks, v_scale=vs)
    qb2, kb2, vb2 = _means(orc, qsc, ksc, vsc, cu)
    est2 = orc.estimate(qb2, kb2, cu, 128, alpha=0.3, tau=TAU)
    assert (est2["kept_cnt"] == est["kept_cnt"]).all()
    b = orc.attend(qsc, ksc, vsc, cu, 128, TAU, est2["kept_cnt"], est2["kept_idx"], correction=True,
                   kbar=kb2, vbar=vb2)
    assert np.abs(a["o"] - b["o"]).max() < 1e-12, "e4m3 dequantisation differs from scaled values"


# ---------------------------------------------------------------------------
# chunked prefill (D0 chunked form): the last Lq_b of Lk_b tokens are the
# queries, at positions P_b = Lk_b - Lq_b onwards; q-blocks keep the absolute
# grid of the request
# ---------------------------------------------------------------------------
def _chunk_of(q_full, cu_k, lq):
    """The query rows of a chunk: the last lq[b] rows of every request."""
    parts = [q_full[int(cu_k[b + 1]) - n:int(cu_k[b + 1])] for b, n in enumerate(lq)]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    return np.ascontiguousarray(np.concatenate(parts)), cu_q


def _chunk_means(orc, q, k, v, cu_q, cu_k):
    from oracle.oracle import chunk_starts
    p0 = chunk_starts(cu_q, cu_k)
    return (orc.block_means(q, cu_q, 128, pos0=p0), orc.block_means(k, cu_k, 128),
            orc.block_means(v, cu_k, 128), p0)


def _sdpa_chunk(q, k, v, cu_q, cu_k, hq, hkv):
    """Dense attention of the chunk rows with torch (fp64), GQA expanded: query t
    of request b sits at position P_b + t and sees keys c <= P_b + t (an
    explicit boolean mask, since torch's is_causal aligns the mask top-left)."""
    g = hq // hkv
    outs, lses = [], []
    for b in range(len(cu_q) - 1):
        qs_, qe, ks_, ke = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        lq, lk = qe - qs_, ke - ks_
        if lq == 0:
            continue
        mask = torch.arange(lk)[None, :] <= (lk - lq + torch.arange(lq))[:, None]
        qt = torch.from_numpy(q[qs_:qe]).double().permute(1, 0, 2)
        kt = torch.from_numpy(k[ks_:ke]).double().repeat_interleave(g, dim=1).permute(1, 0, 2)
        vt = torch.from_numpy(v[ks_:ke]).double().repeat_interleave(g, dim=1).permute(1, 0, 2)
        o = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None], attn_mask=mask,
                                                             scale=TAU)[0]
        logits = (qt @ kt.transpose(1, 2)) * TAU
        lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
        outs.append(o.permute(1, 0, 2).numpy())
        lses.append(lse.permute(1, 0).numpy())
    return np.concatenate(outs), np.concatenate(lses)


def _prefix_pruned(est, p0, lq, lk, hkv):
    """True when some q-block of a chunk drops a key block of the cached prefix."""
    t = 0
    for b in range(len(lq)):
        if lq[b] == 0:
            continue
        i0 = int(p0[b]) // 128
        for i in range(i0, (lk[b] + 127) // 128):
            for g in range(hkv):
                kept = set(est["kept_idx"][t, g, :est["kept_cnt"][t, g]].tolist())
                if any(j not in kept for j in range(i0)):
                    return True
            t += 1
    return False


def pin_chunk_dense_sdpa(orc):
    lk = [700, 700, 129, 256, 383, 300, 700]
    lq = [700, 572, 1, 0, 255, 299, 500]      # P = 0, 128, 128, -, 128, 1, 200
    hq, hkv = 4, 2
    q_full, k, v, cu_k = _rand_inputs(lk, hq, hkv, seed=71)
    q, cu_q = _chunk_of(q_full, cu_k, lq)
    qb, kb, vb, p0 = _chunk_means(orc, q, k, v, cu_q, cu_k)
    est = orc.estimate(qb, kb, cu_q, 128, alpha=0.0, tau=TAU, cu_seqlens_k=cu_k)
    ref_o, ref_lse = _sdpa_chunk(q, k, v, cu_q, cu_k, hq, hkv)
    for corr in (False, True):
        r = orc.attend(q, k, v, cu_q, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=corr,
                       kbar=kb, vbar=vb, cu_seqlens_k=cu_k)
        assert np.abs(r["o"] - ref_o).max() < 1e-12, "chunk output differs from dense masked SDPA"
        assert np.abs(r["lse"] - ref_lse).max() < 1e-12, "chunk LSE differs from torch.logsumexp"


def pin_chunk_equals_full(orc):
    """A chunk that starts on a block boundary has the full prefill's q-blocks, so
    its block means, kept lists, outputs and LSE are the full prefill's rows."""
    lk = [1000, 640, 385]
    lq = [744, 256, 385]                      # P = 256, 384, 0
    wl = _structured(lk, seed=81)
    q_full, k, v = wl.float_inputs()
    cu_k = wl.cu_seqlens
    q, cu_q = _chunk_of(q_full, cu_k, lq)
    qb, kb, vb, p0 = _chunk_means(orc, q, k, v, cu_q, cu_k)
    assert (p0 % 128 == 0).all()
    qb_full = orc.block_means(q_full, cu_k, 128)
    ef = orc.estimate(qb_full, kb, cu_k, 128, alpha=0.2, tau=TAU)
    ec = orc.estimate(qb, kb, cu_q, 128, alpha=0.2, tau=TAU, cu_seqlens_k=cu_k, nb_max=ef["nb_max"])
    assert _prefix_pruned(ec, p0, lq, lk, 2), "case prunes no prefix block"
    full = orc.attend(q_full, k, v, cu_k, 128, TAU, ef["kept_cnt"], ef["kept_idx"], correction=True,
                      kbar=kb, vbar=vb)
    ch = orc.attend(q, k, v, cu_q, 128, TAU, ec["kept_cnt"], ec["kept_idx"], correction=True, kbar=kb,
                    vbar=vb, cu_seqlens_k=cu_k)
    tf = tc = 0
    for b in range(len(lk)):
        nbk, i0 = (lk[b] + 127) // 128, int(p0[b]) // 128
        n = nbk - i0
        for key, a, c in (("qbar", qb_full, qb), ("kept_cnt", ef["kept_cnt"], ec["kept_cnt"]),
                          ("kept_idx", ef["kept_idx"], ec["kept_idx"])):
            assert np.array_equal(c[tc:tc + n], a[tf + i0:tf + nbk]), f"chunk {key} differs from full prefill"
        rows_f = slice(int(cu_k[b]) + int(p0[b]), int(cu_k[b + 1]))
        rows_c = slice(int(cu_q[b]), int(cu_q[b + 1]))
        assert np.array_equal(ch["o"][rows_c], full["o"][rows_f]), "chunk rows differ from full prefill"
        assert np.array_equal(ch["lse"][rows_c], full["lse"][rows_f])
        tf += nbk
        tc += n


def pin_chunk_bilinearity(orc):
    """Chunks whose first q-block is partial: the block score is the mean token
    logit over the query rows that block holds and every key of block j."""
    lk = [700, 300]
    lq = [500, 45]                            # P = 200 (56 rows in block 1), 255 (1 row in block 1)
    hq, hkv = 4, 2
    q_full, k, v, cu_k = _rand_inputs(lk, hq, hkv, seed=91)
    q, cu_q = _chunk_of(q_full, cu_k, lq)
    qb, kb, vb, p0 = _chunk_means(orc, q, k, v, cu_q, cu_k)
    est = orc.estimate(qb, kb, cu_q, 128, alpha=0.1, tau=TAU, cu_seqlens_k=cu_k, want_scores=True)
    s = est["s"]
    t = 0
    for b in range(len(lk)):
        P, L = int(p0[b]), lk[b]
        qq = torch.from_numpy(q[cu_q[b]:cu_q[b + 1]]).double()
        kk = torch.from_numpy(k[cu_k[b]:cu_k[b + 1]]).double()
        for i in range(P // 128, (L + 127) // 128):
            lo, hi = max(P, i * 128), min(L, (i + 1) * 128)
            for h in range(hq):
                g = h // (hq // hkv)
                logits = (qq[lo - P:hi - P, h, :] @ kk[:, g, :].T * TAU).numpy()
                for j in range(i + 1):
                    blk = logits[:, j * 128:min(L, (j + 1) * 128)]
                    assert abs(s[t, h, j] - blk.mean()) < 1e-12, "chunk score is not the mean block logit"
            t += 1
    assert t == s.shape[0]


def pin_chunk_exact_correction(orc):
    """Block-constant K and V under chunks: the corrected output equals dense
    attention with the bottom-right causal mask for any alpha, the pruned
    blocks of the cached prefix included."""
    lk = [1024, 700]
    lq = [600, 572]                           # P = 424 (unaligned), 128
    hq, hkv = 4, 2
    rng = np.random.default_rng(101)
    T = sum(lk)
    q_full = (rng.standard_normal((T, hq, 128)) + rng.standard_normal((1, hq, 128))).astype(np.float32)
    k = np.zeros((T, hkv, 128), np.float32)
    v = np.zeros((T, hkv, 128), np.float32)
    cu_k = np.array([0, lk[0], T], np.int32)
    for b, L in enumerate(lk):
        for j in range((L + 127) // 128):
            s0, e0 = cu_k[b] + j * 128, cu_k[b] + min(L, (j + 1) * 128)
            k[s0:e0] = (rng.standard_normal((hkv, 128)) * 1.5).astype(np.float32)
            v[s0:e0] = rng.standard_normal((hkv, 128)).astype(np.float32)
    q, cu_q = _chunk_of(q_full, cu_k, lq)
    qb, kb, vb, p0 = _chunk_means(orc, q, k, v, cu_q, cu_k)
    ref_o, ref_lse = _sdpa_chunk(q, k, v, cu_q, cu_k, hq, hkv)
    for a in (0.3, 0.9):
        est = orc.estimate(qb, kb, cu_q, 128, alpha=a, tau=TAU, cu_seqlens_k=cu_k)
        assert _prefix_pruned(est, p0, lq, lk, hkv), "case prunes no prefix block"
        r = orc.attend(q, k, v, cu_q, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=True, kbar=kb,
                       vbar=vb, cu_seqlens_k=cu_k)
        assert np.abs(r["o"] - ref_o).max() < 1e-11, "chunk mean correction is not exact on block-constant K/V"
        assert np.abs(r["lse"] - ref_lse).max() < 1e-11
        r0 = orc.attend(q, k, v, cu_q, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=False,
                        cu_seqlens_k=cu_k)
        assert np.abs(r0["o"] - ref_o).max() > 1e-3, "pruning had no effect"


# ---------------------------------------------------------------------------
# D3 variants (approximation studies): variance term and block-pooled logits
# ---------------------------------------------------------------------------
def pin_variance_term(orc):
    """Correction mode 2 adds half the within-block logit variance to each pruned
    block's logit.  Key blocks built as the block mean plus axis-aligned +/- pairs
    have an exactly diagonal covariance, so the per-dimension formula must equal
    the variance of the actual token logits (numpy); the check goes through the
    LSE of rows whose only kept block is the diagonal.  Block variances are also
    checked against numpy.var."""
    L, hq, hkv, d = 640, 2, 1, 128
    rng = np.random.default_rng(111)
    q = (rng.integers(-16, 17, (L, hq, d)) / 16.0).astype(np.float32)
    k = np.zeros((L, hkv, d), np.float32)
    v = rng.standard_normal((L, hkv, d)).astype(np.float32)
    for j in range(L // 128):
        mean = rng.integers(-8, 9, (hkv, d)) / 16.0
        blk = np.repeat(mean[None], 128, axis=0)
        if j != 2:                                   # block 2 stays constant: zero variance
            for t in range(64):
                axis, amp = rng.integers(0, d), rng.integers(1, 17) / 16.0
                blk[2 * t, :, axis] += amp
                blk[2 * t + 1, :, axis] -= amp
        k[j * 128:(j + 1) * 128] = blk.astype(np.float32)
    cu = np.array([0, L], np.int32)
    qb, kb, vb = _means(orc, q, k, v, cu)
    kv = orc.block_vars(k, cu, 128, kb)
    for j in range(L // 128):
        assert np.abs(kv[j] - k[j * 128:(j + 1) * 128].astype(np.float64).var(axis=0)).max() < 1e-14
    nb = L // 128
    cnt = np.ones((nb, hkv), np.int32)
    idx = np.full((nb, hkv, nb), -1, np.int32)
    idx[np.arange(nb), 0, 0] = np.arange(nb)           # only the diagonal block kept
    r = orc.attend(q, k, v, cu, 128, TAU, cnt, idx, correction=2, kbar=kb, vbar=vb, kvar=kv)
    kk = k.astype(np.float64)
    for row in (130, 300, 511, 639):
        i = row // 128
        for h in range(hq):
            qr = q[row, h].astype(np.float64)
            logits = TAU * (kk[:, 0] @ qr)
            den = np.exp(logits[i * 128:row + 1]).sum()
            for j in range(i):
                lj = logits[j * 128:(j + 1) * 128]
                den += 128 * math.exp(lj.mean() + 0.5 * lj.var())
            assert abs(r["lse"][row, h] - math.log(den)) < 1e-12, "variance term differs from the logit variance"


def pin_isotropic_variance_term(orc):
    """Correction mode 4 (the variance averaged over the key dimensions) on key
    blocks with an exactly isotropic covariance: block mean plus a_j times
    columns 1..64 of a 128x128 Hadamard matrix (zero column sums, orthogonal
    columns; d = 64).  It must equal half the numpy variance of the token logits,
    and mode 2 on the same blocks."""
    L, hq, hkv, d = 640, 2, 1, 64
    rng = np.random.default_rng(131)
    h = np.array([[1.0]])
    while h.shape[0] < 128:
        h = np.block([[h, h], [h, -h]])
    dev = h[:, 1:d + 1]                               # [128, 64], columns sum to 0
    q = (rng.integers(-16, 17, (L, hq, d)) / 16.0).astype(np.float32)
    k = np.zeros((L, hkv, d), np.float32)
    v = rng.standard_normal((L, hkv, d)).astype(np.float32)
    for j in range(L // 128):
        mean = rng.integers(-8, 9, (hkv, d)) / 16.0
        amp = 0.0 if j == 1 else rng.integers(1, 17) / 16.0
        k[j * 128:(j + 1) * 128] = (mean[None] + amp * dev[:, None, :]).astype(np.float32)
    cu = np.array([0, L], np.int32)
    qb, kb, vb = _means(orc, q, k, v, cu)
    kv = orc.block_vars(k, cu, 128, kb)
    nb = L // 128
    cnt = np.ones((nb, hkv), np.int32)
    idx = np.full((nb, hkv, nb), -1, np.int32)
    idx[np.arange(nb), 0, 0] = np.arange(nb)           # only the diagonal block kept
    r4 = orc.attend(q, k, v, cu, 128, TAU, cnt, idx, correction=4, kbar=kb, vbar=vb, kvar=kv)
    r2 = orc.attend(q, k, v, cu, 128, TAU, cnt, idx, correction=2, kbar=kb, vbar=vb, kvar=kv)
    assert np.isfinite(r4["lse"]).all() and np.isfinite(r2["lse"]).all(), "non-finite LSE"
    assert np.abs(r4["lse"] - r2["lse"]).max() < 1e-12, "isotropic blocks: mode 4 != mode 2"
    kk = k.astype(np.float64)
    for row in (130, 300, 511, 639):
        i = row // 128
        for hh in range(hq):
            logits = TAU * (kk[:, 0] @ q[row, hh].astype(np.float64))
            den = np.exp(logits[i * 128:row + 1]).sum()
            for j in range(i):
                lj = logits[j * 128:(j + 1) * 128]
                den += 128 * math.exp(lj.mean() + 0.5 * lj.var())
            assert abs(r4["lse"][row, hh] - math.log(den)) < 1e-12, "mode 4 differs from the logit variance"


def pin_pooled_reduces_to_rows(orc):
    """Correction mode 3 (block-pooled logits) equals the row-wise correction when
    every row of a q-block equals the block's mean query."""
    wl = _structured([700], seed=121)
    q, k, v = wl.float_inputs()
    q = np.repeat(q[::128], 128, axis=0)[:700]       # rows constant inside each q-block
    cu = wl.cu_seqlens
    qb, kb, vb = _means(orc, q, k, v, cu)
    est = orc.estimate(qb, kb, cu, 128, alpha=0.3, tau=TAU)
    a = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=1, kbar=kb, vbar=vb)
    b = orc.attend(q, k, v, cu, 128, TAU, est["kept_cnt"], est["kept_idx"], correction=3, kbar=kb, vbar=vb,
                   qbar=qb)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["lse"], b["lse"]), "pooled != row-wise"


def pin_near_threshold(fn):
    """``fn(s, m, Hkv, alpha, None, rel)`` against the hand-derived flags of
    tests/golden/near_threshold_cases.json; alpha <= 0 (nothing pruned) has no
    near-threshold block."""
    with open(os.path.join(GOLDEN, "near_threshold_cases.json")) as f:
        c = json.load(f)
    s = np.array([[[np.nan if x is None else x for x in row] for row in blk] for blk in c["s"]], np.float64)
    m = np.array(c["m"], np.float64)
    want = np.array(c["near"], bool)
    got = np.asarray(fn(s, m, c["num_kv_heads"], c["alpha"], None, c["rel"]))
    assert got.shape == want.shape, f"near-threshold flags of shape {got.shape}, expected {want.shape}"
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"near-threshold flags differ at (q-block, KV head, key block) {bad.tolist()}"
    none = np.asarray(fn(s, m, c["num_kv_heads"], 0.0, None, c["rel"]))
    assert not none.any(), "alpha <= 0 prunes nothing, so no block can be near the threshold"


ALL_PINS = [pin_dense_sdpa, pin_means_numpy, pin_bilinearity, pin_threshold_golden, pin_diagonal_kept,
            pin_nesting, pin_weights_sum, pin_exact_correction, pin_gqa_packing, pin_ragged, pin_e4m3_scales,
            pin_chunk_dense_sdpa, pin_chunk_equals_full, pin_chunk_bilinearity, pin_chunk_exact_correction,
            pin_variance_term, pin_isotropic_variance_term, pin_pooled_reduces_to_rows]

"""GPU (sm_100a) path against the CPU oracle, through the C ABI.

Masks: bit-exact except at blocks whose oracle score lies within 1e-3
(relative) of the threshold.  Outputs, given the GPU's mask (the oracle is
re-run with it): bf16 max-abs 2e-2 and mean-abs 2e-3, e4m3 max-abs 6e-2 and
mean-abs 6e-3 (the mean-abs bound is ours: the bf16 bounds' ratio).
LSE (natural log): max-abs 2e-2 for bf16 and 6e-2 for e4m3 (the attention
weights are rounded to the MMA precision before the PV product).
"""
import os

import numpy as np
import pytest
import torch

from gpu_helpers import (BF16_MAX_ABS, BF16_MEAN_ABS, E4M3_MAX_ABS, E4M3_MEAN_ABS, check_mask_counts,
                         compare_masks, oracle, out_errors, record_output_errors, rows_of_blocks, run_gpu,
                         sample_blocks, sample_blocks_per_request, tau)
from workloads import make_config, make_workload

pytestmark = pytest.mark.gpu


def _kept(g):
    return {"kept_cnt": g["kept_cnt"], "kept_idx": g["kept_idx"]}


def _check_outputs(wl, g, correction, sel=None, max_abs=BF16_MAX_ABS, mean_abs=BF16_MEAN_ABS, lse_abs=2e-2):
    orc = oracle()
    ref = orc.run(wl, kept=_kept(g), correction=correction, sel=sel)
    rows = None if sel is None else rows_of_blocks(wl.cu_seqlens, sel)
    mx, mn = out_errors(g["o"], ref["o"], rows)
    record_output_errors(os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], mx, mn)
    assert mx <= max_abs and mn <= mean_abs, f"output max-abs {mx:.3e} mean-abs {mn:.3e}"
    if g["lse"] is not None:
        lm, _ = out_errors(g["lse"], ref["lse"], rows)
        assert lm < lse_abs, f"lse max-abs {lm:.3e}"
    return mx, mn


def _check_masks(wl, g, alpha=None):
    orc = oracle()
    a = wl.alpha if alpha is None else alpha
    est = orc.run(wl, alpha=a, want_scores=True, sel=np.zeros(0, np.int64))
    check_mask_counts(compare_masks(g, est, a, wl.num_kv_heads, wl.cu_seqlens,
                                    label=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]))
    # block means
    assert np.abs(g["k_mean"] - est["kbar"]).max() < 1e-4 * max(1.0, np.abs(est["kbar"]).max())
    return est


@pytest.mark.parametrize("correction", [True, False])
def test_tiny_config(correction):
    wl = make_config(0)
    g = run_gpu(wl, correction=correction)
    _check_masks(wl, g)
    _check_outputs(wl, g, correction)


@pytest.mark.parametrize("paged", [False, True])
def test_empty_requests_in_a_batch(paged):
    """Empty requests first, in the middle and last get no blocks; the others
    match the oracle as in any ragged batch."""
    wl = make_workload([0, 300, 0, 200, 129, 0], 8, 2, alpha=0.1, seed=17, n_retrieval=1, paged=paged)
    g = run_gpu(wl, paged=paged)
    _check_masks(wl, g)
    _check_outputs(wl, g, True)


def test_all_requests_empty():
    """total_tokens == 0: the call checks cu_seqlens, writes nothing and reports no error."""
    wl = make_workload([0, 0], 4, 2, alpha=0.1, seed=18)
    g = run_gpu(wl)
    assert g["o"].shape[0] == 0 and g["kept_cnt"].shape[0] == 0


def test_dense_alpha_zero():
    wl = make_workload([1000, 300], 4, 2, alpha=0.0, seed=3)
    g = run_gpu(wl, alpha=0.0)
    nb = [(L + 127) // 128 for L in wl.seqlens]
    full = np.concatenate([np.arange(1, n + 1) for n in nb])
    assert (g["kept_cnt"] == full[:, None]).all(), "alpha <= 0 must keep every causal block"
    _check_outputs(wl, g, True)


@pytest.mark.parametrize("G", [1, 2, 3, 4])
def test_ragged_edges(G):
    wl = make_workload([1, 127, 129, 200, 383, 700], 2 * G, 2, alpha=0.2, seed=10 + G, n_retrieval=1)
    g = run_gpu(wl)
    _check_masks(wl, g)
    _check_outputs(wl, g, True)


def test_llama_shape_4k():
    wl = make_config(1, seqlen=4096)
    g = run_gpu(wl, scores=True)
    est = _check_masks(wl, g)
    _check_outputs(wl, g, True)
    # score_dbg = s - m
    s_rel = est["s"] - est["m"][:, :, None]
    m = ~np.isnan(s_rel)
    assert np.abs(g["score_dbg"][m] - s_rel[m]).max() < 1e-3


@pytest.mark.parametrize("alpha", [0.02, 0.05, 0.1, 0.2])
def test_llama_shape_32k_sweep(alpha):
    wl = make_config(1, alpha=alpha)
    g = run_gpu(wl)
    _check_masks(wl, g)
    nblk = g["kept_cnt"].shape[0]
    sel = sample_blocks(nblk, 32, seed=int(alpha * 1000), include=(0, nblk - 1))
    _check_outputs(wl, g, True, sel=sel)


def test_128k_bf16_sampled():
    wl = make_config(2)
    g = run_gpu(wl)
    _check_masks(wl, g)
    nblk = g["kept_cnt"].shape[0]
    sel = sample_blocks(nblk, 64, seed=2, include=(0, nblk - 1))
    _check_outputs(wl, g, True, sel=sel)


def test_e4m3_4k():
    wl = make_config(3, seqlen=4096)
    g = run_gpu(wl)
    _check_masks(wl, g)
    _check_outputs(wl, g, True, max_abs=E4M3_MAX_ABS, mean_abs=E4M3_MEAN_ABS, lse_abs=E4M3_MAX_ABS)


def test_128k_e4m3_sampled():
    wl = make_config(3)
    g = run_gpu(wl)
    _check_masks(wl, g)
    nblk = g["kept_cnt"].shape[0]
    sel = sample_blocks(nblk, 64, seed=3, include=(0, nblk - 1))
    _check_outputs(wl, g, True, sel=sel, max_abs=E4M3_MAX_ABS, mean_abs=E4M3_MEAN_ABS, lse_abs=E4M3_MAX_ABS)


def test_paged_equals_contiguous_small():
    wl = make_workload([900, 130, 2000, 1], 8, 2, alpha=0.1, seed=41, paged=True)
    gp = run_gpu(wl, paged=True)
    gc = run_gpu(wl, paged=False)
    assert (gp["kept_cnt"] == gc["kept_cnt"]).all() and (gp["kept_idx"] == gc["kept_idx"]).all()
    assert np.array_equal(gp["o"], gc["o"], equal_nan=True), "paged output differs from contiguous"
    _check_outputs(wl, gp, True)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_output_16_byte_aligned(dtype):
    """An output that is 16- but not 32-byte aligned (the ABI's minimum) takes the
    epilogue's 128-bit stores; it holds the same bytes as a 32-byte aligned one."""
    wl = make_workload([900, 130, 2000, 1], 8, 2, alpha=0.1, seed=43, dtype=dtype)
    g16 = run_gpu(wl, out_shift=8)
    g32 = run_gpu(wl, out_shift=0)
    assert np.array_equal(g16["o"], g32["o"], equal_nan=True), "output depends on its alignment"
    assert np.array_equal(g16["lse"], g32["lse"], equal_nan=True)
    if dtype == "bf16":
        _check_outputs(wl, g16, True)
    else:
        _check_outputs(wl, g16, True, max_abs=E4M3_MAX_ABS, mean_abs=E4M3_MEAN_ABS, lse_abs=E4M3_MAX_ABS)


def test_e4m3_paged_equals_contiguous():
    """e4m3 page pools (the pooling kernel's byte-wide TMA boxes over pages) give the masks
    and the output of the contiguous e4m3 path, which matches the oracle."""
    wl = make_workload([900, 130, 2000, 1], 8, 2, alpha=0.1, seed=42, dtype="e4m3", paged=True)
    gp = run_gpu(wl, paged=True)
    gc = run_gpu(wl, paged=False)
    assert (gp["kept_cnt"] == gc["kept_cnt"]).all() and (gp["kept_idx"] == gc["kept_idx"]).all()
    assert np.array_equal(gp["o"], gc["o"], equal_nan=True), "paged output differs from contiguous"
    _check_masks(wl, gp)
    _check_outputs(wl, gp, True, max_abs=E4M3_MAX_ABS, mean_abs=E4M3_MEAN_ABS, lse_abs=E4M3_MAX_ABS)


def test_partial_column_slabs_g5():
    """Hq = 20: the query heads span three 8-head pooling slabs, the last one half outside
    the tensor (zero-filled TMA box columns); G = 5 gives work items with one Q tile and a
    score tile of 25 q-blocks whose G rows meet in shared memory."""
    wl = make_workload([700, 300, 129], 20, 4, alpha=0.1, seed=13, n_retrieval=1)
    g = run_gpu(wl)
    _check_masks(wl, g)
    _check_outputs(wl, g, True)


def test_paged_ragged_batch_sampled():
    wl = make_config(4, seqlen=32768)
    g = run_gpu(wl, paged=True)
    _check_masks(wl, g)
    nblk = g["kept_cnt"].shape[0]
    sel = sample_blocks(nblk, 16, seed=4, include=(0, nblk - 1))
    _check_outputs(wl, g, True, sel=sel)


def test_paged_ragged_batch_full_size():
    """The paged continuous batch at its stated size: 8 requests with lengths drawn
    log-uniform in [4096, 131072] (this seed: 4108 .. 74526 tokens, 177104 in all), pool
    pages in a seeded random order.  Every kept list against the oracle; outputs on 16
    seeded q-blocks of every request, its first and last included."""
    wl = make_config(4)
    g = run_gpu(wl, paged=True)
    _check_masks(wl, g)
    sel = sample_blocks_per_request(wl.cu_seqlens, 16, seed=44)
    _check_outputs(wl, g, True, sel=sel)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_paged_attention_on_the_oracle_mask(dtype):
    """fp2_prefill_paged on kept lists given by the caller (here the oracle's): the output
    matches the oracle on the same lists, and the contiguous call on the same lists."""
    wl = make_workload([900, 130, 2000, 1, 385], 8, 2, alpha=0.1, seed=45, dtype=dtype, paged=True)
    est = oracle().run(wl, want_scores=False, sel=np.zeros(0, np.int64))
    kept = {"kept_cnt": est["kept_cnt"], "kept_idx": est["kept_idx"]}
    gp = run_gpu(wl, paged=True, kept=kept)
    gc = run_gpu(wl, paged=False, kept=kept)
    assert (gp["kept_cnt"] == est["kept_cnt"]).all()
    assert np.array_equal(gp["o"], gc["o"], equal_nan=True), "paged output differs from contiguous"
    if dtype == "bf16":
        _check_outputs(wl, gp, True)
    else:
        _check_outputs(wl, gp, True, max_abs=E4M3_MAX_ABS, mean_abs=E4M3_MEAN_ABS, lse_abs=E4M3_MAX_ABS)


def test_e4m3_head_with_zero_scale():
    """An all-zero query head and an all-zero KV head given scale 0: their logits are 0
    (uniform causal weights; every block ties with the maximum, so nothing is pruned in
    their groups), and the masked keys of the diagonal tile stay masked instead of
    turning into -inf * 0 = NaN."""
    wl = make_workload([700, 300], 8, 2, alpha=0.1, seed=46, dtype="e4m3")
    wl.q.view(torch.uint8)[:, 3] = 0     # e4m3 code 0 is +0
    wl.q_scale[3] = 0.0
    wl.k.view(torch.uint8)[:, 1] = 0
    wl.k_scale[1] = 0.0
    g = run_gpu(wl)
    assert np.isfinite(g["o"]).all() and np.isfinite(g["lse"]).all()
    _check_masks(wl, g)
    _check_outputs(wl, g, True, max_abs=E4M3_MAX_ABS, mean_abs=E4M3_MEAN_ABS, lse_abs=E4M3_MAX_ABS)


def _check_variance(wl, g, sel=None, max_abs=BF16_MAX_ABS, mean_abs=BF16_MEAN_ABS, lse_abs=2e-2):
    """Correction 2 against the oracle's correction with the isotropic variance term
    (its mode 4) on the GPU's lists, and the per-block mean key variances."""
    orc = oracle()
    q, k, v = wl.float_inputs()
    cu = wl.cu_seqlens
    kbar = orc.block_means(k, cu, 128, wl.k_scale)
    vbar = orc.block_means(v, cu, 128, wl.v_scale)
    kvar = orc.block_vars(k, cu, 128, kbar, wl.k_scale)
    want = kvar.mean(axis=2)
    assert np.abs(g["k_var"] - want).max() <= 1e-4 * max(1.0, np.abs(want).max()), "block key variances"
    ref = orc.attend(q, k, v, cu, 128, tau(wl), g["kept_cnt"], g["kept_idx"], correction=4, kbar=kbar, vbar=vbar,
                     kvar=kvar, q_scale=wl.q_scale, k_scale=wl.k_scale, v_scale=wl.v_scale, sel=sel)
    rows = None if sel is None else rows_of_blocks(cu, sel)
    mx, mn = out_errors(g["o"], ref["o"], rows)
    record_output_errors(os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], mx, mn)
    assert mx <= max_abs and mn <= mean_abs, f"output max-abs {mx:.3e} mean-abs {mn:.3e}"
    lm, _ = out_errors(g["lse"], ref["lse"], rows)
    assert lm < lse_abs, f"lse max-abs {lm:.3e}"


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_variance_correction(dtype, paged):
    """correction = 2: the mean correction plus (tau^2 / 2) |q_r|^2 kvar_j on every pruned
    block, G = 4 and G = 3 (one query head alone in its last work item)."""
    for hq, hkv, seed in ((8, 2, 61), (6, 2, 62)):
        wl = make_workload([1000, 700, 2000, 129, 1], hq, hkv, alpha=0.1, seed=seed, dtype=dtype, paged=paged)
        g = run_gpu(wl, correction=2, paged=paged)
        _check_masks(wl, g)
        if dtype == "bf16":
            _check_variance(wl, g)
        else:
            _check_variance(wl, g, max_abs=E4M3_MAX_ABS, mean_abs=E4M3_MEAN_ABS, lse_abs=E4M3_MAX_ABS)


def test_variance_correction_32k_sampled():
    wl = make_config(1)
    g = run_gpu(wl, correction=2)
    nblk = g["kept_cnt"].shape[0]
    sel = sample_blocks(nblk, 12, seed=21, include=(0, nblk - 1))
    _check_variance(wl, g, sel=sel)


def test_many_short_requests():
    """200 requests of 1-300 tokens (seeded) in one batch: many requests per score tile
    and per setup pass, tiny diagonal-only items, the cost order over all of them."""
    rng = np.random.default_rng(71)
    lens = [int(x) for x in rng.integers(1, 301, size=200)]
    wl = make_workload(lens, 8, 2, alpha=0.1, seed=71, n_retrieval=1)
    g = run_gpu(wl)
    _check_masks(wl, g)
    _check_outputs(wl, g, True)


def test_eight_query_heads_per_kv_head():
    """G = 8 (Hq = 16, Hkv = 2): four work items per (q-block, KV head), a score tile of 16
    q-blocks whose 8 rows per q-block meet in warp shuffles."""
    wl = make_workload([1500, 700, 1], 16, 2, alpha=0.1, seed=72, n_retrieval=1)
    g = run_gpu(wl)
    _check_masks(wl, g)
    _check_outputs(wl, g, True)

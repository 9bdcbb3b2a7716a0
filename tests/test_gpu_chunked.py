"""Chunked prefill on the GPU (fp2_estimate_chunked + fp2_prefill_chunked) against
the CPU oracle's chunked form, through the C ABI.

A request has Lk keys and computes only its last Lq query rows (the earlier keys
are already in the KV cache), at positions P = Lk - Lq .. Lk - 1; q-blocks keep
the request's absolute 128-position grid, so the first one may hold fewer rows.
Same bars as the plain tests: kept lists bit-exact outside the near-threshold
band; outputs on the GPU's lists within bf16 max-abs 2e-2 / mean-abs 2e-3 and
e4m3 max-abs 6e-2.
"""
import os

import numpy as np
import pytest

from gpu_helpers import (BF16_MAX_ABS, BF16_MEAN_ABS, E4M3_MAX_ABS, E4M3_MEAN_ABS, check_mask_counts,
                         chunk_block_index,
                         chunk_rows_of_blocks, compare_masks, oracle, out_errors, record_output_errors, run_gpu,
                         run_gpu_chunked, sample_blocks)
from workloads import make_chunked_workload, make_workload

pytestmark = pytest.mark.gpu

# chunk starts P = 0, 1, 128, 200, 424, an empty chunk and a one-row chunk
SEQLENS = [1000, 700, 2000, 300, 900, 500, 333]
QUERY_LENS = [1000, 699, 1872, 100, 476, 0, 1]


def _label():
    return os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]


def _check(wl, g, sel=None, e4m3=False):
    orc = oracle()
    est = orc.run(wl, want_scores=True, sel=np.zeros(0, np.int64))
    check_mask_counts(compare_masks(g, est, wl.alpha, wl.num_kv_heads, None, label=_label(),
                                    block_index=chunk_block_index(wl)))
    assert np.abs(g["k_mean"] - est["kbar"]).max() < 1e-4 * max(1.0, np.abs(est["kbar"]).max())
    ref = orc.run(wl, kept={"kept_cnt": g["kept_cnt"], "kept_idx": g["kept_idx"]}, sel=sel)
    rows = None if sel is None else chunk_rows_of_blocks(wl, sel)
    mx, mn = out_errors(g["o"], ref["o"], rows)
    record_output_errors(_label(), mx, mn)
    lm, _ = out_errors(g["lse"], ref["lse"], rows)
    if e4m3:
        assert mx <= E4M3_MAX_ABS and mn <= E4M3_MEAN_ABS and lm < E4M3_MAX_ABS, \
            f"max-abs {mx:.3e} mean-abs {mn:.3e} lse {lm:.3e}"
    else:
        assert mx <= BF16_MAX_ABS and mn <= BF16_MEAN_ABS and lm < 2e-2, \
            f"max-abs {mx:.3e} mean-abs {mn:.3e} lse {lm:.3e}"
    assert not np.isnan(g["o"] if rows is None else g["o"][rows]).any()


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_chunks_at_several_starts(dtype, paged):
    wl = make_chunked_workload(SEQLENS, QUERY_LENS, 8, 2, alpha=0.1, seed=51, dtype=dtype, paged=paged)
    g = run_gpu_chunked(wl, paged=paged)
    _check(wl, g, e4m3=dtype == "e4m3")


def test_chunk_without_correction():
    wl = make_chunked_workload(SEQLENS, QUERY_LENS, 8, 2, alpha=0.1, seed=52)
    g = run_gpu_chunked(wl, correction=False)
    ref = oracle().run(wl, kept={"kept_cnt": g["kept_cnt"], "kept_idx": g["kept_idx"]}, correction=False)
    mx, mn = out_errors(g["o"], ref["o"])
    assert mx <= BF16_MAX_ABS and mn <= BF16_MEAN_ABS


def test_whole_request_chunks_equal_plain_prefill():
    """Lq = Lk for every request: the chunked calls are the plain ones, bit for bit."""
    lens = [900, 130, 2000, 1]
    wl = make_chunked_workload(lens, lens, 8, 2, alpha=0.1, seed=53)
    g = run_gpu_chunked(wl)
    plain = make_workload(lens, 8, 2, alpha=0.1, seed=53)
    gp = run_gpu(plain)
    assert (g["kept_cnt"] == gp["kept_cnt"]).all() and (g["kept_idx"] == gp["kept_idx"]).all()
    assert np.array_equal(g["o"], gp["o"], equal_nan=True)


def test_chunk_paged_on_the_oracle_mask():
    """The chunked paged call on kept lists given by the caller (the oracle's)."""
    wl = make_chunked_workload(SEQLENS, QUERY_LENS, 8, 2, alpha=0.1, seed=54, paged=True)
    est = oracle().run(wl, sel=np.zeros(0, np.int64))
    kept = {"kept_cnt": est["kept_cnt"], "kept_idx": est["kept_idx"]}
    g = run_gpu_chunked(wl, paged=True, kept=kept)
    ref = oracle().run(wl, kept=kept)
    mx, mn = out_errors(g["o"], ref["o"])
    assert mx <= BF16_MAX_ABS and mn <= BF16_MEAN_ABS


@pytest.mark.parametrize("dtype,paged", [("bf16", False), ("e4m3", True)])
def test_16k_chunk_of_a_128k_request_sampled(dtype, paged):
    """The last 16384 rows of the 128K Llama-3-8B-shaped layer (Hq=32, Hkv=8, alpha=0.05,
    the 128K layer's planted structure): every kept list, outputs on 16 q-blocks; in bf16
    on contiguous K/V, in e4m3 on a page pool of the 128K keys."""
    wl = make_chunked_workload([131072], [16384], 32, 8, alpha=0.05, seed=1002, n_retrieval=16, dtype=dtype,
                               paged=paged)
    g = run_gpu_chunked(wl, paged=paged)
    nq = g["kept_cnt"].shape[0]
    sel = sample_blocks(nq, 16, seed=5, include=(0, nq - 1))
    _check(wl, g, sel=sel, e4m3=dtype == "e4m3")


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_chunks_with_the_variance_term(dtype):
    """correction = 2 on chunks (paged): the oracle's isotropic variance mode with the key
    variances of all keys, the cached prefix's pruned blocks included."""
    wl = make_chunked_workload(SEQLENS, QUERY_LENS, 8, 2, alpha=0.1, seed=55, dtype=dtype, paged=True)
    g = run_gpu_chunked(wl, paged=True, correction=2)
    orc = oracle()
    q, k, v = wl.float_inputs()
    cu_q, cu_k = wl.cu_seqlens_q, wl.cu_seqlens
    kbar = orc.block_means(k, cu_k, 128, wl.k_scale)
    vbar = orc.block_means(v, cu_k, 128, wl.v_scale)
    kvar = orc.block_vars(k, cu_k, 128, kbar, wl.k_scale)
    ref = orc.attend(q, k, v, cu_q, 128, 1.0 / np.sqrt(128.0), g["kept_cnt"], g["kept_idx"], correction=4,
                     kbar=kbar, vbar=vbar, kvar=kvar, q_scale=wl.q_scale, k_scale=wl.k_scale,
                     v_scale=wl.v_scale, cu_seqlens_k=cu_k)
    mx, mn = out_errors(g["o"], ref["o"])
    record_output_errors(_label(), mx, mn)
    if dtype == "bf16":
        assert mx <= BF16_MAX_ABS and mn <= BF16_MEAN_ABS, f"max-abs {mx:.3e} mean-abs {mn:.3e}"
    else:
        assert mx <= E4M3_MAX_ABS and mn <= E4M3_MEAN_ABS, f"max-abs {mx:.3e} mean-abs {mn:.3e}"

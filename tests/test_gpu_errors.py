"""Device-side error reporting with host-made bad inputs (no GPU fault).

The kernels check page indices, cu_seqlens and kept lists themselves, record
FP2_ERR_BAD_INDEX in the workspace flag and skip the bad access (a bad page
is read as page 0, a bad kept list as the diagonal block alone).
fp2_get_error() reads and clears the flag.
"""
import numpy as np
import pytest
import torch

import block_sparse_prefill_b200 as fp2
from gpu_helpers import params_for
from workloads import make_workload

pytestmark = pytest.mark.gpu
BAD_INDEX = 6


def _setup(wl, dev="cuda"):
    params = params_for(wl)
    T, B = wl.total_tokens, wl.batch
    meta = fp2.BlockMeta.empty(params, B, T, wl.max_seqlen, dev)
    ws = fp2.Workspace(params, B, T, wl.max_seqlen, dev)
    out = torch.zeros((T, wl.num_q_heads, 128), dtype=torch.bfloat16, device=dev)
    return params, meta, ws, out


def test_bad_page_index_is_reported_and_cleared():
    wl = make_workload([700, 300], 8, 2, alpha=0.1, seed=5, paged=True)
    params, meta, ws, out = _setup(wl)
    cu = torch.from_numpy(wl.cu_seqlens).cuda()
    good = torch.from_numpy(wl.block_table).cuda()
    bt = wl.block_table.copy()
    bt[1, 1] = wl.num_pages + 17                     # outside the pool
    bad = torch.from_numpy(bt).cuda()
    q, kp, vp = wl.q.cuda(), wl.k_pool.cuda(), wl.v_pool.cuda()
    # the estimator's pooling pass checks every page it reads
    fp2.estimate(params, q, kp, vp, cu, wl.max_seqlen, meta, ws, block_table=bad, num_pages=wl.num_pages)
    assert fp2.get_error(ws) == BAD_INDEX
    assert fp2.get_error(ws) == 0, "fp2_get_error must clear the flag"
    # the attention's scheduler checks the pages of the kept blocks (block 1 of request
    # 1 is always kept: it is that q-block's diagonal)
    fp2.estimate(params, q, kp, vp, cu, wl.max_seqlen, meta, ws, block_table=good, num_pages=wl.num_pages)
    fp2.prefill_paged(params, q, kp, vp, cu, wl.max_seqlen, bad, wl.num_pages, meta, out, ws)
    assert fp2.get_error(ws) == BAD_INDEX
    # the same workspace serves a valid call afterwards
    fp2.prefill_paged(params, q, kp, vp, cu, wl.max_seqlen, good, wl.num_pages, meta, out, ws)
    assert fp2.get_error(ws) == 0
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("bad", ["decreasing", "total", "too_long"])
def test_bad_cu_seqlens_is_reported(bad):
    wl = make_workload([700, 300], 8, 2, alpha=0.1, seed=6)
    params, meta, ws, out = _setup(wl)
    cu = wl.cu_seqlens.copy()
    max_seqlen = wl.max_seqlen
    if bad == "decreasing":
        cu[1] = cu[2] + 5
    elif bad == "total":
        cu[2] -= 1
    else:
        max_seqlen = 500                             # shorter than request 0
    q, k, v = wl.q.cuda(), wl.k.cuda(), wl.v.cuda()
    cu_d = torch.from_numpy(cu).cuda()
    fp2.estimate(params, q, k, v, cu_d, max_seqlen, meta, ws)
    assert fp2.get_error(ws) == BAD_INDEX
    fp2.sparse_prefill(params, q, k, v, cu_d, max_seqlen, meta, out, ws)
    assert fp2.get_error(ws) == BAD_INDEX
    assert (out == 0).all(), "no output may be written for a rejected batch"


def test_corrupt_kept_list_is_reported():
    wl = make_workload([1000], 4, 2, alpha=0.1, seed=7)
    params, meta, ws, out = _setup(wl)
    cu = torch.from_numpy(wl.cu_seqlens).cuda()
    q, k, v = wl.q.cuda(), wl.k.cuda(), wl.v.cuda()
    fp2.estimate(params, q, k, v, cu, wl.max_seqlen, meta, ws)
    assert fp2.get_error(ws) == 0
    idx = meta.kept_idx.cpu().numpy()
    cnt = meta.kept_cnt.cpu().numpy()
    t = 5
    idx[t, 0, :cnt[t, 0]] = idx[t, 0, :cnt[t, 0]][::-1]  # descending: invalid
    cnt[t, 1] = 1000                                        # more blocks than exist
    meta.kept_idx.copy_(torch.from_numpy(idx))
    meta.kept_cnt.copy_(torch.from_numpy(cnt))
    fp2.sparse_prefill(params, q, k, v, cu, wl.max_seqlen, meta, out, ws)
    assert fp2.get_error(ws) == BAD_INDEX
    assert torch.isfinite(out.float()).all()


TIMEOUT = 5


def test_wait_timeout_is_reported_and_the_context_stays_usable(monkeypatch):
    """The attention kernel's bounded waits: with the FP2_TEST_WAIT_TIMEOUT hook its MMA issuer
    waits on a barrier that nothing completes.  After about a second (2^31 cycles) the wait
    gives up, records FP2_ERR_TIMEOUT and sets the CTA's abort flag; every role stops, the
    issued TMA copies land, TMEM is freed and the kernel returns.  The same context and
    workspace then run the call again with a bit-identical result."""
    wl = make_workload([1000, 700], 4, 2, alpha=0.1, seed=9)
    params, meta, ws, out = _setup(wl)
    cu = torch.from_numpy(wl.cu_seqlens).cuda()
    q, k, v = wl.q.cuda(), wl.k.cuda(), wl.v.cuda()
    fp2.estimate(params, q, k, v, cu, wl.max_seqlen, meta, ws)
    fp2.sparse_prefill(params, q, k, v, cu, wl.max_seqlen, meta, out, ws)
    assert fp2.get_error(ws) == 0
    ref = out.clone()

    monkeypatch.setenv("FP2_TEST_WAIT_TIMEOUT", "1")
    out.zero_()
    fp2.sparse_prefill(params, q, k, v, cu, wl.max_seqlen, meta, out, ws)
    assert fp2.get_error(ws) == TIMEOUT
    monkeypatch.delenv("FP2_TEST_WAIT_TIMEOUT")

    out.zero_()
    fp2.sparse_prefill(params, q, k, v, cu, wl.max_seqlen, meta, out, ws)
    assert fp2.get_error(ws) == 0
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))

"""fp2_sparse_prefill_noalloc against fp2_sparse_prefill, through the C ABI.

Some callers cannot allocate device memory where they run attention: a plugin
inside a framework that owns every device allocation, code with a memory
budget fixed up front, or latency-critical code that must not take
cudaMalloc's implicit device synchronisation.  For them the library offers an
entry point without a workspace that uses its own fixed device array as
scratch.  It must give what the workspace-based call gives, also when called
twice in a row (the array keeps the previous call's contents).

This file sorts last so that a run stopping at the first failure has already
run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_prefill_b200 as fp2
from block_sparse_prefill_b200 import _lib
from workloads import make_workload

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3   # the bf16 output tolerance of the parity tests


def _noalloc(params, q, k, v, cu, max_seqlen, meta, out, lse, status):
    p, m = params.c(), meta.c()
    return _lib.load().fp2_sparse_prefill_noalloc(
        ctypes.byref(p), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(cu.data_ptr()), cu.numel() - 1, q.shape[0], max_seqlen,
        ctypes.byref(m), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _compare(wl, dev="cuda"):
    params = fp2.Params(num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads, alpha=wl.alpha)
    T, B = wl.total_tokens, wl.batch
    q, k, v = wl.q.to(dev), wl.k.to(dev), wl.v.to(dev)
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    meta = fp2.BlockMeta.empty(params, B, T, wl.max_seqlen, dev)
    ws = fp2.Workspace(params, B, T, wl.max_seqlen, dev)
    fp2.estimate(params, q, k, v, cu, wl.max_seqlen, meta, ws)
    ref = torch.full((T, wl.num_q_heads, 128), float("nan"), dtype=torch.bfloat16, device=dev)
    ref_lse = torch.full((T, wl.num_q_heads), float("nan"), device=dev)
    fp2.sparse_prefill(params, q, k, v, cu, wl.max_seqlen, meta, ref, ws, lse=ref_lse)
    out = torch.full_like(ref, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    rc = _noalloc(params, q, k, v, cu, wl.max_seqlen, meta, out, lse, status)
    assert rc == 0, fp2.status_string(rc)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device-side error in the allocation-free call"
    assert fp2.get_error(ws) == 0
    a, b = out.float().cpu().numpy(), ref.float().cpu().numpy()
    assert not np.isnan(b).any()
    err = np.abs(a - b)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, f"max-abs {err.max():.3e} mean-abs {err.mean():.3e}"
    assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= MAX_ABS


def test_noalloc_matches_workspace_call_twice():
    # two calls in a row on different problems: the second must not see the
    # first call's leftovers in the shared array
    _compare(make_workload([3000, 700, 129], 8, 2, alpha=0.1, seed=77))
    _compare(make_workload([5000], 4, 1, alpha=0.05, seed=78))


def test_noalloc_rejects_problems_over_the_static_maximum():
    params = fp2.Params(num_q_heads=32, num_kv_heads=8)
    T = 1 << 20  # needs ~34 MB of scratch, over the 8 MiB array
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    meta = _lib.fp2_blockmeta(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), None,
                              T // 128, T // 128 + 1)
    p = params.c()
    ptr = ctypes.c_void_p(dummy.data_ptr())
    rc = _lib.load().fp2_sparse_prefill_noalloc(ctypes.byref(p), ptr, ptr, ptr, ptr, 1, T, T, ctypes.byref(meta),
                                                ptr, None, None, None)
    assert rc == 3, f"expected FP2_ERR_WORKSPACE, got {fp2.status_string(rc)}"

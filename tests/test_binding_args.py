"""The Python binding's argument checks, on the host (no GPU, no library call).

The C ABI receives bare addresses, so the binding checks each array's dtype,
shape, layout and device first.  Well-formed arguments, built the way the GPU
tests and the benchmark build them but left on the CPU, must get through every
check except the device check; each malformed argument must be named in the
error."""
import pytest
import torch

import block_sparse_prefill_b200 as fp2
from workloads.synthetic import make_workload

CPU_MSG = "must be on a CUDA device"


def _params(wl):
    p = fp2.Params(num_q_heads=wl.num_q_heads, num_kv_heads=wl.num_kv_heads, alpha=wl.alpha,
                   dtype=fp2.FP2_E4M3 if wl.dtype == "e4m3" else fp2.FP2_BF16)
    if wl.dtype == "e4m3":
        p.q_scale = torch.from_numpy(wl.q_scale)
        p.k_scale = torch.from_numpy(wl.k_scale)
        p.v_scale = torch.from_numpy(wl.v_scale)
    return p


def _io(wl):
    T, H = wl.total_tokens, wl.num_q_heads
    cu = torch.from_numpy(wl.cu_seqlens)
    out = torch.zeros((T, H, 128), dtype=torch.bfloat16)
    lse = torch.zeros((T, H), dtype=torch.float32)
    return cu, out, lse


@pytest.fixture(scope="module")
def bf16():
    return make_workload([300, 129], 8, 2, alpha=0.1, seed=3)


@pytest.fixture(scope="module")
def e4m3():
    return make_workload([300, 129], 8, 2, alpha=0.1, seed=3, dtype="e4m3")


@pytest.fixture(scope="module")
def paged():
    return make_workload([300, 129], 8, 2, alpha=0.1, seed=3, paged=True)


@pytest.mark.parametrize("which", ["bf16", "e4m3"])
def test_well_formed_arguments_reach_the_device_check(which, request):
    wl = request.getfixturevalue(which)
    p = _params(wl)
    cu, out, lse = _io(wl)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.estimate(p, wl.q, wl.k, wl.v, cu, wl.max_seqlen, None, None)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.sparse_prefill(p, wl.q, wl.k, wl.v, cu, wl.max_seqlen, None, out, None, lse=lse)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.sparse_prefill_noalloc(p, wl.q, wl.k, wl.v, cu, wl.max_seqlen, None, out, lse=lse)


def test_well_formed_paged_arguments_reach_the_device_check(paged):
    p = _params(paged)
    cu, out, lse = _io(paged)
    bt = torch.from_numpy(paged.block_table)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.prefill_paged(p, paged.q, paged.k_pool, paged.v_pool, cu, paged.max_seqlen, bt,
                          paged.num_pages, None, out, None, lse=lse)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.estimate(p, paged.q, paged.k_pool, paged.v_pool, cu, paged.max_seqlen, None, None,
                     block_table=bt, num_pages=paged.num_pages)


def test_strided_view_is_rejected(bf16):
    p = _params(bf16)
    cu, out, lse = _io(bf16)
    # q sliced out of a fused [T, Hq + 2 Hkv, d] projection: right shape, wrong strides
    qkv = torch.cat([bf16.q, bf16.k, bf16.v], dim=1)
    q_view = qkv[:, :bf16.num_q_heads]
    assert q_view.shape == bf16.q.shape and not q_view.is_contiguous()
    with pytest.raises(ValueError, match="q must be contiguous"):
        fp2.sparse_prefill(p, q_view, bf16.k, bf16.v, cu, bf16.max_seqlen, None, out, None)
    with pytest.raises(ValueError, match="out must be contiguous"):
        fp2.sparse_prefill(p, bf16.q, bf16.k, bf16.v, cu, bf16.max_seqlen, None,
                           out.transpose(0, 1).contiguous().transpose(0, 1), None)


@pytest.mark.parametrize("case, exc, match", [
    ("q_float32", TypeError, "q has dtype"),
    ("k_e4m3", TypeError, "k has dtype"),
    ("cu_int64", TypeError, "cu_seqlens has dtype"),
    ("out_float32", TypeError, "out has dtype"),
    ("lse_bf16", TypeError, "lse has dtype"),
    ("q_heads", ValueError, "q has shape"),
    ("q_head_dim", ValueError, "q has shape"),
    ("k_rows", ValueError, "k has shape"),
    ("v_heads", ValueError, "v has shape"),
    ("out_rows", ValueError, "out has shape"),
    ("lse_2d_wrong", ValueError, "lse has shape"),
    ("cu_empty", ValueError, "cu_seqlens needs"),
    ("cu_missing", TypeError, "cu_seqlens is required"),
    ("q_not_tensor", TypeError, "q must be a torch.Tensor"),
])
def test_malformed_argument_is_named(bf16, case, exc, match):
    p = _params(bf16)
    cu, out, lse = _io(bf16)
    q, k, v = bf16.q, bf16.k, bf16.v
    if case == "q_float32":
        q = q.float()
    elif case == "k_e4m3":
        k = k.to(torch.float8_e4m3fn)
    elif case == "cu_int64":
        cu = cu.long()
    elif case == "out_float32":
        out = out.float()
    elif case == "lse_bf16":
        lse = lse.bfloat16()
    elif case == "q_heads":
        q = q[:, :4].contiguous()
    elif case == "q_head_dim":
        q = q[:, :, :64].contiguous()
    elif case == "k_rows":
        k = k[:-1].contiguous()
    elif case == "v_heads":
        v = torch.cat([v, v], dim=1)
    elif case == "out_rows":
        out = out[1:].contiguous()
    elif case == "lse_2d_wrong":
        lse = lse.reshape(-1)
    elif case == "cu_empty":
        cu = cu[:0]
    elif case == "cu_missing":
        cu = None
    elif case == "q_not_tensor":
        q = q.numpy(force=True) if q.dtype != torch.bfloat16 else [0]
    with pytest.raises(exc, match=match):
        fp2.sparse_prefill(p, q, k, v, cu, bf16.max_seqlen, None, out, None, lse=lse)


def test_paged_pool_and_table_shapes_are_checked(paged):
    p = _params(paged)
    cu, out, lse = _io(paged)
    bt = torch.from_numpy(paged.block_table)
    n = paged.num_pages
    with pytest.raises(ValueError, match="k has shape"):
        fp2.prefill_paged(p, paged.q, paged.k_pool, paged.v_pool, cu, paged.max_seqlen, bt, n + 1,
                          None, out, None)
    with pytest.raises(TypeError, match="block_table has dtype"):
        fp2.prefill_paged(p, paged.q, paged.k_pool, paged.v_pool, cu, paged.max_seqlen, bt.long(), n,
                          None, out, None)
    with pytest.raises(ValueError, match="block_table has shape"):
        fp2.prefill_paged(p, paged.q, paged.k_pool, paged.v_pool, cu, paged.max_seqlen, bt[:1], n,
                          None, out, None)


def test_e4m3_scales_are_required_and_checked(e4m3):
    cu, out, lse = _io(e4m3)
    p = _params(e4m3)
    p.k_scale = None
    with pytest.raises(ValueError, match="need params.k_scale"):
        fp2.sparse_prefill(p, e4m3.q, e4m3.k, e4m3.v, cu, e4m3.max_seqlen, None, out, None)
    p = _params(e4m3)
    p.q_scale = p.q_scale[:1].clone()
    with pytest.raises(ValueError, match="q_scale has shape"):
        fp2.sparse_prefill(p, e4m3.q, e4m3.k, e4m3.v, cu, e4m3.max_seqlen, None, out, None)
    p = _params(e4m3)
    p.v_scale = p.v_scale.double()
    with pytest.raises(TypeError, match="v_scale has dtype"):
        fp2.sparse_prefill(p, e4m3.q, e4m3.k, e4m3.v, cu, e4m3.max_seqlen, None, out, None)


@pytest.fixture(scope="module")
def chunk():
    from workloads.synthetic import make_chunked_workload
    return make_chunked_workload([300, 200], [100, 200], 8, 2, alpha=0.1, seed=3, paged=True)


def test_well_formed_chunk_arguments_reach_the_device_check(chunk):
    p = _params(chunk)
    cu_q, cu_k = torch.from_numpy(chunk.cu_seqlens_q), torch.from_numpy(chunk.cu_seqlens)
    Tq, Tk = chunk.total_queries, chunk.total_tokens
    out = torch.zeros((Tq, 8, 128), dtype=torch.bfloat16)
    lse = torch.zeros((Tq, 8), dtype=torch.float32)
    bt = torch.from_numpy(chunk.block_table)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.estimate_chunked(p, chunk.q, chunk.k, chunk.v, cu_q, cu_k, Tk, chunk.max_seqlen, None, None)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.prefill_chunked(p, chunk.q, chunk.k, chunk.v, cu_q, cu_k, Tk, chunk.max_seqlen, None, out, None,
                            lse=lse)
    with pytest.raises(ValueError, match=CPU_MSG):
        fp2.prefill_chunked(p, chunk.q, chunk.k_pool, chunk.v_pool, cu_q, cu_k, Tk, chunk.max_seqlen, None, out,
                            None, lse=lse, block_table=bt, num_pages=chunk.num_pages)


def test_malformed_chunk_arguments_are_named(chunk):
    p = _params(chunk)
    cu_q, cu_k = torch.from_numpy(chunk.cu_seqlens_q), torch.from_numpy(chunk.cu_seqlens)
    Tq, Tk = chunk.total_queries, chunk.total_tokens
    out = torch.zeros((Tq, 8, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="same batch"):
        fp2.prefill_chunked(p, chunk.q, chunk.k, chunk.v, cu_q[:-1], cu_k, Tk, chunk.max_seqlen, None, out, None)
    with pytest.raises(ValueError, match="total_k"):
        fp2.estimate_chunked(p, chunk.q, chunk.k, chunk.v, cu_q, cu_k, Tk + 1, chunk.max_seqlen, None, None)
    with pytest.raises(ValueError, match="out has shape"):
        fp2.prefill_chunked(p, chunk.q, chunk.k, chunk.v, cu_q, cu_k, Tk, chunk.max_seqlen, None,
                            torch.zeros((Tk, 8, 128), dtype=torch.bfloat16), None)
    with pytest.raises(TypeError, match="cu_seqlens_k has dtype"):
        fp2.estimate_chunked(p, chunk.q, chunk.k, chunk.v, cu_q, cu_k.long(), Tk, chunk.max_seqlen, None, None)

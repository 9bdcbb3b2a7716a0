"""Seeded input generator: determinism, paging and the e4m3 encoding (no GPU)."""
import numpy as np
import torch

from workloads import make_workload, make_config, quantize_e4m3


def test_deterministic():
    a = make_workload([700, 300], 4, 2, seed=5)
    b = make_workload([700, 300], 4, 2, seed=5)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    c = make_workload([700, 300], 4, 2, seed=6)
    assert not torch.equal(a.q, c.q)


def test_paged_pool_matches_contiguous():
    wl = make_workload([300, 1, 520], 4, 2, seed=9, paged=True)
    bs = wl.block_size
    cu = wl.cu_seqlens
    used = []
    for b, L in enumerate(wl.seqlens):
        for j in range((L + bs - 1) // bs):
            p = int(wl.block_table[b, j])
            used.append(p)
            n = min(bs, L - j * bs)
            assert torch.equal(wl.k_pool[p * bs:p * bs + n], wl.k[cu[b] + j * bs:cu[b] + j * bs + n])
            assert torch.equal(wl.v_pool[p * bs:p * bs + n], wl.v[cu[b] + j * bs:cu[b] + j * bs + n])
    assert sorted(used) == list(range(wl.num_pages)), "pages are not a permutation"
    assert used != sorted(used), "pages are not shuffled"


def test_e4m3_per_head_absmax():
    x = torch.randn(1000, 3, 128) * torch.tensor([1.0, 5.0, 0.0])[None, :, None]
    codes, sc = quantize_e4m3(x)
    assert codes.dtype == torch.float8_e4m3fn
    assert sc[2] == 1.0
    for h in range(2):
        assert np.isclose(sc[h], float(x[:, h].abs().max()) / 448.0)
        assert float(codes[:, h].float().abs().max()) == 448.0
    # decoding recovers x within e4m3 relative precision (3 mantissa bits)
    err = (codes.float() * torch.from_numpy(sc)[None, :, None] - x).abs()
    assert (err <= x.abs() * 2 ** -4 + 2 ** -9 * float(sc.max())).all()


def test_config_shapes():
    wl = make_config(0)
    assert wl.seqlens == [2048] and wl.num_q_heads == 2 and wl.num_kv_heads == 1 and wl.alpha == 0.1
    assert len(wl.planted[0]["retrieval"][0]) == 3
    w3 = make_config(3, seqlen=1024)
    w2 = make_config(2, seqlen=1024)
    assert w3.dtype == "e4m3" and w3.q.dtype == torch.float8_e4m3fn
    # config 3 is config 2 encoded in e4m3
    x = w3.q.float() * torch.from_numpy(w3.q_scale)[None, :, None]
    assert ((x - w2.q.float()).abs() <= w2.q.float().abs() * 2 ** -4 + 1e-2).all()


def test_chunked_workload_rows_and_scales():
    """The queries of a chunked workload are the last rows of the plain workload's
    requests (same seed); e4m3 query scales come from the chunk's rows."""
    from workloads import make_chunked_workload
    lens, lq = [700, 300, 129], [500, 45, 129]
    full = make_workload(lens, 8, 2, alpha=0.1, seed=3)
    ch = make_chunked_workload(lens, lq, 8, 2, alpha=0.1, seed=3)
    cu, cuq = full.cu_seqlens, ch.cu_seqlens_q
    assert list(cuq) == [0, 500, 545, 674] and ch.total_queries == 674 and ch.total_tokens == 1129
    for b, n in enumerate(lq):
        assert torch.equal(ch.q[cuq[b]:cuq[b + 1]], full.q[cu[b + 1] - n:cu[b + 1]])
    assert torch.equal(ch.k, full.k) and torch.equal(ch.v, full.v)
    e = make_chunked_workload(lens, lq, 8, 2, alpha=0.1, seed=3, dtype="e4m3")
    amax = ch.q.float().abs().amax(dim=(0, 2)).numpy()
    assert np.allclose(e.q_scale, amax / 448.0, rtol=1e-6)
    amax_k = full.k.float().abs().amax(dim=(0, 2)).numpy()
    assert np.allclose(e.k_scale, amax_k / 448.0, rtol=1e-6)


def test_chunked_paged_pool_matches_contiguous():
    from workloads import make_chunked_workload
    wl = make_chunked_workload([700, 300], [500, 45], 4, 2, alpha=0.1, seed=4, paged=True)
    cu = wl.cu_seqlens
    for b, L in enumerate(wl.seqlens):
        for j in range((L + 127) // 128):
            page = int(wl.block_table[b, j])
            n = min(128, L - j * 128)
            assert torch.equal(wl.k_pool[page * 128:page * 128 + n], wl.k[cu[b] + j * 128:cu[b] + j * 128 + n])


def test_oracle_run_on_a_block_aligned_chunk_equals_full_rows():
    """Oracle.run on a chunked workload: a chunk starting on a block boundary gives
    the full prefill's rows (the D0 chunked form reduces to the plain one there)."""
    from oracle.oracle import Oracle
    from workloads import make_chunked_workload
    lens, lq = [1000, 640], [744, 256]              # chunks start at 256 and 384
    orc = Oracle()
    full = orc.run(make_workload(lens, 4, 2, alpha=0.2, seed=9))
    ch = orc.run(make_chunked_workload(lens, lq, 4, 2, alpha=0.2, seed=9))
    cu, cuq = np.array([0, 1000, 1640]), np.array([0, 744, 1000])
    for b, n in enumerate(lq):
        assert np.array_equal(ch["o"][cuq[b]:cuq[b + 1]], full["o"][cu[b + 1] - n:cu[b + 1]])
        assert np.array_equal(ch["lse"][cuq[b]:cuq[b + 1]], full["lse"][cu[b + 1] - n:cu[b + 1]])

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

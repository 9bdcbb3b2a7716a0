"""The device-drawn long-request inputs (workloads.long_context), drawn here on the
CPU at a small size: seeded, and with the kept structure their recipe states (the
oracle's estimator keeps the diagonal, the sink and the retrieval blocks, and
prunes every other block)."""
import math

import numpy as np
import torch

from oracle.oracle import Oracle
from workloads import make_long_device_inputs


def test_seeded_and_structured():
    L, every = 128 * 60 - 37, 11
    a = make_long_device_inputs(L, "bf16", 8, 2, 128, 128, seed=5, device="cpu", retrieval_every=every)
    b = make_long_device_inputs(L, "bf16", 8, 2, 128, 128, seed=5, device="cpu", retrieval_every=every)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["k"], b["k"]) and torch.equal(a["v"], b["v"])
    orc = Oracle()
    q, k = a["q"].float().numpy(), a["k"].float().numpy()
    cu = a["cu_seqlens"]
    qbar = orc.block_means(q, cu, 128)
    kbar = orc.block_means(k, cu, 128)
    est = orc.estimate(qbar, kbar, cu, 128, 0.05, 1.0 / math.sqrt(128))
    nb = qbar.shape[0]
    for t in range(nb):
        want = sorted({0, t} | set(range(every, t, every)))
        for g in range(2):
            c = est["kept_cnt"][t, g]
            assert est["kept_idx"][t, g, :c].tolist() == want, (t, g)


def test_e4m3_codes_and_scales():
    d = make_long_device_inputs(128 * 5, "e4m3", 4, 2, 128, 128, seed=1, device="cpu")
    assert d["q"].dtype == torch.float8_e4m3fn and d["k"].dtype == torch.float8_e4m3fn
    assert d["q_scale"].shape == (4,) and d["k_scale"].shape == (2,) and (d["v_scale"] > 0).all()
    assert np.isfinite(d["q"].float().numpy()).all()

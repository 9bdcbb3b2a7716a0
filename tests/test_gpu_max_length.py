"""The longest request the ABI accepts, through the C ABI on the GPU.

One request of FP2_MAX_SEQ_BLOCKS_{BF16,E4M3} blocks (the last one partial: 37
tokens short), so that the attention kernel runs with the largest metadata
buffers its shared memory holds, and Q holds more than 2^31 elements (bf16:
528,475 x 32 x 128; e4m3: 1,033,051 x 32 x 128).  The inputs are drawn on the
device (``workloads.make_long_device_inputs``: a sink block and retrieval blocks,
so the kept lists are short and most blocks enter through the mean correction).

Reference: the oracle on sampled q-blocks, each taken as the query chunk of its
own prefix (the chunked form; on small cases it equals the plain form exactly).
Masks: the GPU's kept lists of the sampled q-blocks against the oracle's, with the
near-threshold band.  Outputs: the oracle re-run with the GPU's kept lists; bf16
2e-2 max-abs / 2e-3 mean-abs, e4m3 6e-2 / 6e-3; LSE 2e-2 / 6e-2.
"""
import math
import os
import re

import numpy as np
import pytest
import torch

import block_sparse_prefill_b200 as fp2
from gpu_helpers import (BF16_MAX_ABS, BF16_MEAN_ABS, E4M3_MAX_ABS, E4M3_MEAN_ABS, check_mask_counts,
                         compare_masks, oracle, record_output_errors)
from workloads import make_long_device_inputs

pytestmark = pytest.mark.gpu

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp2.h")
HQ, HKV, D, BS, ALPHA = 32, 8, 128, 128, 0.05


def _limit(name):
    text = open(HEADER).read()
    return int(re.search(rf"#define FP2_MAX_SEQ_BLOCKS_{name}\s+(\d+)", text).group(1))


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_longest_request(dtype):
    nb = _limit(dtype.upper())
    L = nb * BS - 37
    dev = torch.device("cuda")
    inp = make_long_device_inputs(L, dtype, HQ, HKV, D, BS, seed=17, device=dev)
    e4 = dtype == "e4m3"
    p = fp2.Params(num_q_heads=HQ, num_kv_heads=HKV, alpha=ALPHA, correction=True,
                   dtype=fp2.FP2_E4M3 if e4 else fp2.FP2_BF16)
    if e4:
        p.q_scale = torch.from_numpy(inp["q_scale"]).to(dev)
        p.k_scale = torch.from_numpy(inp["k_scale"]).to(dev)
        p.v_scale = torch.from_numpy(inp["v_scale"]).to(dev)
    cu = torch.from_numpy(inp["cu_seqlens"]).to(dev)
    meta = fp2.BlockMeta.empty(p, 1, L, L, dev)
    ws = fp2.Workspace(p, 1, L, L, dev)
    out = torch.full((L, HQ, D), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((L, HQ), float("nan"), dtype=torch.float32, device=dev)
    fp2.estimate(p, inp["q"], inp["k"], inp["v"], cu, L, meta, ws)
    fp2.sparse_prefill(p, inp["q"], inp["k"], inp["v"], cu, L, meta, out, ws, lse=lse)
    torch.cuda.synchronize()
    assert fp2.get_error(ws) == 0, fp2.status_string(fp2.get_error(ws))

    sel = sorted({0, 1, nb // 3, nb // 2, (2 * nb) // 3, nb - 2, nb - 1})
    gcnt = meta.kept_cnt[:nb].cpu().numpy()
    gidx = meta.kept_idx[:nb].cpu().numpy()
    # every q-block's list: ascending, inside [0, t], ending on the diagonal
    assert (gcnt >= 1).all() and (gcnt <= np.arange(1, nb + 1)[:, None]).all()
    last = np.take_along_axis(gidx, (gcnt - 1)[:, :, None].astype(np.int64), axis=2)[:, :, 0]
    assert (last == np.arange(nb)[:, None]).all(), "a kept list does not end on its diagonal block"

    orc = oracle()
    tau = 1.0 / math.sqrt(D)
    kh = inp["k"].float().cpu().numpy()
    vh = inp["v"].float().cpu().numpy()
    kbar = orc.block_means(kh, [0, L], BS, inp["k_scale"])
    vbar = orc.block_means(vh, [0, L], BS, inp["v_scale"])
    max_abs, mean_abs = (E4M3_MAX_ABS, E4M3_MEAN_ABS) if e4 else (BF16_MAX_ABS, BF16_MEAN_ABS)
    lse_abs = E4M3_MAX_ABS if e4 else 2e-2
    totals = {"outside": 0, "excused": 0, "near": 0, "compared": 0}
    errs, sums, count = [], 0.0, 0
    for t in sel:
        r0 = BS * t
        n = min(BS, L - r0)
        lk = r0 + n
        qrows = inp["q"][r0:r0 + n].float().cpu().numpy()
        qbar = orc.block_means(qrows, [0, n], BS, inp["q_scale"], pos0=[r0])
        est = orc.estimate(qbar, kbar[:t + 1], [0, n], BS, ALPHA, tau, nb_max=t + 1, want_scores=True,
                           cu_seqlens_k=[0, lk])
        g = {"kept_cnt": gcnt[t:t + 1], "kept_idx": gidx[t:t + 1, :, :t + 1]}
        res = compare_masks(g, est, ALPHA, HKV, None, label=f"test_longest_request[{dtype}] q-block {t}",
                            block_index=[t])
        for key in totals:
            totals[key] += res[key]
        ref = orc.attend(qrows, kh[:lk], vh[:lk], [0, n], BS, tau, g["kept_cnt"], g["kept_idx"], correction=True,
                         kbar=kbar[:t + 1], vbar=vbar[:t + 1], q_scale=inp["q_scale"], k_scale=inp["k_scale"],
                         v_scale=inp["v_scale"], cu_seqlens_k=[0, lk])
        o = out[r0:r0 + n].float().cpu().numpy()
        diff = np.abs(o - ref["o"])
        assert np.isfinite(o).all(), f"q-block {t}: non-finite output"
        errs.append(float(diff.max()))
        sums += float(diff.sum())
        count += diff.size
        lm = float(np.abs(lse[r0:r0 + n].cpu().numpy() - ref["lse"]).max())
        assert lm < lse_abs, f"q-block {t}: lse max-abs {lm:.3e}"
    check_mask_counts(totals)
    mx, mn = max(errs), sums / count
    record_output_errors(f"test_longest_request[{dtype}]", mx, mn)
    assert mx <= max_abs and mn <= mean_abs, f"output max-abs {mx:.3e} mean-abs {mn:.3e}"

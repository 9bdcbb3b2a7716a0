"""Seeded synthetic inputs of one very long request, drawn on the device.

The planted generator of ``synthetic.py`` draws on the host in numpy, which at a
million tokens takes minutes and tens of GB.  This one draws with torch's seeded
generator on the given device, so the longest requests the library accepts can be
built in a second.  Like ``synthetic.py`` it holds none of the method's arithmetic.

Recipe (one request of ``length`` tokens, Llama-3-8B-shaped heads):

* ``torch.Generator(device).manual_seed(seed)``; values drawn in fp32, rounded to
  bf16, token-major ``[T, H, d]``.
* Q, K, V ~ N(0, 1).
* ``u``: one seeded unit vector.
* query offset: every Q row gets ``+4u``.
* sink: every K row of key block 0 gets ``+12u``.
* retrieval: every K row of every ``retrieval_every``-th key block gets ``+9u``.
* The block-mean scores then put the sink about 4.2 nats above a plain block and
  the retrieval blocks about 1.1 nats below the sink: at alpha = 0.05 (3 nats) the
  kept lists hold the diagonal, the sink and the retrieval blocks, and every other
  block is pruned and enters through its mean.
* FP8: ``synthetic.quantize_e4m3`` (per-head absmax / 448).
"""
from __future__ import annotations

import numpy as np
import torch

from .synthetic import quantize_e4m3


def make_long_device_inputs(length: int, dtype: str = "bf16", num_q_heads: int = 32, num_kv_heads: int = 8,
                            head_dim: int = 128, block_size: int = 128, seed: int = 0, device="cuda",
                            retrieval_every: int = 509):
    """Returns dict(q, k, v on ``device`` (bf16, or e4m3 codes), q_scale, k_scale, v_scale
    (numpy float32 per head), cu_seqlens (numpy int32), length)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    u = torch.randn(head_dim, generator=g, device=device)
    u = u / u.norm()

    def draw(h):
        return torch.randn((length, h, head_dim), generator=g, device=device)

    q = draw(num_q_heads)
    q += 4.0 * u
    q = q.to(torch.bfloat16)
    k = draw(num_kv_heads)
    k[:block_size] += 12.0 * u
    nb = (length + block_size - 1) // block_size
    for j in range(retrieval_every, nb, retrieval_every):
        k[j * block_size:(j + 1) * block_size] += 9.0 * u
    k = k.to(torch.bfloat16)
    v = draw(num_kv_heads).to(torch.bfloat16)
    if dtype == "e4m3":
        q, qs = quantize_e4m3(q)
        k, ks = quantize_e4m3(k)
        v, vs = quantize_e4m3(v)
    elif dtype == "bf16":
        qs = np.ones(num_q_heads, np.float32)
        ks = np.ones(num_kv_heads, np.float32)
        vs = np.ones(num_kv_heads, np.float32)
    else:
        raise ValueError(dtype)
    return {"q": q, "k": k, "v": v, "q_scale": qs, "k_scale": ks, "v_scale": vs,
            "cu_seqlens": np.array([0, length], np.int32), "length": length}

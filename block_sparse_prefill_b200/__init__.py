"""B200 (sm_100a) block-sparse prefill attention: Python binding of libfp2.

Every function here marshals torch tensors into the C ABI of include/fp2.h;
all work runs in the CUDA kernels of libfp2.so.  There is no CPU path: a
missing library raises.

    params = Params(num_q_heads=32, num_kv_heads=8, alpha=0.05)
    meta = BlockMeta.empty(params, batch, total_tokens, max_seqlen, device)
    ws = Workspace(params, batch, total_tokens, max_seqlen, device)
    estimate(params, q, k, v, cu_seqlens, max_seqlen, meta, ws)
    sparse_prefill(params, q, k, v, cu_seqlens, max_seqlen, meta, out, ws, lse=lse)

Paged KV cache: ``estimate(..., block_table=bt, num_pages=n)`` on the page
pools, then ``prefill_paged(params, q, k_pool, v_pool, cu_seqlens, max_seqlen,
bt, n, meta, out, ws, lse=lse)``.

Chunked prefill (queries are the last rows of each request, the earlier keys
already cached): ``estimate_chunked`` and ``prefill_chunked`` with
``cu_seqlens_q`` (query rows) and ``cu_seqlens_k`` (keys); size the meta and the
workspace by the total keys.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import _lib
from ._lib import FP2_BF16, FP2_E4M3, STATUS

__all__ = ["Params", "BlockMeta", "Workspace", "FP2Error", "max_blocks", "workspace_bytes",
           "estimate", "sparse_prefill", "sparse_prefill_noalloc", "prefill_paged", "estimate_chunked",
           "prefill_chunked", "get_error",
           "status_string", "version",
           "FP2_BF16", "FP2_E4M3"]

BLOCK = 128
HEAD_DIM = 128


class FP2Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({status_string(code)})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(code: int, where: str):
    if code != 0:
        raise FP2Error(code, where)


_E4M3_DTYPES = (torch.float8_e4m3fn, torch.uint8)


def _arg(t, name: str, dtypes, shape, where: str):
    """Checks one array argument before its pointer goes to the C ABI, which
    sees only the address: a dense (contiguous) tensor of one of ``dtypes``
    whose shape matches ``shape`` (None entries match any size).  ``None``
    passes for optional arguments.  The device is checked by ``_same_cuda``
    once every argument's layout has passed."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{where}: {name} must be a torch.Tensor, got {type(t).__name__}")
    if t.dtype not in dtypes:
        raise TypeError(f"{where}: {name} has dtype {t.dtype}, expected one of {list(dtypes)}")
    if t.dim() != len(shape) or any(s is not None and s != n for s, n in zip(shape, t.shape)):
        want = "[" + ", ".join("*" if s is None else str(s) for s in shape) + "]"
        raise ValueError(f"{where}: {name} has shape {list(t.shape)}, expected {want}")
    if not t.is_contiguous():
        raise ValueError(f"{where}: {name} must be contiguous (row-major); pass .contiguous()")


def _same_cuda(where: str, **arrays) -> None:
    """Every array given must sit on one CUDA device (an array on another GPU
    would reach the kernels as a peer address)."""
    dev = None
    for name, t in arrays.items():
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"{where}: {name} must be on a CUDA device, got {t.device}")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{where}: {name} is on {t.device}, the other arrays on {dev}")


def _qkv_args(params: "Params", q, k, v, cu_seqlens, out, lse, where: str, kv_rows=None):
    """Checks the arrays shared by the compute calls: q [T, Hq, d] and k, v
    [kv_rows, Hkv, d] in the input type, cu_seqlens [batch + 1] int32,
    out [T, Hq, d] bf16, lse [T, Hq] fp32."""
    for name, t in (("q", q), ("k", k), ("v", v), ("cu_seqlens", cu_seqlens)):
        if t is None:
            raise TypeError(f"{where}: {name} is required")
    io = (torch.bfloat16,) if params.dtype == FP2_BF16 else _E4M3_DTYPES
    d, hq, hkv = params.head_dim, params.num_q_heads, params.num_kv_heads
    _arg(q, "q", io, (None, hq, d), where)
    T = int(q.shape[0])
    _arg(k, "k", io, (T if kv_rows is None else kv_rows, hkv, d), where)
    _arg(v, "v", io, (T if kv_rows is None else kv_rows, hkv, d), where)
    _arg(cu_seqlens, "cu_seqlens", (torch.int32,), (None,), where)
    if cu_seqlens.numel() < 1:
        raise ValueError(f"{where}: cu_seqlens needs batch + 1 >= 1 entries")
    _arg(out, "out", (torch.bfloat16,), (T, hq, d), where)
    _arg(lse, "lse", (torch.float32,), (T, hq), where)


def _check_args(params: "Params", where: str, q, k, v, cu_seqlens, out=None, lse=None, kv_rows=None,
                **more) -> None:
    """Layout of every array argument of a compute call, then their device.
    ``more`` holds extra arrays already layout-checked by the caller."""
    params.check(where)
    _qkv_args(params, q, k, v, cu_seqlens, out, lse, where, kv_rows=kv_rows)
    _same_cuda(where, q=q, k=k, v=v, cu_seqlens=cu_seqlens, out=out, lse=lse,
               q_scale=params.q_scale, k_scale=params.k_scale, v_scale=params.v_scale, **more)


@dataclasses.dataclass
class Params:
    """Mirror of ``fp2_params``.  Scales are device tensors (e4m3 only).
    ``correction``: False / 0 none, True / 1 the mean correction, 2 the mean
    correction with the variance term (needs ``BlockMeta.k_var``)."""

    num_q_heads: int
    num_kv_heads: int
    alpha: float = 0.05
    sm_scale: float = 0.0
    correction: int = True
    dtype: int = FP2_BF16
    q_scale: Optional[torch.Tensor] = None
    k_scale: Optional[torch.Tensor] = None
    v_scale: Optional[torch.Tensor] = None
    head_dim: int = HEAD_DIM
    block_size: int = BLOCK

    def check(self, where: str) -> None:
        """Checks the e4m3 scale arrays: fp32 device vectors [Hq], [Hkv], [Hkv]."""
        if self.dtype != FP2_E4M3:
            return
        for name, t, n in (("q_scale", self.q_scale, self.num_q_heads),
                           ("k_scale", self.k_scale, self.num_kv_heads),
                           ("v_scale", self.v_scale, self.num_kv_heads)):
            if t is None:
                raise ValueError(f"{where}: e4m3 inputs need params.{name}")
            _arg(t, name, (torch.float32,), (n,), where)

    def c(self) -> _lib.fp2_params:
        return _lib.fp2_params(self.num_q_heads, self.num_kv_heads, self.head_dim, self.block_size,
                               float(self.alpha), float(self.sm_scale), int(self.correction),
                               int(self.dtype), _ptr(self.q_scale), _ptr(self.k_scale),
                               _ptr(self.v_scale))


def max_blocks(batch: int, total_tokens: int, block_size: int = BLOCK) -> int:
    return int(_lib.load().fp2_max_blocks(batch, total_tokens, block_size))


def workspace_bytes(params: Params, batch: int, total_tokens: int, max_seqlen: int) -> int:
    p = params.c()
    return int(_lib.load().fp2_workspace_bytes(ctypes.byref(p), batch, total_tokens, max_seqlen))


class Workspace:
    """Caller-owned scratch memory of the library (a uint8 device tensor)."""

    def __init__(self, params: Params, batch: int, total_tokens: int, max_seqlen: int,
                 device="cuda", stream=None):
        n = workspace_bytes(params, batch, total_tokens, max_seqlen)
        if n == 0:
            raise FP2Error(1, "fp2_workspace_bytes")
        self.buf = torch.empty(n + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.tensor = self.buf[off:off + n]
        self.nbytes = n
        _check(_lib.load().fp2_workspace_init(_ptr(self.tensor), n, _stream(stream)), "fp2_workspace_init")

    @property
    def ptr(self):
        return _ptr(self.tensor)


@dataclasses.dataclass
class BlockMeta:
    """Mirror of ``fp2_blockmeta``, holding the device tensors."""

    kept_cnt: torch.Tensor
    kept_idx: torch.Tensor
    k_mean: torch.Tensor
    v_mean: Optional[torch.Tensor]
    score_dbg: Optional[torch.Tensor]
    nb_max: int
    max_blocks: int
    k_var: Optional[torch.Tensor] = None   # [max_blocks, Hkv] fp32 mean key variance per block

    @staticmethod
    def empty(params: Params, batch: int, total_tokens: int, max_seqlen: int, device="cuda",
              scores: bool = False, nb_max: Optional[int] = None,
              variance: Optional[bool] = None) -> "BlockMeta":
        """Device arrays for ``total_tokens`` keys.  ``variance`` (default: when
        ``params.correction == 2``) also allocates ``k_var``, which the estimator
        then fills (a little extra work in its pooling pass)."""
        if variance is None:
            variance = int(params.correction) == 2
        mb = max(1, max_blocks(batch, total_tokens))
        nbm = nb_max or max(1, (max_seqlen + BLOCK - 1) // BLOCK)
        hkv = params.num_kv_heads
        return BlockMeta(
            kept_cnt=torch.zeros((mb, hkv), dtype=torch.int32, device=device),
            kept_idx=torch.full((mb, hkv, nbm), -1, dtype=torch.int32, device=device),
            k_mean=torch.zeros((mb, hkv, HEAD_DIM), dtype=torch.float32, device=device),
            v_mean=torch.zeros((mb, hkv, HEAD_DIM), dtype=torch.float32, device=device),
            score_dbg=(torch.full((mb, params.num_q_heads, nbm), float("nan"), dtype=torch.float32,
                                  device=device) if scores else None),
            nb_max=nbm, max_blocks=mb,
            k_var=torch.zeros((mb, hkv), dtype=torch.float32, device=device) if variance else None)

    def c(self) -> _lib.fp2_blockmeta:
        return _lib.fp2_blockmeta(_ptr(self.kept_cnt), _ptr(self.kept_idx), _ptr(self.k_mean),
                                  _ptr(self.v_mean), _ptr(self.score_dbg), self.nb_max, self.max_blocks,
                                  _ptr(self.k_var))


def _bt_args(block_table: Optional[torch.Tensor], num_pages: int):
    if block_table is None:
        return None, 0, 0
    return _ptr(block_table), int(block_table.shape[1]), int(num_pages)


def estimate(params: Params, q, k, v, cu_seqlens, max_seqlen: int, meta: BlockMeta, ws: Workspace,
             block_table: Optional[torch.Tensor] = None, num_pages: int = 0, stream=None) -> None:
    """``fp2_estimate``: kept-block lists and block means into ``meta``."""
    where = "fp2_estimate"
    if cu_seqlens is not None:
        _arg(block_table, "block_table", (torch.int32,), (int(cu_seqlens.numel()) - 1, None), where)
    kv_rows = None if block_table is None else int(num_pages) * params.block_size
    _check_args(params, where, q, k, v, cu_seqlens, kv_rows=kv_rows, block_table=block_table)
    p, m = params.c(), meta.c()
    bt, mbps, npg = _bt_args(block_table, num_pages)
    _check(_lib.load().fp2_estimate(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                    int(cu_seqlens.numel()) - 1, int(q.shape[0]), int(max_seqlen), bt,
                                    mbps, npg, ctypes.byref(m), ws.ptr, ws.nbytes, _stream(stream)),
           "fp2_estimate")


def sparse_prefill(params: Params, q, k, v, cu_seqlens, max_seqlen: int, meta: BlockMeta, out,
                   ws: Workspace, lse=None, stream=None) -> None:
    """``fp2_sparse_prefill``: attention over the kept blocks (+ mean correction)."""
    _check_args(params, "fp2_sparse_prefill", q, k, v, cu_seqlens, out, lse)
    p, m = params.c(), meta.c()
    _check(_lib.load().fp2_sparse_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                          int(cu_seqlens.numel()) - 1, int(q.shape[0]), int(max_seqlen),
                                          ctypes.byref(m), _ptr(out), _ptr(lse), ws.ptr, ws.nbytes,
                                          _stream(stream)),
           "fp2_sparse_prefill")


def prefill_paged(params: Params, q, k_pool, v_pool, cu_seqlens, max_seqlen: int, block_table,
                  num_pages: int, meta: BlockMeta, out, ws: Workspace, lse=None, stream=None) -> None:
    """``fp2_prefill_paged``: ``sparse_prefill`` on a paged KV cache (K/V tiles read
    page by page through ``block_table``).  ``meta`` is only read: fill it with
    ``estimate(..., block_table=block_table, num_pages=num_pages)`` on the same
    pools, or pass kept lists of your own."""
    where = "fp2_prefill_paged"
    if block_table is None:
        raise TypeError(f"{where}: block_table is required")
    if cu_seqlens is not None:
        _arg(block_table, "block_table", (torch.int32,), (int(cu_seqlens.numel()) - 1, None), where)
    _check_args(params, where, q, k_pool, v_pool, cu_seqlens, out, lse,
                kv_rows=int(num_pages) * params.block_size, block_table=block_table)
    p, m = params.c(), meta.c()
    _check(_lib.load().fp2_prefill_paged(ctypes.byref(p), _ptr(q), _ptr(k_pool), _ptr(v_pool),
                                         _ptr(cu_seqlens), int(cu_seqlens.numel()) - 1, int(q.shape[0]),
                                         int(max_seqlen), _ptr(block_table), int(block_table.shape[1]),
                                         int(num_pages), ctypes.byref(m), _ptr(out), _ptr(lse), ws.ptr,
                                         ws.nbytes, _stream(stream)),
           "fp2_prefill_paged")


def sparse_prefill_noalloc(params: Params, q, k, v, cu_seqlens, max_seqlen: int, meta: BlockMeta, out,
                           lse=None, device_status=None, stream=None) -> None:
    """``fp2_sparse_prefill_noalloc``: ``sparse_prefill`` without a workspace,
    for callers that cannot allocate device memory where they run attention
    (the library's own fixed device array serves as scratch).  The first call
    on a device must come before any stream capture on it, and calls that
    overlap on the GPU race on the shared array."""
    where = "fp2_sparse_prefill_noalloc"
    _arg(device_status, "device_status", (torch.int32,), (None,), where)
    _check_args(params, where, q, k, v, cu_seqlens, out, lse, device_status=device_status)
    p, m = params.c(), meta.c()
    _check(_lib.load().fp2_sparse_prefill_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                                  int(cu_seqlens.numel()) - 1, int(q.shape[0]),
                                                  int(max_seqlen), ctypes.byref(m), _ptr(out), _ptr(lse),
                                                  _ptr(device_status), _stream(stream)),
           "fp2_sparse_prefill_noalloc")


def _chunk_args(params: Params, where: str, q, k, v, cu_q, cu_k, total_k: int, out=None, lse=None,
                block_table=None, num_pages: int = 0):
    """Layouts of a chunked call: q / out / lse [total_q, ...], k / v [total_k, Hkv, d] (or page
    pools), cu_seqlens_q and cu_seqlens_k [batch + 1] int32; then the device."""
    for name, t in (("cu_seqlens_q", cu_q), ("cu_seqlens_k", cu_k)):
        if t is None:
            raise TypeError(f"{where}: {name} is required")
        _arg(t, name, (torch.int32,), (None,), where)
    if cu_q.numel() != cu_k.numel() or cu_q.numel() < 1:
        raise ValueError(f"{where}: cu_seqlens_q and cu_seqlens_k need the same batch + 1 >= 1 entries")
    _arg(block_table, "block_table", (torch.int32,), (int(cu_q.numel()) - 1, None), where)
    params.check(where)
    io = (torch.bfloat16,) if params.dtype == FP2_BF16 else _E4M3_DTYPES
    d, hq, hkv = params.head_dim, params.num_q_heads, params.num_kv_heads
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            raise TypeError(f"{where}: {name} is required")
    _arg(q, "q", io, (None, hq, d), where)
    rows = None if block_table is None else int(num_pages) * params.block_size
    _arg(k, "k", io, (rows, hkv, d), where)
    _arg(v, "v", io, (int(k.shape[0]), hkv, d), where)
    Tq = int(q.shape[0])
    _arg(out, "out", (torch.bfloat16,), (Tq, hq, d), where)
    _arg(lse, "lse", (torch.float32,), (Tq, hq), where)
    if block_table is None and int(total_k) != int(k.shape[0]):
        raise ValueError(f"{where}: total_k = {total_k} but k has {k.shape[0]} rows")
    _same_cuda(where, q=q, k=k, v=v, cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, out=out, lse=lse,
               block_table=block_table, q_scale=params.q_scale, k_scale=params.k_scale, v_scale=params.v_scale)


def estimate_chunked(params: Params, q, k, v, cu_seqlens_q, cu_seqlens_k, total_k: int, max_seqlen_k: int,
                     meta: BlockMeta, ws: Workspace, block_table: Optional[torch.Tensor] = None,
                     num_pages: int = 0, stream=None) -> None:
    """``fp2_estimate_chunked``: kept lists of the chunk's q-blocks (and the key-block
    means of all keys) into ``meta``.  ``total_k`` = cu_seqlens_k[-1] (the keys of the
    batch; with contiguous K/V, k.shape[0])."""
    where = "fp2_estimate_chunked"
    _chunk_args(params, where, q, k, v, cu_seqlens_q, cu_seqlens_k, total_k, block_table=block_table,
                num_pages=num_pages)
    p, m = params.c(), meta.c()
    bt, mbps, npg = _bt_args(block_table, num_pages)
    _check(_lib.load().fp2_estimate_chunked(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q),
                                            _ptr(cu_seqlens_k), int(cu_seqlens_q.numel()) - 1, int(q.shape[0]),
                                            int(total_k), int(max_seqlen_k), bt, mbps, npg, ctypes.byref(m),
                                            ws.ptr, ws.nbytes, _stream(stream)),
           where)


def prefill_chunked(params: Params, q, k, v, cu_seqlens_q, cu_seqlens_k, total_k: int, max_seqlen_k: int,
                    meta: BlockMeta, out, ws: Workspace, lse=None, block_table: Optional[torch.Tensor] = None,
                    num_pages: int = 0, stream=None) -> None:
    """``fp2_prefill_chunked``: attention of the chunk rows over the kept blocks of all
    keys (+ mean correction), contiguous K/V or page pools through ``block_table``."""
    where = "fp2_prefill_chunked"
    _chunk_args(params, where, q, k, v, cu_seqlens_q, cu_seqlens_k, total_k, out, lse, block_table, num_pages)
    p, m = params.c(), meta.c()
    bt, mbps, npg = _bt_args(block_table, num_pages)
    _check(_lib.load().fp2_prefill_chunked(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens_q),
                                           _ptr(cu_seqlens_k), int(cu_seqlens_q.numel()) - 1, int(q.shape[0]),
                                           int(total_k), int(max_seqlen_k), bt, mbps, npg, ctypes.byref(m),
                                           _ptr(out), _ptr(lse), ws.ptr, ws.nbytes, _stream(stream)),
           where)


def get_error(ws: Workspace, stream=None) -> int:
    """``fp2_get_error``: device-side status since the last read (synchronises)."""
    return int(_lib.load().fp2_get_error(ws.ptr, _stream(stream)))


def status_string(code: int) -> str:
    return _lib.load().fp2_status_string(int(code)).decode()


def version() -> int:
    return int(_lib.load().fp2_version())

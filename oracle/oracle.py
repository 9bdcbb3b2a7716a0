"""Python face of the CPU oracle (``fp2_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg are the only callers.  Nothing here imports the CUDA package, and
the CUDA package never imports this module.

Definitions D0-D4 are stated in the header of ``fp2_oracle.c`` with the
passages of the FlashPrefill V2 write-ups they follow.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp2_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_lock = threading.Lock()
_cache = {}


def lib_path(mutant: int = 0, fp32: bool = False) -> str:
    if fp32:
        return os.path.join(_BUILD, "liboracle_fp32.so")
    return os.path.join(_BUILD, "liboracle.so" if mutant == 0 else f"liboracle_mut{mutant}.so")


def build(mutant: int = 0, force: bool = False, fp32: bool = False) -> str:
    """Compile the oracle with gcc (IEEE double, OpenMP; ``fp32``: the same code in
    float, the timed CPU baseline's build). Returns the .so path."""
    out = lib_path(mutant, fp32)
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
               f"-DORC_MUTANT={mutant}", *(["-DORC_FP32"] if fp32 else []), _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64


def _load(mutant: int = 0, fp32: bool = False):
    key = (mutant, fp32)
    _D = ctypes.c_float if fp32 else ctypes.c_double   # the oracle's `real` scalars
    with _lock:
        if key in _cache:
            return _cache[key]
        lib = ctypes.CDLL(build(mutant, fp32=fp32))
        lib.orc_total_blocks.argtypes = [_P, _P, _I, _I]
        lib.orc_total_blocks.restype = _L
        lib.orc_block_means.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _P]
        lib.orc_block_means.restype = None
        lib.orc_estimate.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _D, _D, _I, _P, _P, _P, _P]
        lib.orc_estimate.restype = _I
        lib.orc_block_vars.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
        lib.orc_block_vars.restype = None
        lib.orc_attend.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _D, _P, _P, _I,
                                   _I, _P, _P, _P, _P, _P, _L, _P, _P, _P]
        lib.orc_attend.restype = _I
        lib.orc_mutant_id.restype = _I
        _cache[key] = lib
        return lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _i64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int64)


def chunk_starts(cu_seqlens_q, cu_seqlens_k) -> np.ndarray:
    """D0 chunked form: position P_b = Lk_b - Lq_b of every request's first query row."""
    lq, lk = np.diff(_i32(cu_seqlens_q)).astype(np.int64), np.diff(_i32(cu_seqlens_k)).astype(np.int64)
    if lq.shape != lk.shape or (lq < 0).any() or (lq > lk).any():
        raise ValueError("every request needs 0 <= query rows <= keys")
    return lk - lq


class Oracle:
    """fp64 CPU reference of the estimator (D1, D2) and the attention (D3)."""

    def __init__(self, mutant: int = 0, fp32: bool = False):
        """``fp32``: the float build of the same code (the timed CPU baseline only;
        every parity check uses the double build)."""
        self.lib = _load(mutant, fp32)
        self.mutant = mutant
        self.real = np.float32 if fp32 else np.float64

    def _r(self, a):
        return np.ascontiguousarray(a, dtype=self.real)

    # D0
    def total_blocks(self, cu_seqlens, block_size: int, pos0=None) -> int:
        """Blocks of a batch; request b's rows start at position pos0[b] (None: 0)."""
        cu, p0 = _i32(cu_seqlens), _i64(pos0)
        return int(self.lib.orc_total_blocks(_ptr(cu), _ptr(p0), len(cu) - 1, block_size))

    # D1
    def block_means(self, x, cu_seqlens, block_size: int, scale=None, pos0=None) -> np.ndarray:
        """x: [T, H, d] stored values; scale: [H] dequantisation scales; pos0: [B]
        position of every request's first row (None: 0; query rows of a chunk:
        ``chunk_starts(cu_q, cu_k)``)."""
        x = _f32(x)
        T, H, d = x.shape
        cu, p0 = _i32(cu_seqlens), _i64(pos0)
        sc = self._r(np.ones(H) if scale is None else scale)
        out = np.zeros((self.total_blocks(cu, block_size, p0), H, d), self.real)
        self.lib.orc_block_means(_ptr(x), _ptr(sc), _ptr(cu), _ptr(p0), len(cu) - 1, H, d, block_size,
                                 _ptr(out))
        return out

    def block_vars(self, x, cu_seqlens, block_size: int, mean, scale=None, pos0=None) -> np.ndarray:
        """Per-dimension variance of the dequantised rows inside every block around
        ``mean`` (``block_means`` of the same arguments); the D3 variance variant."""
        x = _f32(x)
        T, H, d = x.shape
        cu, p0, mean = _i32(cu_seqlens), _i64(pos0), self._r(mean)
        sc = self._r(np.ones(H) if scale is None else scale)
        out = np.zeros_like(mean)
        self.lib.orc_block_vars(_ptr(x), _ptr(sc), _ptr(cu), _ptr(p0), len(cu) - 1, H, d, block_size,
                                _ptr(mean), _ptr(out))
        return out

    # D1 + D2
    def estimate(self, qbar, kbar, cu_seqlens, block_size: int, alpha: float, tau: float,
                 nb_max: Optional[int] = None, want_scores: bool = False, cu_seqlens_k=None):
        """Returns dict(kept_cnt [nb, Hkv], kept_idx [nb, Hkv, nb_max], s, m).
        ``cu_seqlens`` counts query rows, ``cu_seqlens_k`` keys (None: the same,
        plain prefill); nb counts q-blocks."""
        qbar, kbar, cu = self._r(qbar), self._r(kbar), _i32(cu_seqlens)
        cuk = cu if cu_seqlens_k is None else _i32(cu_seqlens_k)
        nblk, Hq, d = qbar.shape
        Hkv = kbar.shape[1]
        lens = np.diff(cuk)
        if nb_max is None:
            nb_max = max(1, int(max([(int(L) + block_size - 1) // block_size for L in lens] or [1])))
        cnt = np.zeros((nblk, Hkv), np.int32)
        idx = np.full((nblk, Hkv, nb_max), -1, np.int32)
        s = np.full((nblk, Hq, nb_max), np.nan, self.real) if want_scores else None
        m = np.full((nblk, Hq), np.nan, self.real) if want_scores else None
        rc = self.lib.orc_estimate(_ptr(qbar), _ptr(kbar), _ptr(cu), _ptr(cuk), len(cu) - 1, Hq, Hkv, d,
                                   block_size, tau, alpha, nb_max, _ptr(cnt), _ptr(idx), _ptr(s), _ptr(m))
        if rc != 0:
            raise ValueError(f"orc_estimate failed: {rc}")
        return {"kept_cnt": cnt, "kept_idx": idx, "s": s, "m": m, "nb_max": nb_max}

    # D3
    def attend(self, q, k, v, cu_seqlens, block_size: int, tau: float, kept_cnt, kept_idx,
               correction: bool = False, kbar=None, vbar=None, q_scale=None, k_scale=None,
               v_scale=None, sel=None, want_wsum: bool = False, cu_seqlens_k=None, kvar=None, qbar=None):
        """Returns dict(o [T, Hq, d], lse [T, Hq], wsum). Rows outside ``sel`` stay NaN.
        ``cu_seqlens_k`` (None: ``cu_seqlens``) gives the keys of every request
        when only its last query rows are computed (D0 chunked form).
        ``correction``: False/0 none, True/1 the mean correction (D3); the D3
        variants 2 (with the variance term, needs ``kvar``), 3 (block-pooled,
        needs ``qbar``) and 4 (the variance averaged over the dimensions, needs
        ``kvar``) are for approximation studies."""
        q, k, v, cu = _f32(q), _f32(k), _f32(v), _i32(cu_seqlens)
        cuk = cu if cu_seqlens_k is None else _i32(cu_seqlens_k)
        T, Hq, d = q.shape
        Hkv = k.shape[1]
        kept_cnt, kept_idx = _i32(kept_cnt), _i32(kept_idx)
        nb_max = kept_idx.shape[2]
        qs = self._r(np.ones(Hq) if q_scale is None else q_scale)
        ks = self._r(np.ones(Hkv) if k_scale is None else k_scale)
        vs = self._r(np.ones(Hkv) if v_scale is None else v_scale)
        mode = int(correction)
        if mode:
            kbar, vbar = self._r(kbar), self._r(vbar)
        kvar = None if mode not in (2, 4) else self._r(kvar)
        qbar = None if mode != 3 else self._r(qbar)
        o = np.full((T, Hq, d), np.nan, self.real)
        lse = np.full((T, Hq), np.nan, self.real)
        ws = np.full((T, Hq), np.nan, self.real) if want_wsum else None
        selv = None if sel is None else np.ascontiguousarray(sel, dtype=np.int64)
        rc = self.lib.orc_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(qs), _ptr(ks), _ptr(vs), _ptr(cu),
                                 _ptr(cuk), len(cu) - 1, Hq, Hkv, d, block_size, tau, _ptr(kept_cnt),
                                 _ptr(kept_idx), nb_max, mode,
                                 _ptr(kbar) if mode else None, _ptr(vbar) if mode else None,
                                 _ptr(kvar), _ptr(qbar), _ptr(selv), 0 if selv is None else len(selv), _ptr(o), _ptr(lse), _ptr(ws))
        if rc != 0:
            raise ValueError(f"orc_attend failed: {rc}")
        return {"o": o, "lse": lse, "wsum": ws}

    # whole path for a workload
    def run(self, wl, alpha: Optional[float] = None, correction: bool = True, sel=None,
            want_scores: bool = False, tau: Optional[float] = None, kept=None):
        """Estimate (unless ``kept`` is given) then attend, on a ``workloads.Workload``
        (chunked workloads: queries are the last ``query_lens[b]`` tokens of each request)."""
        q, k, v = wl.float_inputs()
        cu = wl.cu_seqlens                              # keys
        chunked = getattr(wl, "query_lens", None) is not None
        cu_q = wl.cu_seqlens_q if chunked else cu      # query rows
        pos0 = chunk_starts(cu_q, cu) if chunked else None
        bs = wl.block_size
        tau = 1.0 / math.sqrt(wl.head_dim) if tau is None else tau
        a = wl.alpha if alpha is None else alpha
        qbar = self.block_means(q, cu_q, bs, wl.q_scale, pos0=pos0)
        kbar = self.block_means(k, cu, bs, wl.k_scale)
        vbar = self.block_means(v, cu, bs, wl.v_scale)
        est = kept if kept is not None else self.estimate(qbar, kbar, cu_q, bs, a, tau, want_scores=want_scores,
                                                          cu_seqlens_k=cu)
        att = self.attend(q, k, v, cu_q, bs, tau, est["kept_cnt"], est["kept_idx"], correction=correction,
                          kbar=kbar, vbar=vbar, q_scale=wl.q_scale, k_scale=wl.k_scale,
                          v_scale=wl.v_scale, sel=sel, cu_seqlens_k=cu)
        return {**est, **att, "qbar": qbar, "kbar": kbar, "vbar": vbar}


def near_threshold(s, m, kept_shape_groups: int, alpha: float, nb_per_block, rel: float = 1e-3):
    """Group-level near-threshold flags [nb, Hkv, nb_max] (any head of the group
    within ``rel * max(1, |m + ln alpha|)`` of the threshold)."""
    nblk, Hq, nb_max = s.shape
    G = Hq // kept_shape_groups
    if alpha <= 0:
        return np.zeros((nblk, kept_shape_groups, nb_max), bool)
    thr = m + math.log(alpha)                       # [nb, Hq]
    band = rel * np.maximum(1.0, np.abs(thr))
    with np.errstate(invalid="ignore"):
        near = np.abs(s - thr[:, :, None]) <= band[:, :, None]
    near &= ~np.isnan(s)
    return near.reshape(nblk, kept_shape_groups, G, nb_max).any(axis=2)

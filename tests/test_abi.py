"""The C ABI on the host (no GPU): the library builds, loads and exports every
function include/fp2.h declares, and argument checks fail before any launch."""
import ctypes
import os
import re

import pytest

from block_sparse_prefill_b200 import _lib
from block_sparse_prefill_b200 import build as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp2.h")


@pytest.fixture(scope="module")
def lib():
    b.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp2_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_function(lib):
    names = declared_functions()
    assert set(names) == set(_lib.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), f"missing symbol {n}"


def _params(**kw):
    p = dict(num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=128, alpha=0.05, sm_scale=0.0,
             correction=1, dtype=0, q_scale=None, k_scale=None, v_scale=None)
    p.update(kw)
    return _lib.fp2_params(**p)


def test_sizes(lib):
    assert lib.fp2_max_blocks(1, 131072, 128) == 1025
    assert lib.fp2_max_blocks(8, 1000, 128) == 15
    p = _params()
    n = lib.fp2_workspace_bytes(ctypes.byref(p), 1, 131072, 131072)
    # q-block means dominate: 1025 blocks x 32 heads x 128 x fp32
    assert n >= 1025 * 32 * 128 * 4 and n % 256 == 0
    assert lib.fp2_workspace_bytes(ctypes.byref(_params(num_kv_heads=3)), 1, 100, 100) == 0
    assert lib.fp2_workspace_bytes(None, 1, 100, 100) == 0


def test_status_strings(lib):
    for code in range(7):
        assert lib.fp2_status_string(code)
    assert lib.fp2_version() >= 100


def _estimate(lib, p, **kw):
    a = dict(q=ctypes.c_void_p(4096), k=ctypes.c_void_p(4096), v=ctypes.c_void_p(4096),
             cu=ctypes.c_void_p(4096), batch=1, T=1024, S=1024, bt=None, mbps=0, npages=0,
             ws=ctypes.c_void_p(1 << 20), wsb=1 << 40)
    a.update(kw)
    m = kw.get("meta", _lib.fp2_blockmeta(4096, 4096, 4096, 4096, None, 8, 9))
    return lib.fp2_estimate(ctypes.byref(p) if p is not None else None, a["q"], a["k"], a["v"], a["cu"],
                            a["batch"], a["T"], a["S"], a["bt"], a["mbps"], a["npages"],
                            ctypes.byref(m) if m is not None else None, a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(num_q_heads=0), 1),
    (dict(num_q_heads=6, num_kv_heads=4), 1),
    (dict(head_dim=64), 2),
    (dict(block_size=64), 2),
    (dict(alpha=1.5), 1),
    (dict(alpha=float("nan")), 1),
    (dict(sm_scale=-1.0), 1),
    (dict(correction=2), 1),
    (dict(dtype=7), 1),
    (dict(dtype=1), 1),          # e4m3 without scales
])
def test_bad_params_rejected(lib, kw, code):
    assert _estimate(lib, _params(**kw)) == code


def test_bad_problem_rejected(lib):
    p = _params()
    assert _estimate(lib, None) == 1
    assert _estimate(lib, p, batch=-1) == 1
    assert _estimate(lib, p, cu=None) == 1
    assert _estimate(lib, p, q=None) == 1
    assert _estimate(lib, p, q=ctypes.c_void_p(4097)) == 1           # not 16-byte aligned
    assert _estimate(lib, p, ws=None) == 3
    assert _estimate(lib, p, ws=ctypes.c_void_p((1 << 20) + 8)) == 3  # not 256-byte aligned
    assert _estimate(lib, p, wsb=100) == 3
    assert _estimate(lib, p, meta=None) == 1
    small = _lib.fp2_blockmeta(4096, 4096, 4096, 4096, None, 4, 9)     # nb_max < ceil(1024/128)
    assert _estimate(lib, p, meta=small) == 1
    assert _estimate(lib, p, bt=ctypes.c_void_p(4096), mbps=0, npages=4) == 1
    # page rows (page x 128) must fit the kernels' int32 coordinates
    assert _estimate(lib, p, bt=ctypes.c_void_p(4096), mbps=8, npages=(1 << 24) + 1) == 2


def test_workspace_init_checks(lib):
    assert lib.fp2_workspace_init(None, 1024, None) == 3
    assert lib.fp2_workspace_init(ctypes.c_void_p(4100), 1024, None) == 3
    assert lib.fp2_get_error(None, None) == 3

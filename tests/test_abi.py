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
    (dict(correction=3), 1),
    (dict(correction=-1), 1),
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


PROBE_DIR = os.path.join(ROOT, "tests", "_build")


def _c_probe(name: str, body: str) -> str:
    """Compiles and runs a small C program against include/fp2.h (gcc, host only),
    built in the git-ignored tests/_build folder."""
    import subprocess
    os.makedirs(PROBE_DIR, exist_ok=True)
    src = os.path.join(PROBE_DIR, f"{name}_{os.getpid()}.c")
    exe = src[:-2]
    with open(src, "w") as f:
        f.write('#include <stdio.h>\n#include <stddef.h>\n#include "fp2.h"\n'
                "int main(void) {\n" + body + "return 0;\n}\n")
    try:
        subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), src, "-o", exe],
                       check=True)
        return subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    finally:
        for f in (src, exe):
            if os.path.exists(f):
                os.remove(f)


@pytest.mark.parametrize("struct", ["fp2_params", "fp2_blockmeta"])
def test_struct_mirrors_match_the_header(struct):
    """Every field of the ctypes mirror sits at the C offset with the C size."""
    mirror = getattr(_lib, struct)
    body = f'printf("sizeof %zu\\n", sizeof({struct}));\n'
    for name, _ in mirror._fields_:
        body += (f'printf("{name} %zu %zu\\n", offsetof({struct}, {name}), '
                 f'sizeof((({struct}*)0)->{name}));\n')
    rows = dict((ln.split()[0], ln.split()[1:]) for ln in _c_probe(struct, body).splitlines())
    assert int(rows.pop("sizeof")[0]) == ctypes.sizeof(mirror)
    for name, _ in mirror._fields_:
        off, size = (int(x) for x in rows[name])
        field = getattr(mirror, name)
        assert (field.offset, field.size) == (off, size), name
    # the C struct has no field the mirror lacks: the last field ends the struct
    last = getattr(mirror, mirror._fields_[-1][0])
    assert last.offset + last.size == ctypes.sizeof(mirror)


def test_enum_values_match_the_header():
    names = list(_lib.STATUS.values()) + ["FP2_BF16", "FP2_E4M3"]
    body = "".join(f'printf("{n} %d\\n", (int){n});\n' for n in names)
    vals = {ln.split()[0]: int(ln.split()[1]) for ln in _c_probe("enums", body).splitlines()}
    assert {v: k for k, v in _lib.STATUS.items()} == {n: vals[n] for n in _lib.STATUS.values()}
    assert (vals["FP2_BF16"], vals["FP2_E4M3"]) == (_lib.FP2_BF16, _lib.FP2_E4M3)


def _c_width(decl: str):
    """('ptr', 8) for pointers, else (C type name, byte width) of a declaration."""
    decl = re.sub(r"\bconst\b", "", decl).strip()
    if "*" in decl:
        return ("ptr", 8)
    base = decl.split()[0]
    widths = {"int32_t": 4, "int64_t": 8, "size_t": 8, "int": 4, "fp2_status": 4}
    return (base, widths[base])


def test_prototypes_match_the_ctypes_declarations(lib):
    """Each header prototype: ctypes declares as many arguments, each pointer as a
    pointer and each integer with the C width, and the matching result type."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"^\s*#.*$", "", text, flags=re.M)          # preprocessor lines
    protos = re.findall(r"([A-Za-z_][\w\s\*]*?)\b(fp2_[a-z_]+)\s*\(([^)]*)\)\s*;", text)
    assert {name for _, name, _ in protos} == set(_lib.EXPORTS)
    for ret, name, args in protos:
        fn = getattr(lib, name)
        params = [a.strip() for a in args.split(",") if a.strip() and a.strip() != "void"]
        assert len(fn.argtypes) == len(params), name
        for decl, ct in zip(params, fn.argtypes):
            kind, width = _c_width(decl)
            if kind == "ptr":
                assert ct is ctypes.c_void_p or ct is ctypes.c_char_p or issubclass(ct, ctypes._Pointer), \
                    (name, decl)
            else:
                assert ctypes.sizeof(ct) == width, (name, decl)
                assert (ct(-1).value < 0) == (kind != "size_t"), (name, decl)
        rkind, rwidth = _c_width(ret)
        if rkind == "ptr":
            assert fn.restype is ctypes.c_char_p, name
        else:
            assert ctypes.sizeof(fn.restype) == rwidth, name


def _max_seq_blocks():
    text = open(HEADER).read()
    return {name: int(re.search(rf"#define FP2_MAX_SEQ_BLOCKS_{name}\s+(\d+)", text).group(1))
            for name in ("BF16", "E4M3", "VAR_BF16", "VAR_E4M3")}


def _attention_call(lib, fn, dtype, max_seqlen, correction=1):
    """An attention call with fake (never dereferenced) device addresses."""
    sc = 4096 if dtype else None
    p = _lib.fp2_params(32, 8, 128, 128, 0.05, 0.0, correction, dtype, sc, sc, sc)
    nb = (max_seqlen + 127) // 128
    m = _lib.fp2_blockmeta(4096, 4096, 4096, 4096, None, nb, nb + 1, 4096)
    a = ctypes.c_void_p(4096)
    if fn == "fp2_prefill_paged":
        return lib.fp2_prefill_paged(ctypes.byref(p), a, a, a, a, 1, max_seqlen, max_seqlen, a, nb, nb,
                                     ctypes.byref(m), a, None, ctypes.c_void_p(1 << 20), 1 << 40, None)
    return lib.fp2_sparse_prefill(ctypes.byref(p), a, a, a, a, 1, max_seqlen, max_seqlen, ctypes.byref(m),
                                  a, None, ctypes.c_void_p(1 << 20), 1 << 40, None)


LIMITS = [(0, "BF16", 1), (1, "E4M3", 1), (0, "VAR_BF16", 2), (1, "VAR_E4M3", 2)]


@pytest.mark.parametrize("fn", ["fp2_sparse_prefill", "fp2_prefill_paged"])
@pytest.mark.parametrize("dtype,name,corr", LIMITS)
def test_length_limit_rejected_before_any_launch(lib, fn, dtype, name, corr):
    """One block past the documented limit returns FP2_ERR_UNSUPPORTED before anything
    is enqueued."""
    limit = _max_seq_blocks()[name]
    assert _attention_call(lib, fn, dtype, limit * 128 + 1, corr) == 2


@pytest.mark.skipif(__import__("torch").cuda.is_available(),
                    reason="the accepted call would launch kernels on fake addresses")
@pytest.mark.parametrize("dtype,name,corr", LIMITS)
def test_length_limit_is_tight(lib, dtype, name, corr):
    """At the documented limit every host check passes: without a GPU the call
    gets as far as the first CUDA call and returns FP2_ERR_CUDA."""
    limit = _max_seq_blocks()[name]
    assert _attention_call(lib, "fp2_sparse_prefill", dtype, limit * 128, corr) == 4


def test_missing_library_fails_loudly(monkeypatch):
    """Without libfp2.so every call raises: there is no CPU fallback."""
    import block_sparse_prefill_b200 as fp2
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", os.path.join(ROOT, "tests", "_build", "absent", "libfp2.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        fp2.max_blocks(1, 1024)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        fp2.workspace_bytes(fp2.Params(num_q_heads=4, num_kv_heads=2), 1, 1024, 1024)


def test_plain_c_client_links_and_calls_the_library(lib):
    """A C11 program built with gcc against include/fp2.h links libfp2.so and calls
    the host-only entry points and an argument-error path (no device work)."""
    import subprocess
    os.makedirs(PROBE_DIR, exist_ok=True)
    src = os.path.join(PROBE_DIR, f"c_client_{os.getpid()}.c")
    exe = src[:-2]
    libdir = os.path.dirname(_lib.LIB_PATH)
    with open(src, "w") as f:
        f.write('#include <stdio.h>\n#include "fp2.h"\nint main(void) {\n'
                "    fp2_params p = {32, 8, 128, 128, 0.05f, 0.0f, 1, FP2_BF16, NULL, NULL, NULL};\n"
                '    printf("%d %lld %d %d %s\\n", fp2_version(), (long long)fp2_max_blocks(1, 131072, 128),\n'
                "           fp2_workspace_bytes(&p, 1, 131072, 131072) > 0,\n"
                "           (int)fp2_estimate(NULL, NULL, NULL, NULL, NULL, 0, 0, 0, NULL, 0, 0, NULL, NULL, 0, NULL),\n"
                "           fp2_status_string(FP2_ERR_INVALID_ARG));\n"
                "    return 0;\n}\n")
    try:
        subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), src,
                        "-L", libdir, "-l:libfp2.so", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
        out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split()
    finally:
        for f in (src, exe):
            if os.path.exists(f):
                os.remove(f)
    assert out[:4] == [str(lib.fp2_version()), "1025", "1", "1"], out
    assert " ".join(out[4:]) == "invalid argument"


def test_variance_correction_needs_k_var(lib):
    """correction = 2 reads the block key variances: an attention call whose meta has no
    k_var is an argument error (nothing enqueued); the estimator does not need it."""
    p = _params(correction=2)
    a = ctypes.c_void_p(4096)
    m = _lib.fp2_blockmeta(4096, 4096, 4096, 4096, None, 8, 9)      # k_var NULL
    assert lib.fp2_sparse_prefill(ctypes.byref(p), a, a, a, a, 1, 1024, 1024, ctypes.byref(m), a, None,
                                  ctypes.c_void_p(1 << 20), 1 << 40, None) == 1

"""The C ABI library builds, loads without a GPU and exports every declared entry point."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "prism.h")


@pytest.fixture(scope="module")
def lib():
    from dynamic_block_sparse_indicator_b200 import build, _lib
    build.build_library()
    return _lib.load()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"PRISM_API\s+[\w\s\*]+?\b(prism_\w+)\s*\(", txt)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ("prism_plan", "prism_attn_fwd", "prism_attn_bwd", "prism_plan_workspace_bytes"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in declared_symbols():
        assert hasattr(lib, s), s


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.prism_version()
    from dynamic_block_sparse_indicator_b200 import _lib
    assert _lib.status_string(0) == "ok"
    assert "workspace" in _lib.status_string(2)
    assert _lib.status_string(99) == "unknown status"


def _params(**kw):
    from dynamic_block_sparse_indicator_b200 import _lib
    base = dict(T=8, H=16, W=16, heads=2, head_dim=64, dtype=_lib.PRISM_F32, top_k=4, top_p=0.9,
                eps=1e-6)
    base.update(kw)
    return _lib.make_params(**base)


def test_workspace_bytes_and_validation(lib):
    from dynamic_block_sparse_indicator_b200 import _lib
    n = _lib.workspace_bytes(_params())
    assert n > 0
    # grows with heads; invalid problems give 0
    assert _lib.workspace_bytes(_params(heads=4)) > n
    for bad in (dict(T=12), dict(H=0), dict(head_dim=96), dict(top_k=0, top_p=0.0),
                dict(top_p=1.5), dict(top_p=float("nan")), dict(eps=0.0), dict(dtype=7), dict(out_dtype=3),
                dict(heads=0), dict(tau128=0.1, tau256=0.2)):
        assert _lib.workspace_bytes(_params(**bad)) == 0, bad


def test_invalid_calls_return_status_without_device(lib):
    from dynamic_block_sparse_indicator_b200 import _lib
    p = _params(T=12)
    h = C.c_void_p()
    dummy = C.c_void_p(256)
    st = lib.prism_plan(C.byref(p), dummy, dummy, dummy, None, dummy, 1 << 20, None, C.byref(h))
    assert st == _lib.PRISM_ERR_INVALID_ARG and not h.value
    p = _params()
    st = lib.prism_plan(C.byref(p), None, dummy, dummy, None, dummy, 1 << 20, None, C.byref(h))
    assert st == _lib.PRISM_ERR_INVALID_ARG
    assert lib.prism_attn_fwd(None, dummy, dummy, None) == _lib.PRISM_ERR_INVALID_ARG
    assert lib.prism_attn_bwd(None, dummy, dummy, dummy, dummy, dummy, dummy, None) == \
        _lib.PRISM_ERR_INVALID_ARG
    assert lib.prism_get_status(None, None) == _lib.PRISM_ERR_INVALID_ARG
    lib.prism_plan_destroy(None)


def test_no_cpu_fallback_in_package():
    """The package never imports the oracle (test infrastructure only)."""
    pkg = os.path.join(ROOT, "dynamic_block_sparse_indicator_b200")
    for dp, _, fs in os.walk(pkg):
        for f in fs:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dp, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f


def test_av_norm_validation_without_device(lib):
    """prism_av_norm rejects bad sizes, dtypes and pointers before touching a device."""
    from dynamic_block_sparse_indicator_b200 import _lib
    d = C.c_void_p(256)
    odd = C.c_void_p(264)

    def call(N=2048, M=100, heads=2, D=64, q=d, k=d, v=d, a=d, hh=None, hdt=_lib.PRISM_BF16, st=d):
        return lib.prism_av_norm(N, M, heads, D, q, k, v, a, hh, hdt, st, None)

    for bad in (dict(N=0), dict(N=1 << 31), dict(M=0), dict(M=(1 << 20) + 1), dict(heads=0),
                dict(D=96), dict(hdt=5), dict(q=None), dict(k=None), dict(v=None), dict(a=None),
                dict(st=None), dict(q=odd), dict(a=odd), dict(hh=odd), dict(st=odd)):
        assert call(**bad) == _lib.PRISM_ERR_INVALID_ARG, bad
    assert lib.prism_status_read(None, None, None) == _lib.PRISM_ERR_INVALID_ARG

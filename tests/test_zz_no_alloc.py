"""prism_zone_shapes_noalloc: stage 1 for callers that cannot allocate device memory.

Such callers (a plugin confined to another engine's memory plan, a path where
cudaMalloc's implicit synchronisation is not acceptable, a fixed memory budget)
get the shape ids and block counts from an entry point whose scratch is a
static device array.  This file runs last: it checks, through the C ABI, that
two calls in a row give exactly the shapes and block counts of prism_plan,
which computes them in the caller's workspace.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32_d64": (syn.workload(0), 2, True),
    "grid16x32x32_bf16_d128": (syn.workload(2, T=16, H=32, W=32), 2, True),
    "grid8x16x24_no_audio": (syn.workload(1, T=8, H=16, W=24), 3, False),
}


def _params(w, heads):
    code = _lib.PRISM_F32 if w.dtype == "f32" else _lib.PRISM_BF16
    return _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, code, w.top_k, w.top_p, w.eps)


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_shapes_match_plan(name, cuda_device):
    w, heads, audio = CASES[name]
    Q, K, V = (x.cuda() for x in syn.make_qkv(w, heads=heads))
    a = syn.make_amap(w).cuda() if audio else None
    p = _params(w, heads)
    pl = _lib.plan(Q, K, V, a, p)
    want_sid = pl.export("shape_id")
    want_nb = pl.export("nblocks")
    lib = _lib.load()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):                              # two calls in a row share the scratch
        sid = torch.full((heads * w.zones,), 255, dtype=torch.uint8, device="cuda")
        nb = torch.full((heads,), -1, dtype=torch.int32, device="cuda")
        st = lib.prism_zone_shapes_noalloc(C.byref(p), C.c_void_p(V.data_ptr()),
                                           None if a is None else C.c_void_p(a.data_ptr()),
                                           C.c_void_p(sid.data_ptr()), C.c_void_p(nb.data_ptr()), stream)
        assert st == _lib.PRISM_OK, _lib.status_string(st)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(sid.cpu().numpy(), want_sid)
        np.testing.assert_array_equal(nb.cpu().numpy(), want_nb)


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_device):
    w = syn.workload(3)
    p = _lib.make_params(w.T, w.H, w.W, 200, 128, _lib.PRISM_BF16, 16, 0.9, 1e-4)
    lib = _lib.load()
    dummy = C.c_void_p(1 << 20)
    st = lib.prism_zone_shapes_noalloc(C.byref(p), dummy, None, dummy, dummy, None)
    assert st == _lib.PRISM_ERR_SCRATCH_LIMIT
    assert "scratch" in _lib.status_string(st)

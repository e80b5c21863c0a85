"""The bounds-checking build (libprism_checks.so, -DPRISM_CHECKS=1) on the GPU.

Every gather, scatter and list index of that build is checked on the device
(a failed check records PRISM_ERR_DEVICE_CHECK and skips the access).  A child
process loads it through PRISM_LIB and runs plan, forward and backward of two
workloads (the tiny fp32 head_dim-64 one and a 16x32x32 bf16 grid with adaptive
temporal boundaries on): no check fires, and the outputs equal those of the
default build (O and LSE bit for bit; the gradients to fp32 summation order).
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import build as pbuild
from dynamic_block_sparse_indicator_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
out = {}
for name, w, cut in (("tiny", syn.workload(0), 0.0),
                     ("cuts", syn.workload(2, T=16, H=32, W=32, shot_cuts=[12]), 2.5)):
    Q, K, V = (x.cuda() for x in syn.make_qkv(w, heads=2))
    a = syn.make_amap(w).cuda()
    dt = _lib.PRISM_F32 if w.dtype == "f32" else _lib.PRISM_BF16
    dO = syn.make_dout(w, heads=2, out_dtype=torch.bfloat16).float().cuda()
    prm = _lib.make_params(w.T, w.H, w.W, 2, w.head_dim, dt, w.top_k, w.top_p, w.eps, cut_ratio=cut)
    pl = _lib.plan(Q, K, V, a, prm)
    O, lse = pl.attn_fwd()
    dQ, dK, dV = pl.attn_bwd(dO, O, lse)
    torch.cuda.synchronize()
    out[name] = dict(status=pl.status(), **{k: t.cpu().numpy().tolist() for k, t in
                     (("O", O), ("lse", lse), ("dQ", dQ), ("dK", dK), ("dV", dV))})
print(json.dumps(dict(lib=_lib.load()._name, runs=out)))
"""


def test_checking_build_matches_default_build(cuda_device, tmp_path):
    lib = pbuild.LIB_CHECKS
    if not os.path.exists(lib):
        pbuild.build_library(checks=True)
    env = dict(os.environ, PRISM_LIB=lib)
    script = tmp_path / "child.py"
    script.write_text(CHILD)
    res = subprocess.run([sys.executable, str(script), ROOT], env=env, capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    got = json.loads(res.stdout.strip().splitlines()[-1])
    assert got["lib"].endswith("libprism_checks.so")
    for name, w, cut in (("tiny", syn.workload(0), 0.0),
                         ("cuts", syn.workload(2, T=16, H=32, W=32, shot_cuts=[12]), 2.5)):
        r = got["runs"][name]
        assert r["status"] == _lib.PRISM_OK, f"{name}: a device check fired ({_lib.status_string(r['status'])})"
        Q, K, V = (x.cuda() for x in syn.make_qkv(w, heads=2))
        a = syn.make_amap(w).cuda()
        dt = _lib.PRISM_F32 if w.dtype == "f32" else _lib.PRISM_BF16
        dO = syn.make_dout(w, heads=2, out_dtype=torch.bfloat16).float().cuda()
        prm = _lib.make_params(w.T, w.H, w.W, 2, w.head_dim, dt, w.top_k, w.top_p, w.eps, cut_ratio=cut)
        pl = _lib.plan(Q, K, V, a, prm)
        O, lse = pl.attn_fwd()
        grads = pl.attn_bwd(dO, O, lse)
        torch.cuda.synchronize()
        for key, t in (("O", O), ("lse", lse)):
            np.testing.assert_array_equal(np.asarray(r[key], np.float32), t.cpu().numpy(), err_msg=f"{name} {key}")
        for key, t in zip(("dQ", "dK", "dV"), grads):
            ref = t.cpu().numpy()
            diff = np.abs(np.asarray(r[key], np.float32) - ref).max()
            assert diff <= 1e-5 * np.abs(ref).max(), f"{name} {key}: {diff:.3e}"

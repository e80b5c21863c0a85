"""The Python binding rejects malformed inputs before anything reaches the library
(no device needed: every check below fails before a CUDA call)."""
import pytest
import torch

from dynamic_block_sparse_indicator_b200 import _lib


def _params(**kw):
    base = dict(T=8, H=16, W=16, heads=2, head_dim=64, dtype=_lib.PRISM_BF16, top_k=4, top_p=0.9, eps=1e-6)
    base.update(kw)
    return _lib.make_params(**base)


def test_plan_rejects_host_tensors_and_bad_shapes():
    p = _params()
    x = torch.zeros(2, 2048, 64, dtype=torch.bfloat16)          # host memory: not accepted
    with pytest.raises(ValueError):
        _lib.plan(x, x, x, None, p)
    with pytest.raises(ValueError):
        _lib.plan(x.float(), x.float(), x.float(), None, p)    # wrong dtype for a bf16 plan
    with pytest.raises(ValueError):
        _lib.plan_import(x, x, x, None, None, p)


def test_plan_sharded_rejects_bad_shard_lists():
    p = _params()
    x = torch.zeros(2, 1024, 64, dtype=torch.bfloat16)          # one of 2 shards of 2,048 tokens
    with pytest.raises(ValueError):
        _lib.plan_sharded([], [], [], None, p)                   # no shards
    with pytest.raises(ValueError):
        _lib.plan_sharded([x, x], [x], [x, x], None, p)          # lists of different lengths
    with pytest.raises(ValueError):
        _lib.plan_sharded([x] * 3, [x] * 3, [x] * 3, None, p)    # 3 shards do not divide T = 8
    with pytest.raises(ValueError):
        _lib.plan_sharded([x, x], [x, x], [x, x], None, p)       # host memory
    with pytest.raises(ValueError):
        _lib.plan_sharded([0, 0], [0, 0], [0, 0], None, p)       # addresses only: heads_total needed


def test_av_norm_rejects_bad_inputs():
    q = torch.zeros(2, 256, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        _lib.av_norm(q, q[:, :10].contiguous(), q[:, :10].contiguous())    # host memory
    with pytest.raises(ValueError):
        _lib.av_norm(q.float(), q.float(), q.float())                      # not bf16
    with pytest.raises(ValueError):
        _lib.av_norm(q[0], q[0], q[0])                                     # not [heads, rows, D]


def test_params_round_trip():
    p = _params(alpha=1 / 3, shape_mode=_lib.PRISM_SHAPE_FIXED, fixed_shape=13, top_k_frac=0.05)
    assert (p.T, p.H, p.W, p.heads, p.head_dim) == (8, 16, 16, 2, 64)
    assert p.shape_mode == _lib.PRISM_SHAPE_FIXED and p.fixed_shape == 13
    assert abs(p.alpha - 1 / 3) < 1e-7 and abs(p.top_k_frac - 0.05) < 1e-7
    assert p.out_dtype == _lib.PRISM_F32

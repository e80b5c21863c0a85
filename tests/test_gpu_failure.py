"""Failure detection without a GPU fault: a bounded device wait that runs out.

prism_selftest_timeout launches a thread that waits on a barrier nothing
arrives at.  The wait must give up after about a second, report
PRISM_ERR_TIMEOUT with its site through the plan's status word, and leave the
context usable for the next launches.
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    w = syn.workload(0)
    Q, K, V = (x.cuda() for x in syn.make_qkv(w))
    a = syn.make_amap(w).cuda()
    p = _lib.make_params(w.T, w.H, w.W, w.heads, w.head_dim, _lib.PRISM_F32, w.top_k, w.top_p, w.eps)
    pl = _lib.plan(Q, K, V, a, p)
    O0, _ = pl.attn_fwd()
    assert pl.status() == _lib.PRISM_OK
    ref = O0.clone()
    pl.selftest_timeout()
    st, site = pl.status_ex()
    assert st == _lib.PRISM_ERR_TIMEOUT and site == 9001
    assert pl.status() == _lib.PRISM_OK              # the word was cleared
    O1, lse1 = pl.attn_fwd()                         # the context is still usable
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    np.testing.assert_array_equal(O1.cpu().numpy(), ref.cpu().numpy())
    assert torch.isfinite(lse1).all()

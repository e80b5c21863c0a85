"""The per-head input maxima that set the fp16 copies' power-of-two scales.

The plan's scale pass takes each head's largest magnitude of Q, K and V from the
inputs' bit patterns (sign cleared, integer maximum over 16-byte chunks; per
16-bit half for bf16).  Exported as PRISM_ITEM_QKV_MAX, they must equal the
inputs' max |x| per head exactly (a max is exact in any precision), for bf16
and fp32 inputs, heads of very different magnitudes, and a largest magnitude
that comes from a negative value.
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wid,dtype", [(0, _lib.PRISM_F32), (2, _lib.PRISM_BF16)])
def test_exported_maxima_equal_the_inputs(wid, dtype, cuda_device):
    w = syn.workload(wid, T=8, H=16, W=16)
    heads = 3
    Q, K, V = syn.make_qkv(w, heads=heads)
    tdt = torch.float32 if dtype == _lib.PRISM_F32 else torch.bfloat16
    # head 0 as drawn, head 1 scaled up by 2^17, head 2 down by 2^-21; one
    # element of each head's K made the head's largest magnitude, and negative
    f = torch.tensor([1.0, 2.0 ** 17, 2.0 ** -21]).view(heads, 1, 1)
    Q, K, V = ((x.float() * f).to(tdt) for x in (Q, K, V))
    for h in range(heads):
        K[h, 17, 5] = -1.75 * K[h].float().abs().max().to(tdt)
    prm = _lib.make_params(w.T, w.H, w.W, heads, w.head_dim, dtype, w.top_k, w.top_p, w.eps)
    pl = _lib.plan(Q.cuda(), K.cuda(), V.cuda(), syn.make_amap(w).cuda(), prm)
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    got = pl.export("qkv_max").reshape(heads, 3).view(np.float32)
    want = np.stack([x.float().abs().amax(dim=(1, 2)).numpy() for x in (Q, K, V)], axis=1)
    np.testing.assert_array_equal(got, want)
    assert (got[:, 1] == -K[:, 17, 5].float().numpy()).all()

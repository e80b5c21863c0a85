"""Forward parity when a head runs in several passes over key-tile ranges.

Heads with more than 1,024 key tiles (131,072 tokens) are processed in passes
that each visit one range of key tiles for every query tile and carry the
running (O, max, sum) of every query row to the next pass; the last pass writes
O and LSE.  A 16 x 64 x 144 grid (147,456 tokens, 1,152 key tiles: two passes),
at head_dim 128 and 64, is planned with the oracle's own shapes and selection
(prism_plan_import), so every query row's key set is exactly the oracle's, and O
and LSE are compared on sampled rows spread over all query tiles, the rows of the
first and the last tile included, plus the rows with the most and the fewest
selected keys in the last key range.
"""
import numpy as np
import pytest
import torch

import parity
from dynamic_block_sparse_indicator_b200 import _lib
from dynamic_block_sparse_indicator_b200 import synthetic as syn
from oracle import prism_oracle as po

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("head_dim", [128, 64])
def test_two_pass_forward_matches_oracle(head_dim, cuda_device):
    w = syn.workload(2, T=16, H=64, W=144, head_dim=head_dim)
    assert w.N // 128 > 1024                     # more than one pass
    Q, K, V = syn.make_qkv(w, heads=1)
    a = syn.make_amap(w)
    q, k, v = (x[0].double().numpy() for x in (Q, K, V))
    o = po.plan_head(q, k, v, a.numpy(), w.T, w.H, w.W, w.top_k, w.top_p, w.eps)
    NB, WORDS = w.N // 64, (w.N // 64 + 31) // 32
    sid = torch.from_numpy(o["shape_id"].astype(np.uint8)[None]).cuda()
    bits = torch.from_numpy(parity.sets_to_bits(o["sel"], NB, WORDS)[None].view(np.int32)).cuda()
    p = _lib.make_params(w.T, w.H, w.W, 1, w.head_dim, _lib.PRISM_BF16, w.top_k, w.top_p, w.eps)
    pl = _lib.plan_import(Q.cuda(), K.cuda(), V.cuda(), sid, bits, p)
    O, lse = pl.attn_fwd()
    torch.cuda.synchronize()
    assert pl.status() == _lib.PRISM_OK
    O, lse = O[0].double().cpu().numpy(), lse[0].double().cpu().numpy()
    rng = np.random.default_rng(5)
    starts = o["starts"]
    # keys of each query block that lie in the second pass's range (key tiles >= 1024)
    tail = np.array([sum(starts[j + 1] - starts[j] for j in js if starts[j] >= 1024 * 128) for js in o["sel"]])
    picks = [0, len(o["sel"]) - 1, int(np.argmax(tail)), int(np.argmin(tail))]
    picks += list(rng.integers(0, len(o["sel"]), 120))
    rows = np.unique(np.concatenate([o["src"][starts[i]:starts[i + 1]][:4] for i in picks]))
    Oo, lo, _ = po.attention_rows(q, k, v, o["src"], starts, o["sel"], rows)
    good, rl2, ma = parity.close(O[rows], Oo)
    assert good, f"O relL2 {rl2:.2e} maxabs {ma:.2e}"
    np.testing.assert_allclose(lse[rows], lo, atol=2e-2, rtol=1e-3)

"""The comparison rules of tests/parity.py forgive only what the oracle's own
margins show to be a near-tie, and nothing else."""
import numpy as np

import parity
from oracle import prism_oracle as po


def _stats(shape_id, rho_margin, snap_margin):
    return dict(shape_id=np.asarray(shape_id), rho_margin=np.asarray(rho_margin, float),
                snap_margin=np.asarray(snap_margin, float))


def test_shape_mismatch_needs_a_near_tie():
    st = _stats([3, 8, 13], [0.2, 0.3, 0.1], [0.5, 2.0, 1.0])
    assert parity.shapes_agree([3, 8, 13], st) == (3, [], [])
    # a differing shape with both margins far from zero is a failure
    assert parity.shapes_agree([3, 9, 13], st)[2] == [1]
    # accepted only where a margin is below the tie bound
    assert parity.shapes_agree([3, 9, 13], _stats([3, 8, 13], [0.2, 5e-6, 0.1], [0.5, 2.0, 1.0]))[1] == [1]
    assert parity.shapes_agree([3, 9, 13], _stats([3, 8, 13], [0.2, 0.3, 0.1], [0.5, 5e-6, 1.0]))[1] == [1]


def test_selection_mismatch_needs_a_near_tie():
    rng = np.random.default_rng(3)
    Qb, Kb = rng.normal(size=(1, 32)), rng.normal(size=(12, 32))
    sel, s, P = po.select(Qb, Kb, 3, 0.0)
    want = sel[0]
    assert parity.selection_agrees(want, s[0], P[0], 3, 0.0)
    order = np.argsort(-P[0], kind="stable")
    swapped = np.sort(np.r_[order[:2], order[5]])          # third block replaced by the sixth
    assert not parity.selection_agrees(swapped, s[0], P[0], 3, 0.0)
    assert not parity.selection_agrees(order[:4], s[0], P[0], 3, 0.0)   # one block too many
    # equal logits at the boundary: either block is accepted
    s2 = s[0].copy()
    s2[order[3]] = s2[order[2]]
    assert parity.selection_agrees(np.sort(np.r_[order[:2], order[3]]), s2, P[0], 3, 0.0)


def test_gradient_rule_adds_half_a_bf16_ulp_of_the_tensor_scale():
    ref = np.array([0.5, 170.0, -80.0])
    # 0.3 off anywhere: inside 3e-2 + 170 / 512
    assert parity.close_grad(ref + [0.3, 0.0, 0.0], ref)[0]
    assert parity.close_grad(ref + [0.0, 0.3, 0.0], ref)[0]
    # 0.4 off: outside it
    assert not parity.close_grad(ref + [0.4, 0.0, 0.0], ref)[0]
    # on a unit-scale tensor the bar is the plain 3e-2 (plus 2^-9)
    small = np.array([0.5, -1.0, 0.25])
    assert not parity.close_grad(small + [0.04, 0.0, 0.0], small)[0]
    # the relative-L2 bar still applies
    assert not parity.close_grad(ref * 1.02, ref)[0]

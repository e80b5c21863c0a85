"""Pins of the oracle's guidance-map producer (audio-to-video cross-attention norm).

The map is a_{t,h,w} = ||h_hat_{t,h,w}||_2 with h_hat = CrossAttn(h, K_a, V_a)
(page paper.rainbus.top, section "前置知识", the dual-branch DiT paragraph;
page xyznot.com/id, section "Metode" 1).  Each test checks the oracle against
something other than itself: closed forms (one audio token, identical keys, a
hand-worked two-key softmax, the one-hot limit), invariances that any correct
softmax attention has, PyTorch's own scaled_dot_product_attention in float64,
and a pure-Python brute force on a tiny case.
"""
import math

import numpy as np
import pytest
import torch

from oracle import prism_oracle as po


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_single_audio_token_closed_form():
    # softmax over one key is 1: every video token receives V_a of that token,
    # and the norm runs over all heads' channels together
    rng = np.random.default_rng(1)
    Q, K, V = _rand(rng, 3, 20, 16), _rand(rng, 3, 1, 16), _rand(rng, 3, 1, 16)
    a, hh = po.av_norm_map(Q, K, V)
    want = math.sqrt(sum(float(V[h, 0] @ V[h, 0]) for h in range(3)))
    np.testing.assert_allclose(a, np.full(20, want), rtol=1e-14)
    for h in range(3):
        np.testing.assert_allclose(hh[h], np.tile(V[h, 0], (20, 1)), rtol=1e-14)


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(2)
    Q, V = _rand(rng, 2, 30, 8), _rand(rng, 2, 5, 8)
    K = np.repeat(_rand(rng, 2, 1, 8), 5, axis=1)
    a, hh = po.av_norm_map(Q, K, V)
    for h in range(2):
        np.testing.assert_allclose(hh[h], np.tile(V[h].mean(axis=0), (30, 1)), rtol=1e-12)
    want = math.sqrt(sum(float(V[h].mean(0) @ V[h].mean(0)) for h in range(2)))
    np.testing.assert_allclose(a, want, rtol=1e-12)


def test_two_key_softmax_by_hand():
    # D = 4: q = (1,0,0,0), k0 = (2,0,0,0), k1 = 0 -> logits 2/sqrt(4) = 1 and 0,
    # weights e/(e+1) and 1/(e+1); pins the 1/sqrt(D) scale and the softmax axis
    Q = np.array([[[1.0, 0, 0, 0]]])
    K = np.array([[[2.0, 0, 0, 0], [0, 0, 0, 0]]])
    V = np.array([[[1.0, 2.0, 0, 0], [0, 0, 3.0, 0]]])
    a, hh = po.av_norm_map(Q, K, V)
    e = math.e
    want = np.array([e / (e + 1), 2 * e / (e + 1), 3 / (e + 1), 0.0])
    np.testing.assert_allclose(hh[0, 0], want, rtol=1e-14)
    np.testing.assert_allclose(a[0], np.linalg.norm(want), rtol=1e-14)


def test_one_hot_limit():
    # keys 2000 * e_j and queries e_{j*}: the logit gap of 500 leaves weight
    # exp(-500) on the other keys, so h_hat = V_a[j*] to double precision
    D, M, N, heads = 16, 6, 12, 2
    rng = np.random.default_rng(3)
    K = np.zeros((heads, M, D))
    for h in range(heads):
        for j in range(M):
            K[h, j, j] = 2000.0
    pick = rng.integers(0, M, size=(heads, N))
    Q = np.zeros((heads, N, D))
    for h in range(heads):
        Q[h, np.arange(N), pick[h]] = 1.0
    V = _rand(rng, heads, M, D)
    a, hh = po.av_norm_map(Q, K, V)
    for h in range(heads):
        np.testing.assert_allclose(hh[h], V[h, pick[h]], rtol=1e-13, atol=1e-300)
    want = np.sqrt(sum((V[h, pick[h]] ** 2).sum(axis=1) for h in range(heads)))
    np.testing.assert_allclose(a, want, rtol=1e-13)


def test_shift_of_all_keys_leaves_the_output():
    # adding the same vector u to every audio key shifts each query's logits by
    # the constant q.u / sqrt(D): a softmax over the keys does not see it
    rng = np.random.default_rng(4)
    Q, K, V = _rand(rng, 2, 40, 8), _rand(rng, 2, 9, 8), _rand(rng, 2, 9, 8)
    u = 3.0 * _rand(rng, 2, 1, 8)
    a0, h0 = po.av_norm_map(Q, K, V)
    a1, h1 = po.av_norm_map(Q, K + u, V)
    np.testing.assert_allclose(h1, h0, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(a1, a0, rtol=1e-11)


def test_permutations_and_value_scaling():
    rng = np.random.default_rng(5)
    Q, K, V = _rand(rng, 2, 25, 8), _rand(rng, 2, 7, 8), _rand(rng, 2, 7, 8)
    a0, h0 = po.av_norm_map(Q, K, V)
    p = rng.permutation(7)                       # audio tokens reordered: nothing changes
    a1, _ = po.av_norm_map(Q, K[:, p], V[:, p])
    np.testing.assert_allclose(a1, a0, rtol=1e-13)
    q = rng.permutation(25)                      # video tokens reordered: the map follows
    a2, _ = po.av_norm_map(Q[:, q], K, V)
    np.testing.assert_allclose(a2, a0[q], rtol=1e-13)
    a3, h3 = po.av_norm_map(Q, K, -2.5 * V)      # values scaled: h_hat scales, the norm by |c|
    np.testing.assert_allclose(h3, -2.5 * h0, rtol=1e-13)
    np.testing.assert_allclose(a3, 2.5 * a0, rtol=1e-13)


def test_matches_torch_sdpa_float64():
    rng = np.random.default_rng(6)
    heads, N, M, D = 3, 57, 19, 16
    Q, K, V = _rand(rng, heads, N, D), _rand(rng, heads, M, D), _rand(rng, heads, M, D)
    a, hh = po.av_norm_map(Q, K, V)
    t = lambda x: torch.from_numpy(x).unsqueeze(0)
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V))[0]
    np.testing.assert_allclose(hh, ref.numpy(), rtol=1e-12, atol=1e-13)
    cat = ref.permute(1, 0, 2).reshape(N, heads * D)   # heads concatenated per token
    np.testing.assert_allclose(a, torch.linalg.vector_norm(cat, dim=1).numpy(), rtol=1e-12)


def test_brute_force_loops():
    rng = np.random.default_rng(7)
    heads, N, M, D = 2, 3, 4, 4
    Q, K, V = _rand(rng, heads, N, D), _rand(rng, heads, M, D), _rand(rng, heads, M, D)
    a, hh = po.av_norm_map(Q, K, V)
    for n in range(N):
        tot = 0.0
        for h in range(heads):
            w = [math.exp(sum(Q[h, n, c] * K[h, j, c] for c in range(D)) / math.sqrt(D))
                 for j in range(M)]
            z = sum(w)
            for c in range(D):
                o = sum(w[j] * V[h, j, c] for j in range(M)) / z
                assert o == pytest.approx(hh[h, n, c], rel=1e-12, abs=1e-14)
                tot += o * o
        assert math.sqrt(tot) == pytest.approx(a[n], rel=1e-12)


def test_rows_subset_equals_full_map():
    rng = np.random.default_rng(8)
    Q, K, V = _rand(rng, 2, 300, 8), _rand(rng, 2, 11, 8), _rand(rng, 2, 11, 8)
    a, hh = po.av_norm_map(Q, K, V)
    rows = np.array([0, 17, 299, 150])
    ar, hr = po.av_norm_rows(Q, K, V, rows)
    np.testing.assert_array_equal(ar, a[rows])
    np.testing.assert_array_equal(hr, hh[:, rows])

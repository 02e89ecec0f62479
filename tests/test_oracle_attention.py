"""Pins of the oracle's attention branch: brute-force scalar loops on tiny inputs,
and invariants from the pages.

Sources: "Jamba: Hybrid SSM-Transformer", section 1 (softmax(QK^T/sqrt(d_k))V, MHA
or GQA); the 51cto Hymba-1.5B article, section 2 (GQA, RoPE, sliding-window layers
plus full-attention layers; meta tokens interact with every later token); "Hymba
Guide", Learnable Meta-Tokens (attended by all tokens).
"""
import math

import numpy as np
import pytest

import oracle


def _qkv(seed, H=4, G=2, L=40, dh=8, dv=6):
    g = np.random.default_rng(seed)
    return g.standard_normal((H, L, dh)), g.standard_normal((G, L, dh)), g.standard_normal((G, L, dv))


def _brute_force(q, k, v, m, W):
    """Per query, per key scalar loops with math.exp."""
    H, L, dh = q.shape
    G = k.shape[0]
    out = np.zeros((H, L, v.shape[2]))
    for h in range(H):
        g = h // (H // G)
        for i in range(L):
            keys = [j for j in range(L) if j <= i and (j < m or W <= 0 or i - j < W)]
            scores = []
            for j in keys:
                s = 0.0
                for e in range(dh):
                    s += q[h, i, e] * k[g, j, e]
                scores.append(s / math.sqrt(dh))
            mx = max(scores)
            wts = [math.exp(s - mx) for s in scores]
            tot = sum(wts)
            for e in range(v.shape[2]):
                out[h, i, e] = sum(wt * v[g, j, e] for wt, j in zip(wts, keys)) / tot
    return out


@pytest.mark.parametrize("m,W", [(5, 7), (0, 3), (3, 0), (0, 1)])
def test_attention_matches_brute_force(m, W):
    q, k, v = _qkv(1)
    pos = np.arange(q.shape[1])
    got = oracle.attention(q, k, v, oracle.visibility_mask(pos, pos, m, W))
    np.testing.assert_allclose(got, _brute_force(q, k, v, m, W), rtol=1e-12, atol=1e-12)


def test_mask_matches_scalar_rule():
    pos = np.arange(30)
    for m, W in [(4, 6), (0, 5), (7, 0), (30, 2)]:
        mask = oracle.visibility_mask(pos, pos, m, W)
        for i in pos:
            for j in pos:
                assert mask[i, j] == oracle.key_visible(int(i), int(j), m, W)


def test_window_at_least_length_is_full_causal():
    """A window no shorter than the sequence is plain causal attention."""
    q, k, v = _qkv(2, L=33)
    pos = np.arange(33)
    for W in (33, 34, 1000):
        mask = oracle.visibility_mask(pos, pos, 4, W)
        np.testing.assert_array_equal(mask, np.tril(np.ones((33, 33), dtype=bool)))
        np.testing.assert_allclose(oracle.attention(q, k, v, mask),
                                   oracle.attention(q, k, v, np.tril(np.ones((33, 33), dtype=bool))))


def test_meta_keys_visible_to_every_query():
    """Meta tokens are attended by every later token, also far outside the window:
    give meta key 0 a dominant logit and every query returns v_0."""
    H, G, L, dh, dv, m, W = 2, 1, 50, 4, 3, 3, 4
    q = np.zeros((H, L, dh))
    q[:, :, 0] = 1.0
    k = np.zeros((G, L, dh))
    k[0, 0, 0] = 200.0
    v = np.random.default_rng(3).standard_normal((G, L, dv))
    pos = np.arange(L)
    out = oracle.attention(q, k, v, oracle.visibility_mask(pos, pos, m, W))
    for h in range(H):
        np.testing.assert_allclose(out[h], np.broadcast_to(v[0, 0], (L, dv)), rtol=0, atol=1e-12)


def test_visible_set_recovered_exactly_with_one_hot_values():
    """With equal scores (q = 0) and one-hot position codes as V, each output row is
    1/|S_i| on exactly the visible set S_i."""
    L, m, W = 24, 3, 5
    q = np.zeros((1, L, 4))
    k = np.random.default_rng(4).standard_normal((1, L, 4))
    v = np.eye(L)[None]
    pos = np.arange(L)
    out = oracle.attention(q, k, v, oracle.visibility_mask(pos, pos, m, W))[0]
    for i in range(L):
        vis = [j for j in range(L) if j <= i and (j < m or i - j < W)]
        expect = np.zeros(L)
        expect[vis] = 1.0 / len(vis)
        np.testing.assert_allclose(out[i], expect, rtol=0, atol=1e-15)


def test_gqa_equals_repeated_kv_heads():
    """GQA with G < H equals MHA on K, V heads repeated for consecutive query heads."""
    q, k, v = _qkv(5, H=6, G=2)
    pos = np.arange(q.shape[1])
    mask = oracle.visibility_mask(pos, pos, 2, 9)
    rep = 6 // 2
    np.testing.assert_allclose(oracle.attention(q, k, v, mask),
                               oracle.attention(q, np.repeat(k, rep, axis=0), np.repeat(v, rep, axis=0), mask),
                               rtol=0, atol=0)


def test_softmax_rows_sum_to_one():
    q, k, _ = _qkv(6)
    v = np.ones((k.shape[0], k.shape[1], 1))
    pos = np.arange(q.shape[1])
    out = oracle.attention(q, k, v, oracle.visibility_mask(pos, pos, 3, 4))
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_rope_is_complex_rotation():
    """Rotate-half RoPE = multiplying the complex numbers a_i + i b_i (pairs (i, i+dh/2))
    by exp(i p theta_i), theta_i = base^(-2i/dh)."""
    g = np.random.default_rng(7)
    L, dh, base = 9, 16, 10000.0
    x = g.standard_normal((L, dh))
    pos = np.arange(L) * 37 + 5
    got = oracle.rope(x, pos, base)
    half = dh // 2
    theta = np.array([base ** (-2.0 * i / dh) for i in range(half)])
    z = (x[:, :half] + 1j * x[:, half:]) * np.exp(1j * pos[:, None] * theta[None, :])
    np.testing.assert_allclose(got, np.concatenate([z.real, z.imag], axis=1), rtol=1e-12, atol=1e-12)


def test_rope_scores_depend_on_relative_position_only():
    g = np.random.default_rng(8)
    dh = 64
    a, b = g.standard_normal(dh), g.standard_normal(dh)
    for (i, j, c) in [(10, 3, 100), (0, 0, 5000), (7, 7, 1)]:
        s0 = oracle.rope(a[None], np.array([i]), 10000.0) @ oracle.rope(b[None], np.array([j]), 10000.0).T
        s1 = oracle.rope(a[None], np.array([i + c]), 10000.0) @ oracle.rope(b[None], np.array([j + c]), 10000.0).T
        assert s0[0, 0] == pytest.approx(s1[0, 0], rel=1e-9, abs=1e-9)
    # rotation keeps the norm
    x = g.standard_normal((5, dh))
    np.testing.assert_allclose(np.linalg.norm(oracle.rope(x, np.arange(5) * 11, 10000.0), axis=1),
                               np.linalg.norm(x, axis=1), rtol=1e-13)

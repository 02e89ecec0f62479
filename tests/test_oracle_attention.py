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


# ---------------------------------------------------------------------------
# affine adaptation of shared K, V by a secondary layer ("Hymba Guide",
# Cross-Layer KV Cache Sharing, section 1: K~ = K * w_scale + b_bias)
# ---------------------------------------------------------------------------

def _affine(G, dh, dv, ks, kb, vs, vb):
    return {"kv_scale": np.concatenate([np.ravel(ks), np.ravel(vs)]),
            "kv_bias": np.concatenate([np.ravel(kb), np.ravel(vb)])}


def test_affine_kv_hand_worked_one_head():
    """One query, two keys, dh = 4, dv = 2. Scale ln 3 on K's first dimension makes the
    scores (ln 3, 0), so the weights are (3/4, 1/4); V scaled by (2, 1) and shifted by
    (0, 5) gives rows (2, 5) and (0, 6), so the output is (1.5, 5.25)."""
    q = np.array([[[2.0, 0.0, 0.0, 0.0]]])
    k = np.array([[[1.0, 0.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]]])
    v = np.array([[[1.0, 0.0], [0.0, 1.0]]])
    w = _affine(1, 4, 2, [np.log(3.0), 1.0, 1.0, 1.0], np.zeros(4), [2.0, 1.0], [0.0, 5.0])
    ka, va = oracle.adapt_shared_kv(k, v, w, 1, 4, 2)
    o = oracle.attention(q, ka, va, np.ones((1, 2), dtype=bool))
    np.testing.assert_allclose(o[0, 0], [1.5, 5.25], rtol=1e-14)


def test_affine_kv_identity_is_plain_sharing():
    """Scale 1 and bias 0 reproduce plain sharing bit for bit, and no weights at all
    leave K and V untouched."""
    g = np.random.default_rng(81)
    G, dh, dv = 2, 64, 128
    k, v = g.standard_normal((G, 9, dh)), g.standard_normal((G, 9, dv))
    w = _affine(G, dh, dv, np.ones(G * dh), np.zeros(G * dh), np.ones(G * dv), np.zeros(G * dv))
    ka, va = oracle.adapt_shared_kv(k, v, w, G, dh, dv)
    assert np.array_equal(ka, k) and np.array_equal(va, v)
    kb, vb = oracle.adapt_shared_kv(k, v, {}, G, dh, dv)
    assert kb is k and vb is v


def test_affine_kv_per_head_layout():
    """kv_scale / kv_bias hold the G K vectors first, then the G V vectors. With KV head
    1's K scale 0 its queries see equal scores (a plain mean of its adapted V rows),
    while KV head 0 keeps its softmax; V head 1 is shifted by its own bias only."""
    g = np.random.default_rng(82)
    G, H, dh, dv, L = 2, 4, 8, 6, 5
    q = g.standard_normal((H, 1, dh))
    k = g.standard_normal((G, L, dh))
    v = g.standard_normal((G, L, dv))
    vb1 = g.standard_normal(dv)
    w = _affine(G, dh, dv, np.concatenate([np.ones(dh), np.zeros(dh)]), np.zeros(G * dh),
                np.ones(G * dv), np.concatenate([np.zeros(dv), vb1]))
    ka, va = oracle.adapt_shared_kv(k, v, w, G, dh, dv)
    o = oracle.attention(q, ka, va, np.ones((1, L), dtype=bool))
    for h in range(2):  # group 0: plain attention
        s = q[h, 0] @ k[0].T / np.sqrt(dh)
        p = np.exp(s - s.max())
        np.testing.assert_allclose(o[h, 0], (p / p.sum()) @ v[0], rtol=1e-12)
    for h in range(2, 4):  # group 1: uniform weights over V + its bias
        np.testing.assert_allclose(o[h, 0], v[1].mean(axis=0) + vb1, rtol=1e-12)


def test_affine_kv_key_bias_cancels_and_value_affine_commutes():
    """Two identities of softmax attention that a kernel may rely on: a key bias adds
    q . b to every score of a query (softmax is shift invariant, so it drops out), and
    since the weights sum to 1, attention over V * s + b equals (attention over V) * s + b."""
    g = np.random.default_rng(83)
    G, H, dh, dv, L = 1, 3, 16, 8, 11
    q = g.standard_normal((H, L, dh))
    k = g.standard_normal((G, L, dh))
    v = g.standard_normal((G, L, dv))
    mask = oracle.visibility_mask(np.arange(L), np.arange(L), 2, 4)
    ks, vs, vb = 1.0 + 0.3 * g.standard_normal(dh), 1.0 + 0.3 * g.standard_normal(dv), g.standard_normal(dv)
    w_nob = _affine(G, dh, dv, ks, np.zeros(dh), vs, np.zeros(dv))
    w_bias = _affine(G, dh, dv, ks, 5.0 * g.standard_normal(dh), vs, vb)
    a0 = oracle.attention(q, *oracle.adapt_shared_kv(k, v, w_nob, G, dh, dv), mask)
    a1 = oracle.attention(q, *oracle.adapt_shared_kv(k, v, w_bias, G, dh, dv), mask)
    np.testing.assert_allclose(a1, a0 + vb, rtol=1e-10, atol=1e-12)
    plain = oracle.attention(q * ks, k, v, mask)  # the key scale moved onto the query
    np.testing.assert_allclose(a0, plain * vs, rtol=1e-10, atol=1e-12)

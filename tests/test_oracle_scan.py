"""Pins of the oracle's Mamba branch (selective scan, conv, Delta) against facts
the pages and the mathematics fix, not against the oracle itself.

Sources: "Jamba: Hybrid SSM-Transformer", How It Actually Works section 1 (the
scan equation); "Lecture 04 - Beyond the Dense Transformer", section 2 (Delta -> 0
ignores the token, large Delta resets the state, the state size does not depend
on the sequence length) and section 3 (the scan is a masked semiseparable matrix).
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _rand_scan_inputs(seed, L=48, C=3, N=4):
    g = np.random.default_rng(seed)
    xc = g.standard_normal((L, C))
    delta = np.exp(g.uniform(np.log(1e-3), np.log(0.5), size=(L, C)))
    A = -g.uniform(0.5, 8.0, size=(C, N))
    Bm = g.standard_normal((L, N))
    Cm = g.standard_normal((L, N))
    D = g.standard_normal(C)
    return xc, delta, A, Bm, Cm, D


def test_scan_equals_semiseparable_closed_form():
    """Lecture 04 section 3: y = M x with M[t, s] = sum_n C_t,n exp(A_n (S_t - S_s)) Delta_s B_s,n
    for s <= t (S = cumulative sum of Delta), plus D x. Built from cumulative sums,
    not from a step recurrence."""
    xc, delta, A, Bm, Cm, D = _rand_scan_inputs(1)
    y, _ = oracle.selective_scan(xc, delta, A, Bm, Cm, D)
    L, C = xc.shape
    S = np.cumsum(delta, axis=0)
    for c in range(C):
        M = np.zeros((L, L))
        for t in range(L):
            for s in range(t + 1):
                decay = np.exp(A[c] * (S[t, c] - S[s, c]))
                M[t, s] = np.sum(Cm[t] * decay * Bm[s]) * delta[s, c]
        ref = M @ xc[:, c] + D[c] * xc[:, c]
        np.testing.assert_allclose(y[:, c], ref, rtol=1e-11, atol=1e-11)


def test_scan_final_state_closed_form():
    """h_L[c, n] = sum_s exp(A_n (S_L - S_s)) Delta_s B_s,n x_s (state after the last token)."""
    xc, delta, A, Bm, Cm, D = _rand_scan_inputs(2, L=20)
    _, h = oracle.selective_scan(xc, delta, A, Bm, Cm, D)
    S = np.cumsum(delta, axis=0)
    for c in range(xc.shape[1]):
        ref = sum(np.exp(A[c] * (S[-1, c] - S[s, c])) * delta[s, c] * Bm[s] * xc[s, c]
                  for s in range(xc.shape[0]))
        np.testing.assert_allclose(h[c], ref, rtol=1e-11, atol=1e-12)


def test_scan_single_step_by_hand():
    """One step, N = 1, one channel, worked by hand:
    h0 = 0.5, Delta = 0.1, A = -2, B = 3, x = 4, C = 5, D = 0.25
    h1 = exp(-0.2) * 0.5 + 0.1 * 3 * 4 = 0.40936537653899 + 1.2
    y  = 5 * h1 + 0.25 * 4."""
    y, h = oracle.selective_scan(np.array([[4.0]]), np.array([[0.1]]), np.array([[-2.0]]),
                                 np.array([[3.0]]), np.array([[5.0]]), np.array([0.25]),
                                 h0=np.array([[0.5]]))
    assert h[0, 0] == pytest.approx(1.6093653765389909, abs=1e-14)
    assert y[0, 0] == pytest.approx(9.046826882694955, abs=1e-13)


def test_delta_to_zero_ignores_tokens():
    """Lecture 04 section 2: Delta -> 0 gives A_bar -> I and B_bar -> 0, the state coasts;
    so from h0 = 0 the output is just D x."""
    xc, delta, A, Bm, Cm, D = _rand_scan_inputs(3)
    y, h = oracle.selective_scan(xc, np.zeros_like(delta), A, Bm, Cm, D)
    np.testing.assert_array_equal(h, 0.0)
    np.testing.assert_allclose(y, D[None, :] * xc, rtol=0, atol=0)
    # with a nonzero initial state, Delta = 0 keeps it unchanged
    h0 = np.random.default_rng(4).standard_normal(h.shape)
    _, h1 = oracle.selective_scan(xc, np.zeros_like(delta), A, Bm, Cm, D, h0=h0)
    np.testing.assert_array_equal(h1, h0)


def test_delta_large_resets_to_current_token():
    """Lecture 04 section 2: large Delta gives A_bar -> 0, the state is overwritten by
    the current token: h_t = Delta B_t x_t, so y_t = Delta (C_t . B_t) x_t + D x_t,
    and earlier tokens have no effect."""
    xc, delta, A, Bm, Cm, D = _rand_scan_inputs(5, L=16)
    big = np.full_like(delta, 60.0)  # exp(60 * A) <= exp(-30)
    y, _ = oracle.selective_scan(xc, big, A, Bm, Cm, D)
    ref = 60.0 * np.sum(Cm * Bm, axis=1)[:, None] * xc + D[None, :] * xc
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-9)
    xc2 = xc.copy()
    xc2[:8] += 3.0
    y2, _ = oracle.selective_scan(xc2, big, A, Bm, Cm, D)
    np.testing.assert_allclose(y2[9:], y[9:], rtol=1e-9, atol=1e-9)


def test_state_size_independent_of_length():
    """Lecture 04 section 2: the state is O(d_state) whatever the sequence length."""
    for L in (1, 7, 300):
        xc, delta, A, Bm, Cm, D = _rand_scan_inputs(6, L=L, C=5, N=16)
        _, h = oracle.selective_scan(xc, delta, A, Bm, Cm, D)
        assert h.shape == (5, 16)


def test_conv_impulse_response_and_causality():
    """A depthwise causal filter answers a unit impulse at t0 with its taps in reverse
    order (the newest input meets the last tap) and nothing before t0."""
    g = np.random.default_rng(7)
    L, C, K = 12, 3, 4
    w = g.standard_normal((C, K))
    b = g.standard_normal(C)
    t0 = 5
    x = np.zeros((L, C))
    x[t0] = 1.0
    out = oracle.causal_conv(x, w, b)
    for j in range(L):
        expect = b + (w[:, K - 1 - (j - t0)] if 0 <= j - t0 < K else 0.0)
        np.testing.assert_allclose(out[j], expect, rtol=0, atol=1e-15)
    # causality: changing the future leaves the past alone
    x2 = g.standard_normal((L, C))
    x3 = x2.copy()
    x3[t0:] += 10.0
    np.testing.assert_array_equal(oracle.causal_conv(x2, w, b)[:t0], oracle.causal_conv(x3, w, b)[:t0])


def test_elementwise_special_values():
    assert oracle.softplus(np.array(0.0)) == pytest.approx(math.log(2.0), abs=1e-15)
    assert oracle.softplus(np.array(800.0)) == pytest.approx(800.0)
    assert oracle.softplus(np.array(-50.0)) == pytest.approx(math.exp(-50.0), rel=1e-12)
    assert oracle.silu(np.array(0.0)) == 0.0
    assert oracle.silu(np.array(1.0)) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), abs=1e-15)
    assert oracle.silu(np.array(-40.0)) == pytest.approx(-40.0 * math.exp(-40.0), rel=1e-9)


def _layer(cfg_kw=None, seed=11):
    cfg = synth.tiny_layer_cfg().with_(**(cfg_kw or {}))
    w = synth.perturbed_weights(synth.layer_weights(cfg, seed), cfg, seed)
    x = synth.layer_input(cfg, 1, 24, seed)
    return cfg, w, x


def test_layer_delta_to_zero_gives_gated_skip():
    """Whole layer with Delta forced to ~1e-18 (b_dt = -40, W_dt = 0): the Mamba branch
    reduces to D * SiLU(conv(x)) * SiLU(z) (Lecture 04 section 2, Delta -> 0)."""
    cfg, w, x = _layer()
    w["b_dt"] = np.full_like(w["b_dt"], -40.0)
    w["w_dt"] = np.zeros_like(w["w_dt"])
    r = oracle.mixer_prefill_row(cfg, w, x[0])
    xh = np.concatenate([w["meta"], x[0]]).astype(np.float64)
    blocks = oracle.split_projection(cfg, xh @ w["w_in"].astype(np.float64).T)
    xc = oracle.silu(oracle.causal_conv(blocks["x"], w["conv_w"], w["conv_b"]))
    ref = w["D"][None, :] * xc * oracle.silu(blocks["z"])
    np.testing.assert_allclose(r["y_ssm"], ref, rtol=1e-12, atol=1e-12)


def test_meta_tokens_prepopulate_state():
    """Hymba Guide, Learnable Meta-Tokens: the meta rows enter the SSM before the
    first user token, so the state at the first user token differs from a cold
    start; with zero meta vectors (and zero conv bias) it is a cold start."""
    cfg, w, x = _layer()
    w0 = dict(w)
    w0["meta"] = np.zeros_like(w["meta"])
    w0["conv_b"] = np.zeros_like(w["conv_b"])
    r0 = oracle.mixer_prefill_row(cfg, w0, x[0])
    # cold start: the user tokens alone, no meta rows at all
    cfg_nometa = cfg.with_(n_meta=0)
    w_cold = dict(w0)
    w_cold["meta"] = w0["meta"][:0]
    r_cold = oracle.mixer_prefill_row(cfg_nometa, w_cold, x[0])
    m = cfg.n_meta
    np.testing.assert_allclose(r0["y_ssm"][m:], r_cold["y_ssm"], rtol=1e-10, atol=1e-12)
    r1 = oracle.mixer_prefill_row(cfg, w, x[0])
    assert np.abs(r1["y_ssm"][m] - r0["y_ssm"][m]).max() > 1e-3

"""Pins of the oracle's SSD form of the Mamba heads (cfg.ssm_heads > 0).

Source: "Lecture 04 - Beyond the Dense Transformer", section 3: Mamba-2 makes the state
matrix A a scalar times the identity and gives the SSM a multi-head structure, and the
selective SSM then equals a masked-attention-like product with a semiseparable matrix
(structured state space duality), computable either as the recurrence or as blocks of
matmuls. The oracle computes the recurrence; these tests hold it against the masked
matrix form, the final-state closed form, the chunked block form the tensor-core kernel
follows, the selective form with per-head values written out per channel, and
decode-after-prefill.
"""
import numpy as np
import pytest

import oracle
import synth


def _ssd_cfg(**kw):
    base = synth.tiny_layer_cfg().with_(ssm_heads=4, window=16)  # 4 heads of 128 channels
    return base.with_(**kw)


def _head_inputs(seed, L=40, nh=3, P=5, N=4):
    g = np.random.default_rng(seed)
    xc = g.standard_normal((L, nh * P))
    dh = np.exp(g.uniform(np.log(1e-3), np.log(0.5), size=(L, nh)))  # Delta per head
    a = -g.uniform(0.5, 8.0, size=nh)                                 # A per head
    Bm = g.standard_normal((L, N))
    Cm = g.standard_normal((L, N))
    D = g.standard_normal(nh * P)
    return xc, dh, a, Bm, Cm, D


def _oracle_scan(xc, dh, a, Bm, Cm, D, P):
    """The oracle's scan fed the way ssm_params feeds it in the SSD form."""
    cfg = _ssd_cfg(d_inner=xc.shape[1], ssm_heads=dh.shape[1], d_state=Bm.shape[1])
    w = {"w_dt": np.eye(dh.shape[1]), "b_dt": np.zeros(dh.shape[1]), "A_log": np.log(-a)}
    # softplus^-1 of Delta, so that ssm_params returns Delta itself
    delta, A = oracle.ssm_params(cfg, w, np.log(np.expm1(dh)))
    return oracle.selective_scan(xc, delta, A, Bm, Cm, D)


def test_ssd_equals_masked_attention_form():
    """y[:, head h] = (L_h o (C B^T)) (Delta_h x_h) + D x with L_h[t, s] = exp(a_h (S_t - S_s))
    for s <= t and 0 above the diagonal (S = cumulative sum of the head's Delta): one
    L x L matrix per head, shared by the head's channels and not depending on the state
    index. Built with explicit loops over (t, s)."""
    P = 5
    xc, dh, a, Bm, Cm, D = _head_inputs(3, P=P)
    y, _ = _oracle_scan(xc, dh, a, Bm, Cm, D, P)
    L, nh = dh.shape
    S = np.cumsum(dh, axis=0)
    for h in range(nh):
        M = np.zeros((L, L))
        for t in range(L):
            for s in range(t + 1):
                M[t, s] = np.exp(a[h] * (S[t, h] - S[s, h])) * (Cm[t] @ Bm[s]) * dh[s, h]
        cols = slice(h * P, (h + 1) * P)
        ref = M @ xc[:, cols] + D[cols] * xc[:, cols]
        np.testing.assert_allclose(y[:, cols], ref, rtol=1e-11, atol=1e-11)


def test_ssd_final_state_closed_form():
    """h_L[c, n] = sum_s exp(a_h (S_L - S_s)) Delta_s,h B_s,n x_s,c for c in head h."""
    P = 4
    xc, dh, a, Bm, Cm, D = _head_inputs(4, L=25, nh=2, P=P)
    _, hL = _oracle_scan(xc, dh, a, Bm, Cm, D, P)
    S = np.cumsum(dh, axis=0)
    for c in range(xc.shape[1]):
        h = c // P
        ref = sum(np.exp(a[h] * (S[-1, h] - S[s, h])) * dh[s, h] * Bm[s] * xc[s, c] for s in range(xc.shape[0]))
        np.testing.assert_allclose(hL[c], ref, rtol=1e-11, atol=1e-12)


def _chunked(xc, dh, a, Bm, Cm, D, P, Q):
    """The block form: within a chunk of Q rows the masked product; across chunks an
    [N, P] state per head carried by its total decay. Written from the duality, as a
    second formulation (the tensor-core kernel's steps)."""
    L, nh = dh.shape
    N = Bm.shape[1]
    y = np.zeros_like(xc)
    Sst = np.zeros((nh, N, P))
    for c0 in range(0, L, Q):
        r = slice(c0, min(L, c0 + Q))
        for h in range(nh):
            cols = slice(h * P, (h + 1) * P)
            cs = np.cumsum(a[h] * dh[r, h])                    # log decay from the chunk start
            Lm = np.tril(np.exp(cs[:, None] - cs[None, :]))
            G = Cm[r] @ Bm[r].T
            X = xc[r, cols]
            y_diag = (Lm * G) @ (dh[r, h][:, None] * X)
            y_off = np.exp(cs)[:, None] * (Cm[r] @ Sst[h])
            y[r, cols] = y_diag + y_off + D[cols] * X
            wgt = np.exp(cs[-1] - cs) * dh[r, h]
            Sst[h] = np.exp(cs[-1]) * Sst[h] + Bm[r].T @ (wgt[:, None] * X)
    return y, Sst


@pytest.mark.parametrize("Q", [8, 16, 64])
def test_chunked_block_form_equals_the_recurrence(Q):
    P = 6
    xc, dh, a, Bm, Cm, D = _head_inputs(5, L=45, nh=2, P=P)
    y, hL = _oracle_scan(xc, dh, a, Bm, Cm, D, P)
    yc, Sst = _chunked(xc, dh, a, Bm, Cm, D, P, Q)
    np.testing.assert_allclose(yc, y, rtol=1e-10, atol=1e-11)
    for c in range(xc.shape[1]):
        np.testing.assert_allclose(Sst[c // P][:, c % P], hL[c], rtol=1e-10, atol=1e-12)


def test_ssd_layer_equals_selective_layer_with_values_written_per_channel():
    """The SSD layer is the selective layer whose W_dt rows, b_dt and A_log entries are the
    head's, repeated for each of its channels (and A_log for each state): the whole
    layer (attention, fusion, projections) must agree to rounding."""
    cfg = _ssd_cfg()
    w = synth.perturbed_weights(synth.layer_weights(cfg, 5), cfg, 5)
    P = cfg.d_inner // cfg.ssm_heads
    assert w["w_dt"].shape == (cfg.ssm_heads, cfg.dt_rank) and w["A_log"].shape == (cfg.ssm_heads,)
    sel = cfg.with_(ssm_heads=0)
    ws = dict(w, w_dt=np.repeat(w["w_dt"], P, axis=0), b_dt=np.repeat(w["b_dt"], P),
              A_log=np.repeat(w["A_log"], P)[:, None] * np.ones((1, cfg.d_state), np.float32))
    x = synth.layer_input(cfg, 2, 30, 6)
    r1 = oracle.mixer_prefill(cfg, w, x)
    r2 = oracle.mixer_prefill(sel, ws, x)
    for k in ("y", "h", "conv", "delta"):
        np.testing.assert_allclose(r1[k], r2[k], rtol=1e-12, atol=1e-12)


def test_ssd_heads_are_independent():
    """Changing one head's A_log changes only that head's channels of the SSM branch."""
    cfg = _ssd_cfg()
    w = synth.layer_weights(cfg, 7)
    P = cfg.d_inner // cfg.ssm_heads
    x = synth.layer_input(cfg, 1, 20, 8)
    r1 = oracle.mixer_prefill(cfg, w, x)
    w2 = dict(w, A_log=w["A_log"].copy())
    w2["A_log"][2] += 0.7
    r2 = oracle.mixer_prefill(cfg, w2, x)
    d = np.abs(r1["y_ssm"] - r2["y_ssm"]).max(axis=(0, 1))
    changed = np.nonzero(d > 0)[0]
    assert changed.min() >= 2 * P and changed.max() < 3 * P and len(changed) > P // 2


@pytest.mark.parametrize("window", [6, 0])
def test_ssd_decode_by_decode_equals_prefill(window):
    cfg = _ssd_cfg(window=window)
    w = synth.perturbed_weights(synth.layer_weights(cfg, 9), cfg, 9)
    B, T, T0 = 2, 22, 9
    m = cfg.n_meta
    x = synth.layer_input(cfg, B, T, 10)
    ref = oracle.mixer_prefill(cfg, w, x, residual=True)
    pre = oracle.mixer_prefill(cfg, w, x[:, :T0], residual=True)
    cap = m + (window if window > 0 else T)
    cache = oracle.cache_from_prefill(cfg, pre["k"], pre["v"], cap)
    h, conv = pre["h"].copy(), pre["conv"].copy()
    for t in range(T0, T):
        y = oracle.mixer_decode(cfg, w, x[:, t], cache, h, conv, residual=True)
        np.testing.assert_allclose(y, ref["y"][:, m + t], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(h, ref["h"], rtol=1e-10, atol=1e-12)

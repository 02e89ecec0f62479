"""Pins of the host-side helpers that GPU tests use as references.

merge_split_partials rebuilds a softmax-weighted sum from per-split partials (the
form the decode attention leaves in the workspace); here it must equal the softmax
over all keys computed directly, with splits of unequal length and an empty split."""
import numpy as np

from gpu_helpers import merge_split_partials


def _partials(scores, values, bounds):
    """Per split [a, b): sum of 2^(s - m) v, m = max s (base 2), sum of 2^(s - m)."""
    s2 = scores * np.log2(np.e)
    out = []
    for a, b in bounds:
        if b > a:
            m = s2[a:b].max()
            p = np.exp2(s2[a:b] - m)
            out.append(np.concatenate([(p[:, None] * values[a:b]).sum(0), [m, p.sum()]]))
        else:
            out.append(np.concatenate([np.zeros(values.shape[1]), [-np.inf, 0.0]]))
    return np.array(out)


def test_merge_of_split_partials_equals_full_softmax():
    g = np.random.default_rng(7)
    n, dv = 53, 6
    scores = g.normal(size=n) * 4.0
    values = g.normal(size=(n, dv))
    p = np.exp(scores - scores.max())
    ref = (p[:, None] * values).sum(0) / p.sum()
    for bounds in ([(0, 53)], [(0, 20), (20, 41), (41, 53)], [(0, 9), (9, 9), (9, 53)],
                   [(0, 1), (1, 52), (52, 53), (53, 53)]):
        got = merge_split_partials(_partials(scores, values, bounds))
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_merge_is_independent_of_split_order():
    g = np.random.default_rng(8)
    scores, values = g.normal(size=30) * 3.0, g.normal(size=(30, 4))
    part = _partials(scores, values, [(0, 7), (7, 19), (19, 30)])
    np.testing.assert_allclose(merge_split_partials(part), merge_split_partials(part[::-1]), rtol=1e-13)

"""Pins of the temperature / top-p sampling oracle (CPU only).

Fixed outside the oracle: a hand-worked three-token example of the pages'
rule (including the token that crosses the threshold), the plain categorical
distribution it must reduce to at top_p = 1 (inverse CDF over a fine grid of
uniforms reproduces softmax frequencies), the greedy limits (temperature 0,
top_p -> 0), and invariances (a constant shift of the logits, a relabelling
of the vocabulary).  Forgetting the one-position shift of the removal mask
fails the hand example.
"""

import math

import numpy as np
import pytest

from oracle import sampling as osm

RNG = np.random.default_rng(5)


def test_hand_example_keeps_the_crossing_token():
    # logits [2, 1, 0], T = 1: p = softmax = [e^2, e, 1] / (e^2 + e + 1)
    e2, e1 = math.exp(2.0), math.exp(1.0)
    z = e2 + e1 + 1.0
    p0, p1 = e2 / z, e1 / z                       # 0.665, 0.245
    assert p0 < 0.7 < p0 + p1
    # top_p = 0.7: token 0 always kept; token 1 kept (p0 <= 0.7); token 2 dropped (p0 + p1 > 0.7)
    ids, q = osm.nucleus(np.array([2.0, 1.0, 0.0]), 1.0, 0.7)
    assert list(ids) == [0, 1]
    assert q[0] == pytest.approx(e2 / (e2 + e1), rel=1e-14)
    cut = e2 / (e2 + e1)                           # 0.731
    logits = np.array([[2.0, 1.0, 0.0]] * 3)
    got = osm.sample_top_p(logits, 1.0, 0.7, np.array([0.0, cut - 1e-9, cut + 1e-9]))
    assert list(got) == [0, 0, 1]
    assert osm.sample_top_p(logits[:1], 1.0, 0.7, np.array([0.999999]))[0] == 1   # never token 2


def test_top_p_one_is_plain_categorical_sampling():
    V, N = 7, 20000
    logits = RNG.standard_normal(V) * 2
    u = (np.arange(N) + 0.5) / N
    got = osm.sample_top_p(np.tile(logits, (N, 1)), 0.8, 1.0, u)
    p = np.exp(logits / 0.8 - np.max(logits / 0.8))
    p /= p.sum()
    freq = np.bincount(got, minlength=V) / N
    assert np.all(np.abs(freq - p) <= 2.0 / N)


def test_greedy_limits():
    logits = RNG.standard_normal((4, 50))
    arg = np.argmax(logits, axis=1)
    assert np.array_equal(osm.sample_top_p(logits, 0, 0.9, np.zeros(4)), arg)
    assert np.array_equal(osm.sample_top_p(logits, 1e-6, 0.9, RNG.uniform(size=4)), arg)
    assert np.array_equal(osm.sample_top_p(logits, 1.0, 1e-12, RNG.uniform(size=4)), arg)


def test_shift_and_relabelling_invariance():
    V = 40
    logits = RNG.standard_normal((3, V))
    u = RNG.uniform(size=3)
    a = osm.sample_top_p(logits, 0.9, 0.8, u)
    assert np.array_equal(osm.sample_top_p(logits + 7.5, 0.9, 0.8, u), a)
    perm = RNG.permutation(V)                      # token perm[i] of the new vocabulary is token i
    relab = np.empty_like(logits)
    relab[:, perm] = logits
    assert np.array_equal(osm.sample_top_p(relab, 0.9, 0.8, u), perm[a])


def test_kept_set_is_the_smallest_prefix_reaching_top_p():
    for _ in range(50):
        logits = RNG.standard_normal(30) * 1.5
        top_p = RNG.uniform(0.05, 0.99)
        ids, q = osm.nucleus(logits, 1.0, top_p)
        p = np.exp(logits - logits.max())
        p /= p.sum()
        ps = np.sort(p)[::-1]
        k = len(ids)
        assert ps[:k].sum() >= top_p - 1e-12            # reaches top_p ...
        assert k == 1 or ps[:k - 1].sum() <= top_p      # ... and one token fewer does not exceed it
        assert q.sum() == pytest.approx(1.0, rel=1e-14)


def test_planted_unshifted_mask_fails_the_hand_example(monkeypatch):
    # the mistake: drop a token when the cumulative probability INCLUDING it exceeds top_p
    def nucleus_unshifted(logits_row, temperature, top_p):
        z = np.asarray(logits_row, np.float64) / float(temperature)
        order = np.lexsort((np.arange(z.shape[0]), -z))
        p = np.exp(z[order] - z[order][0])
        p /= p.sum()
        keep = np.cumsum(p) <= top_p
        keep[0] = True
        k = int(np.argmin(keep)) if not keep.all() else len(keep)
        return order[:k], p[:k] / p[:k].sum()

    monkeypatch.setattr(osm, "nucleus", nucleus_unshifted)
    with pytest.raises(AssertionError):
        test_hand_example_keeps_the_crossing_token()

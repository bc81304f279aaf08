"""Pins of the 4-bit group-wise quantised Linear oracle (CPU only).

Each test pins the oracle to a fact that does not come from the oracle: a
hand-derived packed word, the half-step error bound of rounding to a uniform
grid, exact cases (constant groups, weights already on the grid, the group's
minimum and maximum), and the per-group factorisation of the quantised
product.  A wrong nibble order, a wrong group index (tiling instead of
repeating the per-group terms), a dropped offset or a transposed operand
each fail at least one of them.
"""

import numpy as np
import pytest

from oracle import quant as oq

RNG = np.random.default_rng(11)


def test_pack_golden_word_low_nibble_first():
    # codes 1..8 of one 8-code word: code k in bits 4k..4k+3 -> 0x87654321
    codes = np.arange(1, 9, dtype=np.uint8)[None, :]
    assert int(oq.pack_int4(codes)[0, 0]) == 0x87654321
    # and 15, 0, 0, ... -> 0x0000000F ; 0, ..., 0, 15 -> 0xF0000000
    c = np.zeros((2, 8), np.uint8)
    c[0, 0] = 15
    c[1, 7] = 15
    w = oq.pack_int4(c)
    assert int(w[0, 0]) == 0x0000000F and int(w[1, 0]) == 0xF0000000


def test_pack_unpack_round_trip_bit_exact():
    codes = RNG.integers(0, 16, size=(5, 128), dtype=np.uint8)
    assert np.array_equal(oq.unpack_int4(oq.pack_int4(codes), 128), codes)


def test_rounding_error_within_half_a_step():
    w = RNG.standard_normal((12, 256)) * 0.05
    q, s, b = oq.quantize(w)
    err = np.abs(oq.dequantize(q, s, b) - w)
    half_step = np.repeat(s, 64, axis=1) / 2
    assert np.all(err <= half_step * (1 + 1e-9) + 1e-15)
    assert q.max() <= 15 and q.min() >= 0


def test_group_extremes_and_constant_groups_are_exact():
    w = RNG.standard_normal((3, 128))
    w[1, 64:] = 0.375                       # a constant group
    q, s, b = oq.quantize(w)
    d = oq.dequantize(q, s, b)
    assert np.all(d[1, 64:] == 0.375) and s[1, 1] == 0.0
    for o in range(3):
        for g in range(2):
            grp, dq = w[o, 64 * g:64 * g + 64], d[o, 64 * g:64 * g + 64]
            assert dq[np.argmin(grp)] == grp.min()
            assert abs(dq[np.argmax(grp)] - grp.max()) <= 4 * np.finfo(float).eps * max(1.0, abs(grp.max()))


def test_weights_on_the_grid_come_back_unchanged():
    # w = s*q + b with integer q that reach 0 and 15 in every group
    s = np.array([[0.25, 0.125]]) * np.array([[1.0], [2.0]])
    b = np.array([[-1.0, 0.5], [2.0, -3.0]])
    q = RNG.integers(0, 16, size=(2, 128)).astype(np.uint8)
    q[:, 0], q[:, 1], q[:, 64], q[:, 65] = 0, 15, 15, 0
    w = np.repeat(s, 64, axis=1) * q + np.repeat(b, 64, axis=1)
    q2, s2, b2 = oq.quantize(w)
    assert np.array_equal(q2, q) and np.allclose(s2, s, rtol=0, atol=1e-15) and np.array_equal(b2, b)
    assert np.array_equal(oq.dequantize(q2, s2, b2), w)


def test_quantized_linear_matches_the_per_group_factorisation():
    # y[n, o] = sum_g ( s[o,g] * sum_{i in g} x[n,i] q[o,i] + b[o,g] * sum_{i in g} x[n,i] )
    n, out_f, in_f = 3, 5, 192
    x = RNG.standard_normal((n, in_f))
    q = RNG.integers(0, 16, size=(out_f, in_f)).astype(np.uint8)
    s = RNG.uniform(0.01, 0.1, size=(out_f, in_f // 64))
    b = RNG.uniform(-0.5, 0.5, size=(out_f, in_f // 64))
    y = oq.quantized_linear(x, oq.pack_int4(q), s, b, in_f)
    ref = np.zeros((n, out_f))
    for g in range(in_f // 64):
        xs = x[:, 64 * g:64 * g + 64]
        ref += (xs @ q[:, 64 * g:64 * g + 64].astype(np.float64).T) * s[:, g][None, :]
        ref += xs.sum(axis=1)[:, None] * b[:, g][None, :]
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_planted_group_index_mistake_is_caught():
    # tiling the per-group scales instead of repeating them breaks the factorisation pin
    n, out_f, in_f = 2, 3, 128
    x = RNG.standard_normal((n, in_f))
    q = RNG.integers(0, 16, size=(out_f, in_f)).astype(np.uint8)
    s = np.array([[0.1, 0.7]] * out_f)
    b = np.zeros((out_f, 2))
    wrong = np.tile(s, (1, 64)) * q                   # element i gets group i % 2
    good = oq.dequantize(q, s, b)
    assert not np.allclose(x @ wrong.T, x @ good.T)


@pytest.mark.parametrize("bad", [np.zeros((1, 7), np.uint8), np.full((1, 8), 16, np.uint8)])
def test_pack_rejects_bad_input(bad):
    with pytest.raises(ValueError):
        oq.pack_int4(bad)

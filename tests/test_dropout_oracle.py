"""Pins of the dropout oracle (oracle/dropout_ref.py), CPU only.

The generator is pinned by the known-answer vectors published with the
Random123 implementation of Philox4x32-10 (Salmon et al., SC '11); the
attention with dropout by p = 0 reducing to the oracle without dropout,
p = 1 giving zeros, central finite differences of <dO, O> under a fixed
mask, the rowsum(dO o O) identity, and the keep rate, layout and
determinism of the mask."""

from __future__ import annotations

import numpy as np
import pytest

from oracle import attn_ref as ref
from oracle import dropout_ref as dr

INF, CTL, CBR = ref.WINDOW_INF, ref.CAUSAL_TOP_LEFT, ref.CAUSAL_BOTTOM_RIGHT


@pytest.mark.parametrize("ctr,key,want", [
    ((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff,) * 4, (0xffffffff,) * 2, (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
])
def test_philox_known_answers(ctr, key, want):
    got = dr.philox4x32_10(np.array(ctr, dtype=np.uint64), key)
    assert tuple(int(x) for x in got) == want


def test_philox_is_elementwise_over_counters():
    ctrs = np.array([[1, 2, 3, 4], [0, 0, 0, 0], [5, 6, 7, 8]], dtype=np.uint64)
    batch = dr.philox4x32_10(ctrs, (11, 12))
    for c, b in zip(ctrs, batch):
        assert np.array_equal(dr.philox4x32_10(c, (11, 12)), b)


def test_mask_layout_follows_the_counter_reading():
    seed, offset, bh, p = 0x1234_5678_9ABC_DEF0, 7, 5, 0.3
    m = dr.keep_mask(seed, offset, bh, np.arange(9), 13, p)
    t = dr.keep_threshold(p)
    for i, j in [(0, 0), (3, 5), (8, 12), (4, 7)]:
        words = dr.philox4x32_10(np.array([j // 4, i, bh, offset], dtype=np.uint64),
                                 (seed & 0xFFFFFFFF, seed >> 32))
        assert m[i, j] == (int(words[j % 4]) < t)


def test_mask_rate_and_determinism():
    p = 0.25
    m = dr.keep_mask(99, 3, 1, np.arange(256), 256, p)
    n = m.size
    # binomial: 6 standard deviations
    assert abs(m.mean() - (1 - p)) <= 6 * np.sqrt(p * (1 - p) / n)
    assert np.array_equal(m, dr.keep_mask(99, 3, 1, np.arange(256), 256, p))
    assert not np.array_equal(m, dr.keep_mask(99, 4, 1, np.arange(256), 256, p))
    assert not np.array_equal(m, dr.keep_mask(99, 3, 2, np.arange(256), 256, p))
    # a row subset is the same rows of the full mask
    assert np.array_equal(dr.keep_mask(99, 3, 1, [5, 200], 256, p), m[[5, 200]])


def test_threshold_edges():
    assert dr.keep_threshold(0.0) == 2 ** 32 and dr.keep_threshold(1.0) == 0
    assert dr.keep_mask(1, 0, 0, np.arange(4), 8, 0.0).all()
    assert not dr.keep_mask(1, 0, 0, np.arange(4), 8, 1.0).any()
    with pytest.raises(ValueError):
        dr.keep_threshold(1.5)


def _inputs(sq, sk, d, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal(s) for s in ((sq, d), (sk, d), (sk, d), (sq, d))]


WINDOWS = [(INF, INF, False), (CTL, 0, False), (CBR, 0, True), (2, 1, False), (-1, 3, True)]


@pytest.mark.parametrize("w", WINDOWS, ids=str)
def test_p_zero_equals_no_dropout(w):
    q, k, v, do = _inputs(6, 9, 4, 1)
    o, lse = dr.forward(q, k, v, 0.4, *w, 0.0, 5, 0, 0)
    eo, el = ref.forward(q, k, v, 0.4, *w)
    np.testing.assert_array_equal(o, eo)
    np.testing.assert_array_equal(lse, el)
    for g, e in zip(dr.backward(q, k, v, do, 0.4, *w, 0.0, 5, 0, 0),
                    ref.backward(q, k, v, do, 0.4, *w)):
        np.testing.assert_allclose(g, e, rtol=0, atol=1e-12)


def test_p_one_gives_zeros():
    q, k, v, do = _inputs(5, 7, 3, 2)
    o, lse = dr.forward(q, k, v, 0.5, INF, INF, False, 1.0, 9, 1, 2)
    assert not o.any() and np.isfinite(lse).all()
    for g in dr.backward(q, k, v, do, 0.5, INF, INF, False, 1.0, 9, 1, 2):
        assert not g.any()


@pytest.mark.parametrize("w", WINDOWS, ids=str)
def test_finite_differences_under_a_fixed_mask(w):
    q, k, v, do = _inputs(5, 7, 3, 3)
    args = (0.7, *w, 0.3, 1234, 9, 4)
    grads = dr.backward(q, k, v, do, *args)
    h = 1e-6
    for idx, x in enumerate((q, k, v)):
        num = np.zeros_like(x)
        for pos in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[pos] += h
            xm[pos] -= h
            ins_p = [q, k, v]
            ins_m = [q, k, v]
            ins_p[idx], ins_m[idx] = xp, xm
            lp = (dr.forward(*ins_p, *args)[0] * do).sum()
            lm = (dr.forward(*ins_m, *args)[0] * do).sum()
            num[pos] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grads[idx], num, rtol=1e-5, atol=1e-7)


def test_delta_identity_with_dropout():
    # rowsum(dO o O) equals sum_j P_ij dP_ij with dP taken through the mask
    q, k, v, do = _inputs(6, 8, 4, 4)
    p, seed, offset, bh = 0.4, 77, 2, 3
    o, _ = dr.forward(q, k, v, 0.5, INF, INF, False, p, seed, offset, bh)
    probs = ref.probabilities(q, k, 0.5, INF, INF, False)
    ms = dr.keep_mask(seed, offset, bh, np.arange(6), 8, p) / (1 - p)
    dp = (do @ v.T) * ms
    np.testing.assert_allclose(ref.delta(o, do), (probs * dp).sum(1), rtol=1e-12, atol=1e-12)


def test_dropout_is_unbiased_over_masks():
    # E[O with dropout] = O: the 1 / (1 - p) scale restores the expectation
    q, k, v, _ = _inputs(6, 16, 4, 5)
    eo, _ = ref.forward(q, k, v, 0.6, INF, INF, False)
    samples = np.stack([dr.forward(q, k, v, 0.6, INF, INF, False, 0.3, 42, off, 0)[0]
                        for off in range(600)])
    err = np.abs(samples.mean(0) - eo)
    se = samples.std(0, ddof=1) / np.sqrt(len(samples))
    assert (err <= 6 * se + 1e-12).all(), (err / (se + 1e-30)).max()


@pytest.mark.parametrize("w", WINDOWS[:3], ids=str)
def test_bias_with_dropout_p_zero_equals_the_bias_oracle(w):
    q, k, v, do = _inputs(6, 9, 4, 6)
    bias = 1.5 * np.random.default_rng(7).standard_normal((6, 9))
    o, lse = dr.forward(q, k, v, 0.4, *w, 0.0, 5, 0, 0, bias=bias)
    eo, el = ref.forward(q, k, v, 0.4, *w, bias=bias)
    np.testing.assert_array_equal(o, eo)
    np.testing.assert_array_equal(lse, el)
    for g, e in zip(dr.backward(q, k, v, do, 0.4, *w, 0.0, 5, 0, 0, bias=bias),
                    ref.backward(q, k, v, do, 0.4, *w, bias=bias)):
        np.testing.assert_allclose(g, e, rtol=0, atol=1e-12)


@pytest.mark.parametrize("w", WINDOWS[:2], ids=str)
def test_bias_gradient_under_dropout_matches_central_differences(w):
    q, k, v, do = _inputs(5, 7, 3, 9)
    bias = np.sin(np.arange(35, dtype=np.float64).reshape(5, 7))
    args = (0.7, *w, 0.3, 1234, 9, 4)
    *_, db = dr.backward(q, k, v, do, *args, bias=bias)
    h = 1e-6
    num = np.zeros_like(bias)
    for pos in np.ndindex(bias.shape):
        bp, bm = bias.copy(), bias.copy()
        bp[pos] += h
        bm[pos] -= h
        lp = (dr.forward(q, k, v, *args, bias=bp)[0] * do).sum()
        lm = (dr.forward(q, k, v, *args, bias=bm)[0] * do).sum()
        num[pos] = (lp - lm) / (2 * h)
    np.testing.assert_allclose(db, num, rtol=1e-5, atol=1e-7)

"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test fixes the oracle to something the pages or the mathematics fix:
hand-derived masks (tests/golden/masks.txt), central finite differences of the
forward, an independent dense brute force through torch autograd, closed forms
(window (0, 0), scale 0, one token) and invariants.  The planted-mistake tests
at the end show that a plausible slip in the oracle fails one of these pins.
"""

import os

import numpy as np
import pytest
import torch

from oracle import attn_ref as ref

INF = ref.WINDOW_INF
CTL = ref.CAUSAL_TOP_LEFT
CBR = ref.CAUSAL_BOTTOM_RIGHT
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "masks.txt")

# (window_left, window_right, bottom_right): every kind of window, including
# ones that leave rows fully masked when Sq != Sk.
WINDOWS = [
    (INF, INF, False), (CTL, 0, False), (CTL, 0, True), (CBR, 0, False), (CBR, 0, True),
    (INF, 0, False), (INF, 0, True), (2, 1, False), (2, 1, True), (-1, 3, False),
    (-1, 3, True), (3, -2, False), (0, 0, False), (0, 0, True), (0, -1, False),
    (1, INF, True),
]


def _parse_golden():
    names = {"INF": INF, "CAUSAL_TL": CTL, "CAUSAL_BR": CBR}
    cases, cur = [], None
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("case"):
                _, sq, sk, wl, wr, diag = line.split()
                cur = dict(sq=int(sq), sk=int(sk), wl=names.get(wl, None) if wl in names else int(wl),
                           wr=names.get(wr) if wr in names else int(wr), br=(diag == "BR"), rows=[])
                cases.append(cur)
            else:
                cur["rows"].append([c == "1" for c in line])
    return cases


GOLDEN_CASES = _parse_golden()


@pytest.mark.parametrize("case", GOLDEN_CASES, ids=lambda c: f"{c['sq']}x{c['sk']}_{c['wl']}_{c['wr']}_{'BR' if c['br'] else 'TL'}")
def test_mask_matches_hand_derived(case):
    want = np.array(case["rows"], dtype=bool)
    assert want.shape == (case["sq"], case["sk"])
    got = ref.allowed(case["sq"], case["sk"], case["wl"], case["wr"], case["br"])
    np.testing.assert_array_equal(got, want)
    lo, hi, cnt = ref.row_extent(case["sq"], case["sk"], case["wl"], case["wr"], case["br"])
    np.testing.assert_array_equal(cnt, want.sum(1))
    for i in range(case["sq"]):
        if want[i].any():
            idx = np.nonzero(want[i])[0]
            assert lo[i] == idx[0] and hi[i] == idx[-1]
        else:
            assert lo[i] > hi[i]


def _interval_count(sq, sk, wl, wr, br):
    """Closed-form pair count: each row sees one interval of keys."""
    L, R = ref.effective_window(wl, wr, br, sq, sk)
    total = 0
    for i in range(sq):
        lo = 0 if L is None else max(0, i - L)
        hi = sk - 1 if R is None else min(sk - 1, i + R)
        total += max(0, hi - lo + 1)
    return total


@pytest.mark.parametrize("sq,sk", [(1, 1), (7, 5), (5, 7), (130, 300), (600, 513)])
@pytest.mark.parametrize("w", WINDOWS)
def test_allowed_count_closed_form(sq, sk, w):
    assert ref.allowed_count(sq, sk, *w) == _interval_count(sq, sk, *w)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _loss(q, k, v, do, c, w):
    o, _ = ref.forward(q, k, v, c, *w)
    return float((o * do).sum())


@pytest.mark.parametrize("w", WINDOWS)
@pytest.mark.parametrize("c", [0.7, -0.4, 0.0])
def test_backward_matches_central_differences(w, c):
    sq, sk, d = 5, 7, 3
    q, k, v, do = (_rand(s, i) for i, s in enumerate([(sq, d), (sk, d), (sk, d), (sq, d)]))
    dq, dk, dv = ref.backward(q, k, v, do, c, *w)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            fp = _loss(q, k, v, do, c, w)
            x[idx] = old - h
            fm = _loss(q, k, v, do, c, w)
            x[idx] = old
            num[idx] = (fp - fm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7)


def _brute(q, k, v, do, c, w):
    """Independent formulation: dense mask, torch.softmax/logsumexp, autograd."""
    sq, sk = q.shape[0], k.shape[0]
    wl, wr, br = w
    d = sk - sq
    mask = torch.zeros(sq, sk, dtype=torch.bool)
    for i in range(sq):
        for j in range(sk):
            if wl == CTL:
                ok = j <= i
            elif wl == CBR:
                ok = j <= i + d
            else:
                lo_ok = True if wl == INF else (j >= i - (wl - d if br else wl))
                hi_ok = True if wr == INF else (j <= i + (wr + d if br else wr))
                ok = lo_ok and hi_ok
            mask[i, j] = ok
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    s = (tq @ tk.T) * c
    s = s.masked_fill(~mask, float("-inf"))
    rows = mask.any(1)
    lse = torch.logsumexp(s, dim=1)
    o = torch.zeros(sq, v.shape[1], dtype=torch.float64)
    if rows.any():
        p = torch.softmax(s[rows], dim=1)
        o = o.index_put((rows.nonzero()[:, 0],), p @ tv)
    # the zero term keeps the graph alive when every row is masked
    ((o * torch.tensor(do)).sum() + 0.0 * (tq.sum() + tk.sum() + tv.sum())).backward()
    return o.detach().numpy(), lse.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("w", WINDOWS)
@pytest.mark.parametrize("shape", [(5, 7, 4), (9, 6, 8), (1, 1, 2)])
def test_matches_independent_brute_force(w, shape):
    sq, sk, d = shape
    q, k, v, do = (_rand(s, 10 + i) for i, s in enumerate([(sq, d), (sk, d), (sk, d), (sq, d)]))
    c = 0.37
    o, lse = ref.forward(q, k, v, c, *w)
    dq, dk, dv = ref.backward(q, k, v, do, c, *w)
    bo, blse, bdq, bdk, bdv = _brute(q, k, v, do, c, w)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(blse))
    fin = np.isfinite(blse)
    np.testing.assert_allclose(lse[fin], blse[fin], rtol=1e-12, atol=1e-12)
    for a, b in ((dq, bdq), (dk, bdk), (dv, bdv)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("w", WINDOWS)
def test_probability_rows_sum_to_one(w):
    q, k = _rand((11, 5), 1), _rand((13, 5), 2)
    p = ref.probabilities(q, k, 0.9, *w)
    m = ref.allowed(11, 13, *w)
    s = p.sum(1)
    np.testing.assert_allclose(s[m.any(1)], 1.0, rtol=1e-13)
    assert np.all(s[~m.any(1)] == 0)
    assert np.all(p[~m] == 0)


@pytest.mark.parametrize("w", WINDOWS)
def test_ones_value_gives_ones_output(w):
    q, k = _rand((9, 4), 3), _rand((12, 4), 4)
    v = np.ones((12, 6))
    o, lse = ref.forward(q, k, v, 1.3, *w)
    m = ref.allowed(9, 12, *w).any(1)
    np.testing.assert_allclose(o[m], 1.0, rtol=1e-13)
    assert np.all(o[~m] == 0) and np.all(np.isneginf(lse[~m]))


def test_full_window_equals_no_mask():
    q, k, v = _rand((8, 4), 5), _rand((10, 4), 6), _rand((10, 4), 7)
    base = ref.forward(q, k, v, 0.5, INF, INF, False)
    for wl, wr, br in [(10, 10, False), (100, 100, True), (INF, 10, False), (10, INF, True)]:
        o, lse = ref.forward(q, k, v, 0.5, wl, wr, br)
        np.testing.assert_allclose(o, base[0], rtol=1e-14)
        np.testing.assert_allclose(lse, base[1], rtol=1e-14)
    # and the unmasked result is plain softmax attention
    s = 0.5 * q @ k.T
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(base[0], p @ v, rtol=1e-12)


@pytest.mark.parametrize("wl,wr", [(2, 1), (-1, 3), (INF, 0), (0, INF), (3, -2)])
def test_bottom_right_with_equal_lengths_is_top_left(wl, wr):
    q, k, v = _rand((9, 4), 8), _rand((9, 4), 9), _rand((9, 4), 10)
    a = ref.forward(q, k, v, 0.8, wl, wr, False)
    b = ref.forward(q, k, v, 0.8, wl, wr, True)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("br", [False, True])
def test_numeric_causal_equals_top_left_sentinel(br):
    # (INF, 0) under TOP_LEFT is the top-left causal sentinel; the sentinel
    # keeps its meaning whatever the diagonal bit says.
    for sq, sk in [(6, 6), (4, 7), (7, 4)]:
        q, k, v = _rand((sq, 4), 11), _rand((sk, 4), 12), _rand((sk, 4), 13)
        a = ref.forward(q, k, v, 0.6, INF, 0, False)
        b = ref.forward(q, k, v, 0.6, CTL, 0, br)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("br", [False, True])
def test_bottom_right_sentinel_equals_shifted_numeric(br):
    for sq, sk in [(6, 6), (4, 7), (7, 4)]:
        d = sk - sq
        q, k, v = _rand((sq, 4), 14), _rand((sk, 4), 15), _rand((sk, 4), 16)
        a = ref.forward(q, k, v, 0.6, INF, d, False)
        b = ref.forward(q, k, v, 0.6, CBR, 0, br)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("w", [(256, 0, False), (3, 1, True), (CBR, 0, True), (-2, 4, True)])
def test_packed_equals_per_sequence_dense(w):
    sq = [3, 1, 7, 5]
    sk = [5, 2, 7, 9]
    cu_q = np.concatenate([[0], np.cumsum(sq)])
    cu_k = np.concatenate([[0], np.cumsum(sk)])
    H, D = 2, 4
    q, k, v, do = _rand((cu_q[-1], H, D), 20), _rand((cu_k[-1], H, D), 21), _rand((cu_k[-1], H, D), 22), _rand((cu_q[-1], H, D), 23)
    o, lse = ref.forward_packed(q, k, v, cu_q, cu_k, 0.5, *w)
    dq, dk, dv = ref.backward_packed(q, k, v, do, cu_q, cu_k, 0.5, *w)
    for s in range(4):
        for h in range(H):
            qs, ks = slice(cu_q[s], cu_q[s + 1]), slice(cu_k[s], cu_k[s + 1])
            eo, el = ref.forward(q[qs, h], k[ks, h], v[ks, h], 0.5, *w)
            np.testing.assert_array_equal(o[qs, h], eo)
            np.testing.assert_array_equal(lse[h, qs], el)
            g = ref.backward(q[qs, h], k[ks, h], v[ks, h], do[qs, h], 0.5, *w)
            np.testing.assert_array_equal(dq[qs, h], g[0])
            np.testing.assert_array_equal(dk[ks, h], g[1])
            np.testing.assert_array_equal(dv[ks, h], g[2])
    th = ref.lse_ht_to_th(lse)
    assert th.shape == (cu_q[-1], H) and th[4, 1] == lse[1, 4]


@pytest.mark.parametrize("br,sq,sk", [(False, 6, 6), (False, 5, 8), (True, 5, 8), (True, 8, 5)])
def test_window_zero_zero_closed_form_keeps_fp16_subnormals(br, sq, sk):
    # Window (0, 0): each row sees exactly key i (+d under BOTTOM_RIGHT), so
    # P = 1, O_i = v_{i(+d)}, LSE_i = S_{i,i(+d)}, dQ = dK = 0, dV_j = dO_i.
    # fp16 subnormal inputs must come through unchanged (0.15b release notes,
    # "Known Problems": hardware that flushes fp16 subnormals fails these).
    d = sk - sq if br else 0
    rng = np.random.default_rng(30)
    q = rng.standard_normal((sq, 4)).astype(np.float16).astype(np.float64)
    k = rng.standard_normal((sk, 4)).astype(np.float16).astype(np.float64)
    v = (rng.integers(1, 1000, (sk, 4)) * 2.0**-24).astype(np.float16).astype(np.float64)
    assert np.all(np.abs(v) < 2.0**-14)          # fp16 subnormals
    do = rng.standard_normal((sq, 4))
    o, lse = ref.forward(q, k, v, 0.5, 0, 0, br)
    dq, dk, dv = ref.backward(q, k, v, do, 0.5, 0, 0, br)
    want_dv = np.zeros_like(v)
    for i in range(sq):
        j = i + d
        if 0 <= j < sk:
            np.testing.assert_array_equal(o[i], v[j])
            assert lse[i] == pytest.approx(0.5 * q[i] @ k[j], abs=1e-15)
            want_dv[j] = do[i]
        else:
            assert np.all(o[i] == 0) and np.isneginf(lse[i])
    np.testing.assert_allclose(dq, 0, atol=1e-15)
    np.testing.assert_allclose(dk, 0, atol=1e-15)
    np.testing.assert_allclose(dv, want_dv, atol=1e-15)


@pytest.mark.parametrize("w", WINDOWS)
def test_zero_scale_closed_form(w):
    # c = 0: P is uniform over the allowed keys, LSE = ln(count), O = their
    # mean, dQ = dK = 0, dV_j = sum over rows i that see j of dO_i / count_i.
    sq, sk = 6, 9
    q, k, v, do = _rand((sq, 4), 40), _rand((sk, 4), 41), _rand((sk, 3), 42), _rand((sq, 3), 43)
    m = ref.allowed(sq, sk, *w)
    cnt = m.sum(1)
    o, lse = ref.forward(q, k, v, 0.0, *w)
    dq, dk, dv = ref.backward(q, k, v, do, 0.0, *w)
    want_dv = np.zeros_like(v)
    for i in range(sq):
        if cnt[i]:
            np.testing.assert_allclose(o[i], v[m[i]].mean(0), rtol=1e-13, atol=1e-15)
            assert lse[i] == pytest.approx(np.log(cnt[i]), rel=1e-15)
            want_dv[m[i]] += do[i] / cnt[i]
        else:
            assert np.all(o[i] == 0) and np.isneginf(lse[i])
    assert np.all(dq == 0) and np.all(dk == 0)
    np.testing.assert_allclose(dv, want_dv, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("w", WINDOWS[:6])
def test_negative_scale_mirrors_key_sign(w):
    q, k, v = _rand((7, 4), 50), _rand((8, 4), 51), _rand((8, 4), 52)
    a = ref.forward(q, k, v, 0.45, *w)
    b = ref.forward(q, -k, v, -0.45, *w)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_single_token_returns_value():
    q, k, v = _rand((1, 4), 60), _rand((1, 4), 61), _rand((1, 5), 62)
    o, lse = ref.forward(q, k, v, 2.0, INF, INF)
    np.testing.assert_array_equal(o, v)
    assert lse[0] == pytest.approx(2.0 * float(q[0] @ k[0]))


def test_delta_equals_probability_weighted_form():
    # delta_i = <dO_i, O_i> = sum_j P_ij <dO_i, v_j>: a second route to it.
    q, k, v, do = _rand((7, 4), 70), _rand((9, 4), 71), _rand((9, 4), 72), _rand((7, 4), 73)
    o, _ = ref.forward(q, k, v, 0.8, 3, 1, True)
    p = ref.probabilities(q, k, 0.8, 3, 1, True)
    np.testing.assert_allclose(ref.delta(o, do), (p * (do @ v.T)).sum(1), rtol=1e-12, atol=1e-14)


def test_row_blocking_is_invisible():
    # Sizes that span several oracle row blocks give the unblocked result.
    q, k, v, do = _rand((1100, 3), 80), _rand((700, 3), 81), _rand((700, 3), 82), _rand((1100, 3), 83)
    o, lse = ref.forward(q, k, v, 0.3, 300, 20, True)
    old = ref.ROW_BLOCK
    try:
        ref.ROW_BLOCK = 4096
        o2, lse2 = ref.forward(q, k, v, 0.3, 300, 20, True)
        g2 = ref.backward(q, k, v, do, 0.3, 300, 20, True)
    finally:
        ref.ROW_BLOCK = old
    g = ref.backward(q, k, v, do, 0.3, 300, 20, True)
    np.testing.assert_allclose(o, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse, lse2, rtol=1e-14)
    for a, b in zip(g, g2):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------------------
# Planted mistakes: each variant of the oracle below carries one plausible slip
# (planted on the CPU, in a copy); a pin above must catch it.
# ---------------------------------------------------------------------------

def _planted_backward_missing_delta(q, k, v, do, c, wl, wr, br):
    mask = ref.allowed(q.shape[0], k.shape[0], wl, wr, br)
    p, _ = ref._probs_block(q, k, c, mask)
    ds = p * (do @ v.T)                       # dropped "- delta"
    return c * ds @ k, c * ds.T @ q, p.T @ do


def _planted_window_sign(sq, sk, wl, wr, br):
    d = sk - sq
    i = np.arange(sq)[:, None]
    j = np.arange(sk)[None, :]
    L, R = (wl + d, wr - d) if br else (wl, wr)   # d applied with the wrong sign
    return (j >= i - L) & (j <= i + R)


def test_planted_missing_delta_is_caught():
    sq, sk, d = 5, 7, 3
    q, k, v, do = (_rand(s, i) for i, s in enumerate([(sq, d), (sk, d), (sk, d), (sq, d)]))
    good = ref.backward(q, k, v, do, 0.7, 2, 1, False)
    bad = _planted_backward_missing_delta(q, k, v, do, 0.7, 2, 1, False)
    assert not np.allclose(good[0], bad[0], atol=1e-3)
    assert not np.allclose(good[1], bad[1], atol=1e-3)


def test_planted_window_sign_is_caught_by_golden():
    caught = False
    for c in GOLDEN_CASES:
        if c["wl"] in (CTL, CBR) or c["wl"] == INF or c["wr"] == INF:
            continue
        want = np.array(c["rows"], dtype=bool)
        if not np.array_equal(_planted_window_sign(c["sq"], c["sk"], c["wl"], c["wr"], c["br"]), want):
            caught = True
    assert caught


def test_row_subset_equals_full_rows():
    q, k, v = _rand((300, 4), 90), _rand((260, 4), 91), _rand((260, 4), 92)
    o, lse = ref.forward(q, k, v, 0.4, 50, 3, True)
    rows = [0, 7, 128, 299]
    o2, lse2 = ref.forward(q, k, v, 0.4, 50, 3, True, rows=rows)
    np.testing.assert_array_equal(o2, o[rows])
    np.testing.assert_array_equal(lse2, lse[rows])


# ---------------------------------------------------------------------------
# The dense BHSD wrappers: every (b, h) slice is the independent brute force of
# that slice's own inputs, and a wrapper that mixes up batch and head indices
# (planted below) fails the same check.
# ---------------------------------------------------------------------------

def _check_dense_wrappers(fwd_dense, bwd_dense, w):
    B_, H, sq, sk, d = 2, 3, 6, 9, 4
    q, k, v, do = (_rand(s, 40 + i) for i, s in
                   enumerate([(B_, H, sq, d), (B_, H, sk, d), (B_, H, sk, d), (B_, H, sq, d)]))
    c = 0.45
    o, lse = fwd_dense(q, k, v, c, *w)
    dq, dk, dv = bwd_dense(q, k, v, do, c, *w)
    assert o.shape == q.shape and lse.shape == (B_, H, sq)
    for b in range(B_):
        for h in range(H):
            bo, blse, bdq, bdk, bdv = _brute(q[b, h], k[b, h], v[b, h], do[b, h], c, w)
            np.testing.assert_allclose(o[b, h], bo, rtol=1e-12, atol=1e-12)
            np.testing.assert_array_equal(np.isneginf(lse[b, h]), np.isneginf(blse))
            fin = np.isfinite(blse)
            np.testing.assert_allclose(lse[b, h][fin], blse[fin], rtol=1e-12, atol=1e-12)
            for a, e in ((dq[b, h], bdq), (dk[b, h], bdk), (dv[b, h], bdv)):
                np.testing.assert_allclose(a, e, rtol=1e-10, atol=1e-12)
    # a subset of heads: those computed, the rest left NaN
    sub = [(1, 2), (0, 0)]
    o2, lse2 = fwd_dense(q, k, v, c, *w, heads=sub)
    g2 = bwd_dense(q, k, v, do, c, *w, heads=sub)
    for b in range(B_):
        for h in range(H):
            if (b, h) in sub:
                np.testing.assert_array_equal(o2[b, h], o[b, h])
                for a, e in zip(g2, (dq, dk, dv)):
                    np.testing.assert_array_equal(a[b, h], e[b, h])
            else:
                assert np.isnan(o2[b, h]).all() and np.isnan(lse2[b, h]).all()
                assert all(np.isnan(a[b, h]).all() for a in g2)


@pytest.mark.parametrize("w", [(INF, INF, False), (CTL, 0, False), (2, -1, True), (CBR, 0, True)])
def test_dense_wrappers_equal_the_brute_force_per_head(w):
    _check_dense_wrappers(ref.forward_dense, ref.backward_dense, w)


def _planted_forward_dense_wrong_head(q, k, v, c, wl, wr, br=False, heads=None):
    B_, H = q.shape[:2]
    o, lse = ref.forward_dense(q, k, v, c, wl, wr, br, heads=heads)
    for b, h in heads if heads is not None else [(b, h) for b in range(B_) for h in range(H)]:
        # K of the neighbouring head
        o[b, h], lse[b, h] = ref.forward(q[b, h], k[b, (h + 1) % H], v[b, h], c, wl, wr, br)
    return o, lse


def _planted_backward_dense_batch_swap(q, k, v, do, c, wl, wr, br=False, heads=None):
    B_, H = q.shape[:2]
    dq, dk, dv = ref.backward_dense(q, k, v, do, c, wl, wr, br, heads=heads)
    for b, h in heads if heads is not None else [(b, h) for b in range(B_) for h in range(H)]:
        # dK stored into the other batch's slot
        dk[(b + 1) % B_, h] = ref.backward(q[b, h], k[b, h], v[b, h], do[b, h], c, wl, wr, br)[1]
    return dq, dk, dv


def test_planted_dense_wrapper_index_slips_are_caught():
    w = (INF, INF, False)
    with pytest.raises(AssertionError):
        _check_dense_wrappers(_planted_forward_dense_wrong_head, ref.backward_dense, w)
    with pytest.raises(AssertionError):
        _check_dense_wrappers(ref.forward_dense, _planted_backward_dense_batch_swap, w)


# ---------------------------------------------------------------------------
# Additive bias (AOTriton 0.10b "Known Problems", 0.14b "Kernel Bug Fixes"):
# logits c <q_i, k_j> + B_ij on allowed pairs, dB = dS.
# ---------------------------------------------------------------------------

BIAS_WINDOWS = [(INF, INF, False), (CTL, 0, False), (2, 1, True), (CBR, 0, True), (3, -2, False)]


def _brute_bias(q, k, v, do, c, w, bias):
    """Independent formulation: dense mask, torch softmax over c QK^T + B,
    autograd for every input including the bias."""
    sq, sk = q.shape[0], k.shape[0]
    wl, wr, br = w
    d = sk - sq
    mask = torch.zeros(sq, sk, dtype=torch.bool)
    for i in range(sq):
        for j in range(sk):
            if wl == CTL:
                ok = j <= i
            elif wl == CBR:
                ok = j <= i + d
            else:
                lo_ok = True if wl == INF else (j >= i - (wl - d if br else wl))
                hi_ok = True if wr == INF else (j <= i + (wr + d if br else wr))
                ok = lo_ok and hi_ok
            mask[i, j] = ok
    tq, tk, tv, tb = (torch.tensor(a, dtype=torch.float64, requires_grad=True)
                      for a in (q, k, v, bias))
    s = (tq @ tk.T) * c + tb
    s = s.masked_fill(~mask, float("-inf"))
    rows = mask.any(1)
    lse = torch.logsumexp(s, dim=1)
    o = torch.zeros(sq, v.shape[1], dtype=torch.float64)
    if rows.any():
        p = torch.softmax(s[rows], dim=1)
        o = o.index_put((rows.nonzero()[:, 0],), p @ tv)
    ((o * torch.tensor(do)).sum() + 0.0 * (tq.sum() + tk.sum() + tv.sum() + tb.sum())).backward()
    return (o.detach().numpy(), lse.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(),
            tv.grad.numpy(), tb.grad.numpy())


@pytest.mark.parametrize("w", BIAS_WINDOWS)
@pytest.mark.parametrize("c", [0.6, -0.3])
def test_bias_matches_independent_brute_force(w, c):
    sq, sk, d = 6, 9, 4
    q, k, v, do = (_rand(s, 60 + i) for i, s in enumerate([(sq, d), (sk, d), (sk, d), (sq, d)]))
    bias = 2.0 * _rand((sq, sk), 70)
    o, lse = ref.forward(q, k, v, c, *w, bias=bias)
    dq, dk, dv, db = ref.backward(q, k, v, do, c, *w, bias=bias)
    bo, blse, bdq, bdk, bdv, bdb = _brute_bias(q, k, v, do, c, w, bias)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(blse))
    fin = np.isfinite(blse)
    np.testing.assert_allclose(lse[fin], blse[fin], rtol=1e-12, atol=1e-12)
    for a, b in ((dq, bdq), (dk, bdk), (dv, bdv), (db, bdb)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("w", BIAS_WINDOWS[:3])
def test_bias_gradient_matches_central_differences(w):
    sq, sk, d = 5, 7, 3
    q, k, v, do = (_rand(s, 80 + i) for i, s in enumerate([(sq, d), (sk, d), (sk, d), (sq, d)]))
    bias = _rand((sq, sk), 90)
    *_, db = ref.backward(q, k, v, do, 0.7, *w, bias=bias)

    def loss(b):
        o, _ = ref.forward(q, k, v, 0.7, *w, bias=b)
        return float((o * do).sum())
    h = 1e-6
    num = np.zeros_like(bias)
    for idx in np.ndindex(bias.shape):
        old = bias[idx]
        bias[idx] = old + h
        fp = loss(bias)
        bias[idx] = old - h
        fm = loss(bias)
        bias[idx] = old
        num[idx] = (fp - fm) / (2 * h)
    np.testing.assert_allclose(db, num, rtol=1e-6, atol=1e-7)
    assert np.all(db[~ref.allowed(sq, sk, *w)] == 0)


def test_bias_constant_along_rows_shifts_lse_only():
    sq, sk, d = 7, 10, 4
    q, k, v = _rand((sq, d), 1), _rand((sk, d), 2), _rand((sk, d), 3)
    shift = _rand((sq, 1), 4)
    o, lse = ref.forward(q, k, v, 0.5, INF, INF)
    ob, lseb = ref.forward(q, k, v, 0.5, INF, INF, bias=np.broadcast_to(shift, (sq, sk)))
    np.testing.assert_allclose(ob, o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lseb, lse + shift[:, 0], rtol=1e-13)
    oz, lsez = ref.forward(q, k, v, 0.5, 2, 1, True, bias=np.zeros((sq, sk)))
    o2, lse2 = ref.forward(q, k, v, 0.5, 2, 1, True)
    np.testing.assert_array_equal(oz, o2)
    np.testing.assert_array_equal(lsez, lse2)


def test_planted_bias_inside_the_scale_is_caught():
    # a slip that adds the bias before the scale, c (qk + B), fails the brute force
    sq, sk, d = 4, 6, 3
    q, k, v, do = (_rand(s, 95 + i) for i, s in enumerate([(sq, d), (sk, d), (sk, d), (sq, d)]))
    bias = _rand((sq, sk), 99)
    c = 0.4
    mask = ref.allowed(sq, sk, INF, INF, False)
    bad = ref._probs_block(q, k, c, mask, c * bias)[0] @ v   # c (qk + B)
    bo = _brute_bias(q, k, v, do, c, (INF, INF, False), bias)[0]
    assert not np.allclose(bad, bo, atol=1e-6)

"""fp64 CPU oracle for masked softmax attention and its gradient.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only the tests, the smoke check in ``__graft_entry__`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (no helpers, no tables, no constants module).

What it computes
----------------
FlashAttention, as the aotriton README (awesome.ecosyste.ms mirror, section
"Kernel Support") names it, reaches exactly -- up to rounding order -- plain
masked softmax attention.  So this oracle is that definition written out, per
(sequence, head), in float64:

    S_ij  = c * <q_i, k_j>                         (c = sm_scale, any real)
    row i with no allowed j:  O_i = 0, LSE_i = -inf
    otherwise LSE_i = log sum_{allowed j} exp(S_ij)   (natural log)
              P_ij  = exp(S_ij - LSE_i) on allowed j, 0 elsewhere
              O_i   = sum_j P_ij v_j

and the gradient of the scalar <dO, O> (no gradient flows through LSE):

    dV = P^T dO,  dP = dO V^T,  delta_i = sum_d dO_id O_id,
    dS = P o (dP - delta),  dQ = c dS K,  dK = c dS^T Q.

The mask is the Generalized Sliding Window of the AOTriton 0.10b release notes
(newreleases.io, section "Major Changes from Release 0.9 Beta": causal masks
are windows, and window_left / window_right may be negative) with the
principal-diagonal choice of the 0.15b release notes (github.com releases,
section "Bottom-Right Aligned Sliding Windows": a numeric window becomes
L = wl - d, R = wr + d with d = seqlen_k - seqlen_q taken per sequence;
sentinel windows are never shifted).

Additive bias (the AOTriton 0.10b release notes, "Known Problems", and the
0.14b notes, "Kernel Bug Fixes", where the bias is converted to fp32 before
it is added): an optional matrix B [Sq, Sk] per (sequence, head) enters the
logits, S_ij = c * <q_i, k_j> + B_ij on allowed (i, j) only (a bias never
unmasks a pair); its gradient is dB = dS.

Readings where the pages are silent:
  * a row i may attend key j iff j >= i - L and j <= i + R, both ends
    inclusive, an unbounded side imposing nothing;
  * the causal sentinels name their own diagonal: CAUSAL_TOP_LEFT allows
    j <= i, CAUSAL_BOTTOM_RIGHT allows j <= i + d, whatever the diagonal bit;
    window_right is ignored when window_left holds a sentinel;
  * LSE is the natural log with the scale inside the exponent;
  * fully masked rows give O = 0 and LSE = -inf and no gradient.

Parity pins: every function here is pinned in ``tests/test_oracle.py`` by
central finite differences, an independent dense brute force, closed forms
(window (0, 0), scale 0, S_q = S_k = 1), invariants and hand-derived mask
fixtures under ``tests/golden/``.  No function is left unpinned.
"""

from __future__ import annotations

import numpy as np

# Window encodings of the C interface (values chosen by this library; the
# pages do not print them).  They are restated here, not imported, so the
# oracle shares nothing with the product.
WINDOW_INF = 2**31 - 1
CAUSAL_TOP_LEFT = -(2**31)
CAUSAL_BOTTOM_RIGHT = -(2**31) + 1

ROW_BLOCK = 512


def effective_window(window_left, window_right, bottom_right, seqlen_q, seqlen_k):
    """(L, R) of one sequence; None marks an unbounded side.

    0.15b release notes, "Bottom-Right Aligned Sliding Windows": TOP_LEFT keeps
    the numeric window, BOTTOM_RIGHT shifts it to L = wl - d, R = wr + d with
    d = seqlen_k - seqlen_q of this sequence; sentinel windows are not shifted.
    """
    d = int(seqlen_k) - int(seqlen_q)
    if window_left == CAUSAL_TOP_LEFT:
        return None, 0
    if window_left == CAUSAL_BOTTOM_RIGHT:
        return None, d
    L = None if window_left == WINDOW_INF else int(window_left)
    R = None if window_right == WINDOW_INF else int(window_right)
    if bottom_right:
        if L is not None:
            L = L - d
        if R is not None:
            R = R + d
    return L, R


def allowed(seqlen_q, seqlen_k, window_left, window_right, bottom_right, rows=None):
    """Boolean mask [len(rows), seqlen_k]: may query row i attend key j."""
    L, R = effective_window(window_left, window_right, bottom_right, seqlen_q, seqlen_k)
    if rows is None:
        rows = np.arange(seqlen_q)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(seqlen_k, dtype=np.int64)[None, :]
    m = np.ones((i.shape[0], seqlen_k), dtype=bool)
    if L is not None:
        m &= j >= i - L
    if R is not None:
        m &= j <= i + R
    return m


def allowed_count(seqlen_q, seqlen_k, window_left, window_right, bottom_right):
    """Number of allowed (i, j) pairs of one sequence, by summing the mask."""
    total = 0
    for r0 in range(0, seqlen_q, ROW_BLOCK):
        rows = np.arange(r0, min(r0 + ROW_BLOCK, seqlen_q))
        total += int(allowed(seqlen_q, seqlen_k, window_left, window_right,
                             bottom_right, rows).sum())
    return total


def row_extent(seqlen_q, seqlen_k, window_left, window_right, bottom_right):
    """Per row: first and last allowed key and the count (first > last if none)."""
    lo = np.zeros(seqlen_q, dtype=np.int64)
    hi = np.full(seqlen_q, -1, dtype=np.int64)
    cnt = np.zeros(seqlen_q, dtype=np.int64)
    for r0 in range(0, seqlen_q, ROW_BLOCK):
        rows = np.arange(r0, min(r0 + ROW_BLOCK, seqlen_q))
        a = allowed(seqlen_q, seqlen_k, window_left, window_right, bottom_right, rows)
        c = a.sum(axis=1)
        cnt[rows] = c
        first = np.argmax(a, axis=1)
        last = seqlen_k - 1 - np.argmax(a[:, ::-1], axis=1)
        lo[rows] = np.where(c > 0, first, 1)
        hi[rows] = np.where(c > 0, last, 0)
    return lo, hi, cnt


def _probs_block(q, k, sm_scale, mask, bias=None):
    """P and LSE for a block of rows (fp64), fully masked rows -> 0 / -inf;
    ``bias`` [rows, Sk] is added to the scaled scores."""
    s = sm_scale * (q @ k.T)
    if bias is not None:
        s = s + np.asarray(bias, dtype=np.float64)
    nonempty = mask.any(axis=1)
    m = np.where(mask, s, -np.inf).max(axis=1, initial=-np.inf)
    m = np.where(nonempty, m, 0.0)
    e = np.where(mask, np.exp(s - m[:, None]), 0.0)
    l = e.sum(axis=1)
    lse = np.where(nonempty, m + np.log(np.where(nonempty, l, 1.0)), -np.inf)
    p = e / np.where(nonempty, l, 1.0)[:, None]
    return p, lse


def forward(q, k, v, sm_scale, window_left, window_right, bottom_right=False, rows=None,
            bias=None):
    """One (sequence, head): q [Sq, D], k [Sk, D], v [Sk, Dv] -> (O, LSE).

    ``rows`` (optional) computes only those query rows (each row of the
    definition depends on its own query only) and returns [len(rows), ...].
    ``bias`` (optional) [Sq, Sk] is added to the scaled scores.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    sq, sk = q.shape[0], k.shape[0]
    idx = np.arange(sq) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.zeros((len(idx), v.shape[1]), dtype=np.float64)
    lse = np.full(len(idx), -np.inf, dtype=np.float64)
    for r0 in range(0, len(idx), ROW_BLOCK):
        r1 = min(r0 + ROW_BLOCK, len(idx))
        sel = idx[r0:r1]
        mask = allowed(sq, sk, window_left, window_right, bottom_right, sel)
        p, lse[r0:r1] = _probs_block(q[sel], k, sm_scale, mask,
                                     None if bias is None else np.asarray(bias)[sel])
        o[r0:r1] = p @ v
    return o, lse


def probabilities(q, k, sm_scale, window_left, window_right, bottom_right=False):
    """The full P matrix of one (sequence, head); small inputs only."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    mask = allowed(q.shape[0], k.shape[0], window_left, window_right, bottom_right)
    p, _ = _probs_block(q, k, sm_scale, mask)
    return p


def delta(o, do):
    """Row sums of dO o O, the quantity the backward preprocess step produces
    (0.14b release notes, "Minor Changes": bwd_preprocess)."""
    return (np.asarray(do, dtype=np.float64) * np.asarray(o, dtype=np.float64)).sum(axis=-1)


def backward(q, k, v, do, sm_scale, window_left, window_right, bottom_right=False,
             rows=None, bias=None):
    """One (sequence, head): gradient of <dO, O> -> (dQ, dK, dV), or
    (dQ, dK, dV, dBias) when ``bias`` [Sq, Sk] is given (dBias = dS, zero on
    masked pairs).

    ``rows`` (optional) restricts dQ to those query rows; dK and dV always sum
    over every query row (they need all of them).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    sq, sk = q.shape[0], k.shape[0]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    db = None if bias is None else np.zeros((sq, sk), dtype=np.float64)
    for r0 in range(0, sq, ROW_BLOCK):
        r1 = min(r0 + ROW_BLOCK, sq)
        mask = allowed(sq, sk, window_left, window_right, bottom_right, np.arange(r0, r1))
        p, _ = _probs_block(q[r0:r1], k, sm_scale, mask,
                            None if bias is None else np.asarray(bias)[r0:r1])
        o_blk = p @ v
        dv += p.T @ do[r0:r1]
        dp = do[r0:r1] @ v.T
        dlt = delta(o_blk, do[r0:r1])
        ds = p * (dp - dlt[:, None])
        dq[r0:r1] = sm_scale * (ds @ k)
        dk += sm_scale * (ds.T @ q[r0:r1])
        if db is not None:
            db[r0:r1] = ds
    if rows is not None:
        dq = dq[np.asarray(rows)]
    if db is not None:
        return dq, dk, dv, db
    return dq, dk, dv


# ----------------------------------------------------------------------------
# Whole-tensor wrappers: dense BHSD and packed 1THD (0.14b release notes,
# "VarlenBits supersedes VarlenType": BHSD or 1THD, cumulative seqlens, LSE in
# HT or TH layout).
# ----------------------------------------------------------------------------

def forward_dense(q, k, v, sm_scale, window_left, window_right, bottom_right=False,
                  heads=None):
    """q [B, H, Sq, D], k/v [B, H, Sk, D] -> O [B, H, Sq, D], LSE [B, H, Sq].

    ``heads``: optional list of (b, h) pairs to compute; others stay NaN.
    """
    B, H, sq, _ = q.shape
    o = np.full(q.shape[:3] + (v.shape[3],), np.nan)
    lse = np.full((B, H, sq), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        o[b, h], lse[b, h] = forward(q[b, h], k[b, h], v[b, h], sm_scale,
                                     window_left, window_right, bottom_right)
    return o, lse


def backward_dense(q, k, v, do, sm_scale, window_left, window_right, bottom_right=False,
                   heads=None):
    """Dense BHSD gradient -> (dQ, dK, dV); ``heads`` as in forward_dense."""
    B, H = q.shape[:2]
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in pairs:
        dq[b, h], dk[b, h], dv[b, h] = backward(q[b, h], k[b, h], v[b, h], do[b, h],
                                                sm_scale, window_left, window_right,
                                                bottom_right)
    return dq, dk, dv


def forward_packed(q, k, v, cu_q, cu_k, sm_scale, window_left, window_right,
                   bottom_right=False, seqs=None):
    """Packed: q [Tq, H, D], k/v [Tk, H, D], cu_q/cu_k cumulative sums [n+1].

    Returns O [Tq, H, D] and LSE in HT layout [H, Tq].  Rows of sequences not in
    ``seqs`` stay NaN.
    """
    n = len(cu_q) - 1
    H = q.shape[1]
    o = np.full(q.shape[:2] + (v.shape[2],), np.nan)
    lse = np.full((H, q.shape[0]), np.nan)
    for s in (range(n) if seqs is None else seqs):
        q0, q1, k0, k1 = int(cu_q[s]), int(cu_q[s + 1]), int(cu_k[s]), int(cu_k[s + 1])
        for h in range(H):
            o[q0:q1, h], lse[h, q0:q1] = forward(q[q0:q1, h], k[k0:k1, h], v[k0:k1, h],
                                                 sm_scale, window_left, window_right,
                                                 bottom_right)
    return o, lse


def backward_packed(q, k, v, do, cu_q, cu_k, sm_scale, window_left, window_right,
                    bottom_right=False, seqs=None):
    """Packed gradient -> (dQ [Tq,H,D], dK [Tk,H,D], dV [Tk,H,Dv])."""
    n = len(cu_q) - 1
    H = q.shape[1]
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    for s in (range(n) if seqs is None else seqs):
        q0, q1, k0, k1 = int(cu_q[s]), int(cu_q[s + 1]), int(cu_k[s]), int(cu_k[s + 1])
        for h in range(H):
            g = backward(q[q0:q1, h], k[k0:k1, h], v[k0:k1, h], do[q0:q1, h], sm_scale,
                         window_left, window_right, bottom_right)
            dq[q0:q1, h], dk[k0:k1, h], dv[k0:k1, h] = g
    return dq, dk, dv


def lse_ht_to_th(lse_ht):
    """HT [H, T] (or dense [B, H, S]) -> TH [T, H] (or [B, S, H])."""
    return np.swapaxes(np.asarray(lse_ht), -1, -2)

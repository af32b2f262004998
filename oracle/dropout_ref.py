"""Dropout on the attention probabilities, for the oracle.

TEST INFRASTRUCTURE ONLY, like attn_ref: imported by tests/ alone, never by
the product path, and sharing nothing with the CUDA sources.

The pages draw the dropout randoms from Philox with 32-bit words in groups
of four (AOTriton 0.10b release notes, "Major Changes from Release 0.9
Beta": tl.randint4x moved from Philox64x4 to Philox32x4), the four randoms
of one counter used in generation order (AOTriton 0.14b release notes,
"Minor Changes from Release 0.13 Beta": the fast_philox word-order fix and
test_dropout_layout).  Philox4x32-10 is a counter-based generator with a
published definition (J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel
Random Numbers: As Easy as 1, 2, 3", SC '11); it is written here from that
definition: ten rounds of two 32 x 32 -> 64-bit multiplications (multipliers
0xD2511F53, 0xCD9E8D57), the key bumped by the Weyl constants (0x9E3779B9,
0xBB67AE85) between rounds.

Readings where the pages are silent (they fix the generator and the word
order, not the counter layout):
  * element (i, j) of head index bh = b * H + h (query row i, key column j,
    both sequence-local) takes word j % 4, in generation order, of
    Philox4x32-10 applied to the counter (j // 4, i, bh, offset) under the
    key (seed & 0xFFFFFFFF, seed >> 32);
  * the element is kept iff that word < floor((1 - p) * 2^32), and kept
    probabilities are scaled by 1 / (1 - p) (p = 1 keeps nothing: O = 0);
  * dropout applies to P after the softmax; LSE is that of the softmax
    without dropout, and the backward regenerates the same mask.

With a mask m and s = 1 / (1 - p), for the loss <dO, O>:
  O = (P o m s) V,  dV = (P o m s)^T dO,  dP = (dO V^T) o m s,
  delta_i = sum_j P_ij dP_ij = rowsum(dO o O),  dS = P o (dP - delta),
  dQ = c dS K,  dK = c dS^T Q.
"""

from __future__ import annotations

import numpy as np

from . import attn_ref as ref

PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(counter, key):
    """Philox4x32-10 on counters [..., 4] (uint32 values) with key [2]."""
    c = np.asarray(counter, dtype=np.uint64).copy()
    k0, k1 = np.uint64(int(key[0]) & 0xFFFFFFFF), np.uint64(int(key[1]) & 0xFFFFFFFF)
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = np.uint64(PHILOX_M0) * c[..., 0]   # < 2^64: exact in uint64
        p1 = np.uint64(PHILOX_M1) * c[..., 2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c = np.stack([hi1 ^ c[..., 1] ^ k0, lo1, hi0 ^ c[..., 3] ^ k1, lo0], axis=-1)
    return c.astype(np.uint32)


def keep_threshold(p):
    """Words below this integer are kept: floor((1 - p) * 2^32) in [0, 2^32]."""
    if not 0.0 <= p <= 1.0:
        raise ValueError("dropout probability must be in [0, 1]")
    return int(np.floor((1.0 - float(p)) * 2.0 ** 32))


def keep_mask(seed, offset, bh, rows, seqlen_k, p):
    """Boolean keep mask [len(rows), seqlen_k] of head index bh (seed: 64-bit,
    offset: 32-bit)."""
    rows = np.asarray(rows, dtype=np.int64)
    groups = np.arange((seqlen_k + 3) // 4, dtype=np.int64)
    ctr = np.zeros((len(rows), len(groups), 4), dtype=np.uint64)
    ctr[..., 0] = groups[None, :]
    ctr[..., 1] = rows[:, None]
    ctr[..., 2] = bh
    ctr[..., 3] = offset & 0xFFFFFFFF
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    words = words.reshape(len(rows), -1)[:, :seqlen_k].astype(np.uint64)
    return words < np.uint64(keep_threshold(p))


def _scale(p):
    return 0.0 if p >= 1.0 else 1.0 / (1.0 - p)


def forward(q, k, v, sm_scale, window_left, window_right, bottom_right, p, seed, offset, bh,
            bias=None):
    """One (sequence, head) with dropout -> (O, LSE); LSE without dropout.
    ``bias`` [Sq, Sk] (optional) is added to the scaled scores."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    sq, sk = q.shape[0], k.shape[0]
    mask = ref.allowed(sq, sk, window_left, window_right, bottom_right)
    probs, lse = ref._probs_block(q, k, sm_scale, mask, bias)
    m = keep_mask(seed, offset, bh, np.arange(sq), sk, p)
    return (probs * m * _scale(p)) @ v, lse


def backward(q, k, v, do, sm_scale, window_left, window_right, bottom_right, p, seed, offset,
             bh, bias=None):
    """One (sequence, head) with dropout: gradient of <dO, O> -> (dQ, dK, dV),
    or (dQ, dK, dV, dBias) with a ``bias`` (dBias = dS)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    sq, sk = q.shape[0], k.shape[0]
    mask = ref.allowed(sq, sk, window_left, window_right, bottom_right)
    probs, _ = ref._probs_block(q, k, sm_scale, mask, bias)
    ms = keep_mask(seed, offset, bh, np.arange(sq), sk, p) * _scale(p)
    pd = probs * ms
    o = pd @ v
    dv = pd.T @ do
    dp = (do @ v.T) * ms
    dlt = ref.delta(o, do)
    ds = probs * (dp - dlt[:, None])
    if bias is not None:
        return sm_scale * (ds @ k), sm_scale * (ds.T @ q), dv, ds
    return sm_scale * (ds @ k), sm_scale * (ds.T @ q), dv

"""Exact checks of the window mask and the varlen indexing on the GPU.

Count probe: with sm_scale = 0 every allowed key has the same score, so
exp(LSE_i) is the number of keys row i may see; it must round to the oracle's
count exactly, and LSE must be -inf exactly on the oracle's empty rows.

Edge probe: scores strictly increasing in the key index with gaps of 32 (so
softmax puts all but ~2^-46 of the weight on one key) and V_j holding the
base-16 digits of j make O_i read out the last allowed key hi(i); negating the
query reads out the first allowed key lo(i).  Both are compared with the
oracle's mask integers.  All probe values are exact in fp16 and bf16.
"""

import numpy as np
import pytest
import torch

from attn_cases import CBR, CTL, INF, binding
from oracle import attn_ref as ref

pytestmark = pytest.mark.gpu

WINDOWS = [(INF, INF, False), (CTL, 0, False), (CTL, 0, True), (CBR, 0, False), (CBR, 0, True),
           (INF, 0, True), (256, 0, False), (256, 0, True), (-64, 128, False), (-64, 128, True),
           (7, -3, True), (0, 0, False), (2, -5, False), (-300, 500, True)]
SIZES = [(300, 300), (200, 517), (517, 200), (1, 129), (1000, 1100)]


def _count_probe_inputs(B_, H, sq, sk, D, dtype, dev):
    g = torch.Generator().manual_seed(sq * 7 + sk)
    q = torch.randn(B_, H, sq, D, generator=g).to(dtype).to(dev)
    k = torch.randn(B_, H, sk, D, generator=g).to(dtype).to(dev)
    v = torch.randn(B_, H, sk, D, generator=g).to(dtype).to(dev)
    return q, k, v


def _check_counts(lse, sq, sk, w):
    _, _, cnt = ref.row_extent(sq, sk, *w)
    lse = lse.astype(np.float64)
    empty = cnt == 0
    assert np.array_equal(np.isneginf(lse), np.broadcast_to(empty, lse.shape))
    got = np.rint(np.exp(np.where(np.isneginf(lse), 0.0, lse)))
    want = np.broadcast_to(cnt, lse.shape)
    assert np.array_equal(got[..., ~empty], want[..., ~empty].astype(np.float64))


@pytest.mark.parametrize("w", WINDOWS, ids=str)
@pytest.mark.parametrize("sq,sk", SIZES, ids=str)
@pytest.mark.parametrize("D", [64, 128])
def test_count_probe_dense(D, sq, sk, w):
    B = binding()
    dev = torch.device("cuda")
    q, k, v = _count_probe_inputs(2, 2, sq, sk, D, torch.bfloat16, dev)
    _, lse = B.forward(q, k, v, sm_scale=0.0, window=w[:2], bottom_right=w[2])
    torch.cuda.synchronize()
    _check_counts(lse.cpu().numpy(), sq, sk, w)


@pytest.mark.parametrize("w", WINDOWS, ids=str)
def test_count_probe_packed(w):
    B = binding()
    dev = torch.device("cuda")
    sq = [1, 300, 0, 129, 700, 513]
    sk = [5, 300, 40, 100, 900, 1]
    from scaled_dot_product_12_b200 import synth
    cu_q, cu_k = synth.cumsum0(sq), synth.cumsum0(sk)
    H, D = 3, 128
    g = torch.Generator().manual_seed(3)
    q = torch.randn(sum(sq), H, D, generator=g).bfloat16().to(dev)
    k = torch.randn(sum(sk), H, D, generator=g).bfloat16().to(dev)
    v = torch.randn(sum(sk), H, D, generator=g).bfloat16().to(dev)
    _, lse = B.forward(q, k, v, sm_scale=0.0, window=w[:2], bottom_right=w[2],
                       cu_seqlens_q=cu_q.to(dev), cu_seqlens_k=cu_k.to(dev),
                       max_seqlen_q=max(sq), max_seqlen_k=max(sk), lse_layout="TH")
    torch.cuda.synchronize()
    lse = lse.cpu().numpy()  # [T, H]
    for s in range(len(sq)):
        if sq[s] == 0:
            continue
        _check_counts(lse[cu_q[s]:cu_q[s + 1]].T, sq[s], sk[s], w)


def _edge_inputs(sq, sk, D, dtype, sign):
    """q = sign * (2048, 32, 0...), k_j = (j // 64, j % 64, 0...): S_ij = sign * 32 j.
    V_j = base-16 digits of j in columns 0..3."""
    j = torch.arange(sk)
    q = torch.zeros(sq, D)
    q[:, 0] = 2048.0 * sign
    q[:, 1] = 32.0 * sign
    k = torch.zeros(sk, D)
    k[:, 0] = (j // 64).float()
    k[:, 1] = (j % 64).float()
    v = torch.zeros(sk, D)
    for c in range(4):
        v[:, c] = ((j >> (4 * c)) & 15).float()
    return q.to(dtype), k.to(dtype), v.to(dtype)


def _decode(o):
    d = np.rint(o[..., :4].astype(np.float64)).astype(np.int64)
    return d[..., 0] + 16 * d[..., 1] + 256 * d[..., 2] + 4096 * d[..., 3]


@pytest.mark.parametrize("w", WINDOWS, ids=str)
@pytest.mark.parametrize("sq,sk", SIZES, ids=str)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
def test_edge_probe_dense(dtype, sq, sk, w):
    B = binding()
    dev = torch.device("cuda")
    lo, hi, cnt = ref.row_extent(sq, sk, *w)
    nonempty = cnt > 0
    for sign, want in ((1.0, hi), (-1.0, lo)):
        q, k, v = _edge_inputs(sq, sk, 64, dtype, sign)
        o, lse = B.forward(q[None, None].to(dev), k[None, None].to(dev), v[None, None].to(dev),
                           sm_scale=1.0, window=w[:2], bottom_right=w[2])
        torch.cuda.synchronize()
        o = o[0, 0].float().cpu().numpy()
        assert np.array_equal(_decode(o)[nonempty], want[nonempty])
        assert np.all(o[~nonempty] == 0)


@pytest.mark.parametrize("w", WINDOWS, ids=str)
def test_edge_probe_packed(w):
    B = binding()
    dev = torch.device("cuda")
    from scaled_dot_product_12_b200 import synth
    sq = [3, 400, 129, 1000, 1]
    sk = [700, 300, 129, 1100, 64]
    cu_q, cu_k = synth.cumsum0(sq), synth.cumsum0(sk)
    for sign in (1.0, -1.0):
        parts = [_edge_inputs(a, b, 64, torch.bfloat16, sign) for a, b in zip(sq, sk)]
        q = torch.cat([p[0] for p in parts])[:, None].to(dev)
        k = torch.cat([p[1] for p in parts])[:, None].to(dev)
        v = torch.cat([p[2] for p in parts])[:, None].to(dev)
        o, _ = B.forward(q, k, v, sm_scale=1.0, window=w[:2], bottom_right=w[2],
                         cu_seqlens_q=cu_q.to(dev), cu_seqlens_k=cu_k.to(dev),
                         max_seqlen_q=max(sq), max_seqlen_k=max(sk))
        torch.cuda.synchronize()
        o = o[:, 0].float().cpu().numpy()
        for s in range(len(sq)):
            lo, hi, cnt = ref.row_extent(sq[s], sk[s], *w)
            rows = o[cu_q[s]:cu_q[s + 1]]
            ne = cnt > 0
            want = hi if sign > 0 else lo
            assert np.array_equal(_decode(rows)[ne], want[ne]), (s, sign)
            assert np.all(rows[~ne] == 0)


# ---------------------------------------------------------------------------
# Backward edge probe.  Row i's scores are centred on the oracle's edge key
# e(i) = hi(i) (or lo(i) with the sign flipped): S_ij = 32 (j - e(i)), exact
# in fp16 / bf16 operands and in fp32.  If the backward admits exactly the
# oracle's keys, P_i is one-hot on e(i) to within e^-32, and with
# dO_i = unit vector (i mod 8), dV_j[c] is the number of rows i = c (mod 8)
# whose edge key is j: an exact small integer.  A key the backward wrongly
# admits past the edge would carry a positive score and take the weight; a
# dropped edge key would move it inwards; either changes the counts.  V holds
# base-16 digits of the key index, and O / LSE are the oracle's, so
# dS = P o (dP - delta) vanishes wherever P is right: dQ and dK must be ~0.
# Keys that no row may see get dK = dV = 0 exactly.
# ---------------------------------------------------------------------------

def _bwd_edge_inputs(sq, sk, D, dtype, edge, sign):
    j = torch.arange(sk)
    e = torch.as_tensor(np.maximum(edge, 0), dtype=torch.int64)
    q = torch.zeros(sq, D)
    q[:, 0], q[:, 1] = 2048.0 * sign, 32.0 * sign
    q[:, 2], q[:, 3] = -2048.0 * sign * (e // 64).float(), -32.0 * sign * (e % 64).float()
    k = torch.zeros(sk, D)
    k[:, 0], k[:, 1], k[:, 2], k[:, 3] = (j // 64).float(), (j % 64).float(), 1.0, 1.0
    v = torch.zeros(sk, D)
    for c in range(4):
        v[:, c] = ((j >> (4 * c)) & 15).float()
    do = torch.zeros(sq, D)
    do[torch.arange(sq), torch.arange(sq) % 8] = 1.0
    return q.to(dtype), k.to(dtype), v.to(dtype), do.to(dtype)


def _bwd_edge_expect(sq, sk, edge, cnt):
    want = np.zeros((sk, 8))
    for i in range(sq):
        if cnt[i] > 0:
            want[edge[i], i % 8] += 1
    return want


def _bwd_edge_run(B, q, k, v, do, w, dev, **kw):
    """Forward on the oracle side (O rounded to the dtype, LSE in fp32), then
    the GPU backward with those as its O and LSE."""
    from attn_cases import f64
    packed = "cu_seqlens_q" in kw
    if packed:
        cq, ck = kw["cu_seqlens_q"].cpu().numpy(), kw["cu_seqlens_k"].cpu().numpy()
        eo, el = ref.forward_packed(f64(q), f64(k), f64(v), cq, ck, 1.0, *w)
        lse = torch.tensor(el, dtype=torch.float32)            # HT [H, T]
    else:
        eo, el = ref.forward(f64(q), f64(k), f64(v), 1.0, *w)
        lse = torch.tensor(el, dtype=torch.float32)[None, None]
    o = torch.tensor(eo, dtype=torch.float32).to(q.dtype)
    if not packed:
        q, k, v, do, o = (t[None, None] for t in (q, k, v, do, o))
    dq, dk, dv, _ = B.backward(do.to(dev), q.to(dev), k.to(dev), v.to(dev), o.to(dev),
                               lse.to(dev), sm_scale=1.0, window=w[:2], bottom_right=w[2], **kw)
    torch.cuda.synchronize()
    assert B.device_status(dev) == 0
    sq_ = (lambda t: t.float().cpu().numpy().reshape(-1, t.shape[-1]))
    return sq_(dq), sq_(dk), sq_(dv)


def _bwd_edge_check(dq, dk, dv, sq, sk, w, sign):
    lo, hi, cnt = ref.row_extent(sq, sk, *w)
    edge = hi if sign > 0 else lo
    want = _bwd_edge_expect(sq, sk, edge, cnt)
    got = dv[:, :8].astype(np.float64)
    assert np.abs(got - np.rint(got)).max(initial=0) < 1e-3
    assert np.array_equal(np.rint(got), want), "dV edge counts differ"
    assert np.abs(dq).max(initial=0) <= 1e-3 and np.abs(dk).max(initial=0) <= 1e-3
    seen = ref.allowed(sq, sk, *w).any(axis=0)
    assert np.all(dk[~seen] == 0) and np.all(dv[~seen] == 0), "unseen keys must get 0"


@pytest.mark.parametrize("w", WINDOWS, ids=str)
@pytest.mark.parametrize("sq,sk", SIZES, ids=str)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
def test_backward_edge_probe_dense(dtype, D, sq, sk, w):
    B = binding()
    dev = torch.device("cuda")
    lo, hi, cnt = ref.row_extent(sq, sk, *w)
    for sign, edge in ((1.0, hi), (-1.0, lo)):
        q, k, v, do = _bwd_edge_inputs(sq, sk, D, dtype, edge, sign)
        dq, dk, dv = _bwd_edge_run(B, q, k, v, do, w, dev)
        _bwd_edge_check(dq, dk, dv, sq, sk, w, sign)


@pytest.mark.parametrize("w", WINDOWS, ids=str)
def test_backward_edge_probe_packed(w):
    B = binding()
    dev = torch.device("cuda")
    from scaled_dot_product_12_b200 import synth
    sq = [3, 400, 129, 1000, 1, 0]
    sk = [700, 300, 129, 1100, 64, 5]
    cu_q, cu_k = synth.cumsum0(sq), synth.cumsum0(sk)
    for sign in (1.0, -1.0):
        parts = []
        for a, b in zip(sq, sk):
            lo, hi, _ = ref.row_extent(a, b, *w)
            parts.append(_bwd_edge_inputs(a, b, 64, torch.bfloat16, hi if sign > 0 else lo, sign))
        q, k, v, do = (torch.cat([p[n] for p in parts])[:, None] for n in range(4))
        dq, dk, dv = _bwd_edge_run(B, q, k, v, do, w, dev, cu_seqlens_q=cu_q.to(dev),
                                   cu_seqlens_k=cu_k.to(dev), max_seqlen_q=max(sq),
                                   max_seqlen_k=max(sk))
        for s in range(len(sq)):
            rq = slice(int(cu_q[s]), int(cu_q[s + 1]))
            rk = slice(int(cu_k[s]), int(cu_k[s + 1]))
            _bwd_edge_check(dq[rq], dk[rk], dv[rk], sq[s], sk[s], w, sign)

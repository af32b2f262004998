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

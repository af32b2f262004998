"""Dropout in the kernels against the dropout oracle (oracle/dropout_ref.py).

* The keep mask is compared bit for bit: with V the identity (Sk = D) the
  forward's O_ij is P_ij m_ij / (1 - p), zero exactly where the element was
  dropped; with dO the identity (Sq = D) the backward's dV_j[i] is the same
  for query i, over many key tiles.  Both zero patterns must equal the
  oracle's Philox4x32-10 mask (AOTriton 0.10b release notes, "Major Changes
  from Release 0.9 Beta": Philox with 32-bit words in groups of four; 0.14b,
  "Minor Changes from Release 0.13 Beta": words used in generation order).
* O, LSE, dQ, dK, dV match the oracle within the usual tolerances, dense and
  packed, under several windows; LSE equals the LSE without dropout.
"""

import numpy as np
import pytest
import torch

from attn_cases import (CBR, CTL, INF, assert_grads, assert_o_lse, binding, dense_inputs, f64,
                        packed_inputs)
from oracle import dropout_ref as dr

pytestmark = pytest.mark.gpu
SEED = 0x0123_4567_89AB_CDEF


def _f32(p):
    return float(np.float32(p))


@pytest.mark.parametrize("p", [0.5, 0.17])
@pytest.mark.parametrize("H,Sq", [(3, 300), (1, 129)])
def test_forward_keep_mask_is_exact(p, H, Sq):
    B = binding()
    dev = torch.device("cuda")
    D = Sk = 128
    g = torch.Generator().manual_seed(3)
    q = torch.randn(2, H, Sq, D, generator=g).bfloat16()
    k = torch.randn(2, H, Sk, D, generator=g).bfloat16()
    v = torch.eye(Sk, D).expand(2, H, Sk, D).contiguous().bfloat16()
    o, _ = B.forward(q.to(dev), k.to(dev), v.to(dev), sm_scale=D ** -0.5, dropout_p=p,
                     philox_seed=SEED, philox_offset=11)
    torch.cuda.synchronize()
    o = o.float().cpu().numpy()
    for b in range(2):
        for h in range(H):
            want = dr.keep_mask(SEED, 11, b * H + h, np.arange(Sq), Sk, _f32(p))
            assert np.array_equal(o[b, h] != 0, want), (b, h)


@pytest.mark.parametrize("p", [0.5, 0.3])
@pytest.mark.parametrize("D", [64, 128])
def test_backward_keep_mask_is_exact(p, D):
    B = binding()
    dev = torch.device("cuda")
    H, Sq, Sk = 2, D, 700
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, H, Sq, D, generator=g).bfloat16().to(dev)
    k = torch.randn(1, H, Sk, D, generator=g).bfloat16().to(dev)
    v = torch.randn(1, H, Sk, D, generator=g).bfloat16().to(dev)
    do = torch.eye(Sq, D).expand(1, H, Sq, D).contiguous().bfloat16().to(dev)
    kw = dict(sm_scale=D ** -0.5, dropout_p=p, philox_seed=SEED, philox_offset=5)
    o, lse = B.forward(q, k, v, **kw)
    _, _, dv, _ = B.backward(do, q, k, v, o, lse, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    dv = dv.float().cpu().numpy()
    for h in range(H):
        want = dr.keep_mask(SEED, 5, h, np.arange(Sq), Sk, _f32(p))   # [Sq, Sk]
        assert np.array_equal(dv[0, h][:, :Sq] != 0, want.T), h


WINDOWS = [(INF, INF, False), (CTL, 0, False), (256, 0, True), (-64, 128, False), (CBR, 0, True)]


def _zero_bound(q, k, o, do, scale):
    """Where the oracle's gradient is exactly 0 by cancellation (a query row
    with one allowed key: dS = P (m dP / (1 - p) - delta) = 0), the kernel's
    delta comes from the 16-bit O, off by up to 2^-8 relative per term, so
    |dQ| <= scale * max|K| * max_i sum_d |dO_id O_id| * 2^-8 (2^-8: twice the
    bf16 rounding)."""
    s = (np.abs(f64(do) * f64(o))).sum(axis=-1).max()
    return scale * np.abs(f64(k)).max() * s * 2.0 ** -8 + 1e-3


@pytest.mark.parametrize("w", WINDOWS, ids=str)
@pytest.mark.parametrize("D,dtype", [(64, torch.float16), (128, torch.bfloat16)], ids=["64fp16", "128bf16"])
@pytest.mark.parametrize("p", [0.17, 0.5])
def test_dense_dropout_matches_the_oracle(p, D, dtype, w):
    B = binding()
    dev = torch.device("cuda")
    Bn, H, Sq, Sk = 2, 2, 333, 300
    q, k, v, do = dense_inputs(Bn, H, Sq, Sk, D, dtype, 77)
    kw = dict(sm_scale=D ** -0.5, window=w[:2], bottom_right=w[2], dropout_p=p,
              philox_seed=SEED + 1, philox_offset=3)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = B.forward(qd, kd, vd, **kw)
    o0, lse0 = B.forward(qd, kd, vd, **dict(kw, dropout_p=0.0))
    dq, dk, dv, _ = B.backward(dod, qd, kd, vd, o, lse, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.equal(lse, lse0), "LSE is that of the softmax without dropout"
    for b in range(Bn):
        for h in range(H):
            args = (f64(q[b, h]), f64(k[b, h]), f64(v[b, h]))
            dargs = (D ** -0.5, *w, _f32(p), SEED + 1, 3, b * H + h)
            eo, el = dr.forward(*args, *dargs)
            assert_o_lse(o[b, h].float().cpu().numpy(), lse[b, h].cpu().numpy(), eo, el, dtype,
                         what=f"{(b, h)}")
            eg = dr.backward(*args, f64(do[b, h]), *dargs)
            zb = _zero_bound(q[b, h], k[b, h], o[b, h].cpu(), do[b, h], D ** -0.5)
            assert_grads([t[b, h].float().cpu().numpy() for t in (dq, dk, dv)], eg,
                         what=f"{(b, h)}", zero_abs=zb)


@pytest.mark.parametrize("w", [(256, 0, True), (CTL, 0, False)], ids=str)
def test_packed_dropout_matches_the_oracle(w):
    B = binding()
    dev = torch.device("cuda")
    sq, sk = [300, 1, 129, 517], [310, 64, 129, 400]
    H, D, p = 2, 128, 0.25
    q, k, v, do, cu_q, cu_k = packed_inputs(sq, sk, H, D, torch.bfloat16, 8)
    kw = dict(sm_scale=D ** -0.5, window=w[:2], bottom_right=w[2], cu_seqlens_q=cu_q.to(dev),
              cu_seqlens_k=cu_k.to(dev), max_seqlen_q=max(sq), max_seqlen_k=max(sk),
              lse_layout="TH", dropout_p=p, philox_seed=SEED + 2, philox_offset=0)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = B.forward(qd, kd, vd, **kw)
    dq, dk, dv, _ = B.backward(dod, qd, kd, vd, o, lse, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    o, lse, dq, dk, dv = (t.float().cpu() for t in (o, lse, dq, dk, dv))
    for s in range(len(sq)):
        rq = slice(int(cu_q[s]), int(cu_q[s + 1]))
        rk = slice(int(cu_k[s]), int(cu_k[s + 1]))
        for h in range(H):
            args = (f64(q[rq, h]), f64(k[rk, h]), f64(v[rk, h]))
            dargs = (D ** -0.5, *w, _f32(p), SEED + 2, 0, s * H + h)
            eo, el = dr.forward(*args, *dargs)
            assert_o_lse(o[rq, h].numpy(), lse[rq, h].numpy(), eo, el, torch.bfloat16,
                         what=f"seq {s} head {h}")
            eg = dr.backward(*args, f64(do[rq, h]), *dargs)
            zb = _zero_bound(q[rq, h], k[rk, h], o[rq, h], do[rq, h], D ** -0.5)
            assert_grads([dq[rq, h].numpy(), dk[rk, h].numpy(), dv[rk, h].numpy()], eg,
                         what=f"seq {s} head {h}", zero_abs=zb)

"""Additive attention bias (AOTriton 0.10b release notes, "Known Problems";
0.14b notes, "Kernel Bug Fixes": the bias converted to fp32 before it is
added) and its gradient, against the fp64 oracle.

The bias is a [B, H, Sq, Sk] tensor in the dtype of Q, added to the scaled
scores on allowed pairs; dbias = dS.  Bias buffers carry NaN in the columns
past Sk (row strides rounded up) and, for varlen problems, in every element
past a sequence's lengths: none of them may reach a result.  dbias buffers
start as NaN: every element of a sequence must be written (0 on masked
pairs) and nothing past it."""

import numpy as np
import pytest
import torch

from attn_cases import (CBR, CTL, INF, TOL_GRAD, TOL_O, assert_grads, assert_o_lse, binding, f64,
                        local_errors, rel_fro, seed_of)
from oracle import attn_ref as ref
from oracle import dropout_ref as dr
from scaled_dot_product_12_b200 import synth

pytestmark = pytest.mark.gpu
NAN = float("nan")


def _bias_buffer(bias, fill=NAN):
    """bias [B, H, Sq, Sk] inside a NaN-filled buffer whose rows are padded
    by 16 columns past Sk rounded up to 8 (on the GPU)."""
    Bn, H, Sq, Sk = bias.shape
    pitch = (Sk + 7) // 8 * 8 + 16
    buf = torch.full((Bn, H, Sq, pitch), fill, dtype=bias.dtype, device="cuda")
    buf[..., :Sk] = bias.to("cuda")
    return buf, buf[..., :Sk]


def assert_dbias(got, want, w, what=""):
    """dbias [..., Sq, Sk] against the oracle: relative Frobenius error, per
    block too, and exactly 0 on the pairs window w masks (P = 0 there)."""
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: dbias not finite / not written"
    e = rel_fro(got, want)
    assert e <= TOL_GRAD, f"{what}: dbias relative Frobenius error {e}"
    worst = max(local_errors(got, want), key=lambda t: t[1])
    assert worst[1] <= TOL_GRAD, f"{what}: dbias block {worst[0]} error {worst[1]}"
    allowed = ref.allowed(got.shape[-2], got.shape[-1], *w)
    assert (got[..., ~allowed] == 0).all(), f"{what}: dbias non-zero on a masked pair"


def _dense_oracle(q, k, v, do, bias, scale, w):
    Bn, H = q.shape[:2]
    qn, kn, vn, don, bn = f64(q), f64(k), f64(v), f64(do), f64(bias)
    o = np.zeros(q.shape[:3] + (v.shape[3],))
    lse = np.zeros(q.shape[:3])
    dq, dk, dv = np.zeros(qn.shape), np.zeros(kn.shape), np.zeros(vn.shape)
    db = np.zeros(bn.shape)
    for b in range(Bn):
        for h in range(H):
            o[b, h], lse[b, h] = ref.forward(qn[b, h], kn[b, h], vn[b, h], scale, *w, bias=bn[b, h])
            dq[b, h], dk[b, h], dv[b, h], db[b, h] = ref.backward(
                qn[b, h], kn[b, h], vn[b, h], don[b, h], scale, *w, bias=bn[b, h])
    return o, lse, (dq, dk, dv), db


WINDOWS = [(INF, INF, False), (CTL, 0, False), (CBR, 0, True), (-64, 128, True), (100, 3, False),
           (0, -1, False)]


@pytest.mark.parametrize("w", WINDOWS, ids=str)
@pytest.mark.parametrize("dtype,D,scale", [(torch.bfloat16, 128, 0.09), (torch.float16, 64, -0.2),
                                           (torch.bfloat16, 72, 0.0)], ids=str)
def test_dense_bias_forward_backward(w, dtype, D, scale):
    B = binding()
    Bn, H, Sq, Sk = 2, 2, 300, 333
    q, k, v, do = synth.qkv_do((Bn, H, Sq, D), (Bn, H, Sk, D), seed_of("bias", w, D), dtype)
    bias = synth.bias((Bn, H, Sq, Sk), seed_of("bias-b", w, D), dtype, std=2.0)
    bbuf, bview = _bias_buffer(bias)
    dbuf, dview = _bias_buffer(torch.zeros_like(bias))
    dview.fill_(NAN)
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kw = dict(sm_scale=scale, window=w[:2], bottom_right=w[2], bias=bview)
    o, lse = B.forward(qd, kd, vd, **kw)
    dq, dk, dv, _ = B.backward(do.to(dev), qd, kd, vd, o, lse, dbias=dview, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    assert torch.isnan(dbuf[..., Sk:].float()).all(), "dbias written past Sk"
    eo, el, eg, edb = _dense_oracle(q, k, v, do, bias, scale, w)
    assert_o_lse(f64(o), f64(lse), eo, el, dtype, what=str(w))
    assert_grads([f64(t) for t in (dq, dk, dv)], list(eg), what=str(w))
    assert_dbias(f64(dview), edb, w, what=str(w))


@pytest.mark.parametrize("shape", [(1, 3), (2, 1), (1, 1)], ids=str)
def test_broadcast_bias(shape):
    # one bias for all batches and / or heads (stride 0 through expand)
    B = binding()
    Bn, H, Sq, Sk, D = 2, 3, 200, 264, 64  # rows of 528 bytes: a multiple of 16
    dtype = torch.bfloat16
    q, k, v, do = synth.qkv_do((Bn, H, Sq, D), (Bn, H, Sk, D), seed_of("bcast", shape), dtype)
    small = synth.bias(shape + (Sq, Sk), seed_of("bcast-b", shape), dtype, std=1.5)
    bias = small.to("cuda").expand(Bn, H, Sq, Sk)
    w = (CTL, 0, False)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = B.forward(qd, kd, vd, sm_scale=0.125, window=w[:2], bias=bias)
    dbias = torch.full((Bn, H, Sq, Sk), NAN, dtype=dtype, device="cuda")
    dq, dk, dv, _ = B.backward(do.cuda(), qd, kd, vd, o, lse, sm_scale=0.125, window=w[:2],
                               bias=bias, dbias=dbias)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    eo, el, eg, edb = _dense_oracle(q, k, v, do, bias.cpu(), 0.125, w)
    assert_o_lse(f64(o), f64(lse), eo, el, dtype)
    assert_grads([f64(t) for t in (dq, dk, dv)], list(eg))
    assert_dbias(f64(dbias), edb, w)


@pytest.mark.parametrize("D", [128, 64])
def test_dbias_without_bias_is_the_gradient_at_zero_bias(D):
    B = binding()
    Bn, H, Sq, Sk = 1, 2, 257, 300
    dtype = torch.float16
    q, k, v, do = synth.qkv_do((Bn, H, Sq, D), (Bn, H, Sk, D), seed_of("dbias0", D), dtype)
    w = (-10, 90, True)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = B.forward(qd, kd, vd, sm_scale=0.1, window=w[:2], bottom_right=w[2])
    dbuf, dbias = _bias_buffer(torch.zeros((Bn, H, Sq, Sk), dtype=dtype))
    dbias.fill_(NAN)
    dq, dk, dv, _ = B.backward(do.cuda(), qd, kd, vd, o, lse, sm_scale=0.1, window=w[:2],
                               bottom_right=w[2], dbias=dbias)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    eo, el, eg, edb = _dense_oracle(q, k, v, do, torch.zeros(Bn, H, Sq, Sk), 0.1, w)
    assert_grads([f64(t) for t in (dq, dk, dv)], list(eg))
    assert_dbias(f64(dbias), edb, w)


def test_large_position_bias_moves_the_row_maximum():
    # a bias that favours far keys (-slope |i - j| flipped) and spans ~ +-60:
    # the row maximum is set by the bias, not by the scores, and the running
    # maximum has to move many times along a row
    B = binding()
    Bn, H, Sq, Sk, D = 1, 2, 384, 640, 64
    dtype = torch.bfloat16
    q, k, v, do = synth.qkv_do((Bn, H, Sq, D), (Bn, H, Sk, D), seed_of("alibi"), dtype)
    i = torch.arange(Sq).view(Sq, 1).float()
    j = torch.arange(Sk).view(1, Sk).float()
    slopes = torch.tensor([0.1, -0.05]).view(H, 1, 1)
    bias = (slopes * (j - i)).view(1, H, Sq, Sk).to(dtype)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = B.forward(qd, kd, vd, sm_scale=0.125, bias=bias.cuda())
    dbias = torch.empty((Bn, H, Sq, Sk), dtype=dtype, device="cuda")
    dq, dk, dv, _ = B.backward(do.cuda(), qd, kd, vd, o, lse, sm_scale=0.125, bias=bias.cuda(),
                               dbias=dbias)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    eo, el, eg, edb = _dense_oracle(q, k, v, do, bias, 0.125, (INF, INF, False))
    assert_o_lse(f64(o), f64(lse), eo, el, dtype)
    assert_grads([f64(t) for t in (dq, dk, dv)], list(eg))
    assert_dbias(f64(dbias), edb, (INF, INF, False))


@pytest.mark.parametrize("D", [80, 64])
@pytest.mark.parametrize("w", [(INF, INF, False), (CBR, 0, True), (-32, 64, True)], ids=str)
def test_packed_bias(w, D):
    # bias [B, H, max_q, max_k], (i, j) within each sequence; NaN past every
    # sequence's lengths (head dim 64 stages the bias tiles in shared memory,
    # 80 loads them per thread)
    B = binding()
    sq, sk = [1, 130, 257, 64], [5, 300, 128, 64]
    H, dtype = 2, torch.bfloat16
    tq, tk = sum(sq), sum(sk)
    q, k, v, do = synth.qkv_do((tq, H, D), (tk, H, D), seed_of("pbias", w, D), dtype)
    Mq, Mk = max(sq), max(sk)
    full = synth.bias((len(sq), H, Mq, Mk), seed_of("pbias-b", w), dtype, std=2.0)
    for s in range(len(sq)):
        full[s, :, sq[s]:, :] = NAN
        full[s, :, :, sk[s]:] = NAN
    bbuf, bview = _bias_buffer(full)
    dbuf, dview = _bias_buffer(torch.zeros_like(full))
    dview.fill_(NAN)
    cu_q, cu_k = synth.cumsum0(sq).cuda(), synth.cumsum0(sk).cuda()
    kw = dict(sm_scale=0.11, window=w[:2], bottom_right=w[2], cu_seqlens_q=cu_q,
              cu_seqlens_k=cu_k, max_seqlen_q=Mq, max_seqlen_k=Mk, bias=bview)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o, lse = B.forward(qd, kd, vd, **kw)
    dq, dk, dv, _ = B.backward(do.cuda(), qd, kd, vd, o, lse, dbias=dview, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    got_db = f64(dview)
    cq, ck = [0], [0]
    for s in range(len(sq)):
        cq.append(cq[-1] + sq[s])
        ck.append(ck[-1] + sk[s])
    eo = np.zeros((tq, H, D))
    el = np.zeros((H, tq))
    eg = [np.zeros((tq, H, D)), np.zeros((tk, H, D)), np.zeros((tk, H, D))]
    qn, kn, vn, don, bn = f64(q), f64(k), f64(v), f64(do), f64(full)
    # dbias is compared over the whole [B, H, Mq, Mk] tensor (0 past the
    # sequences on both sides), like dQ / dK / dV: a one-row sequence alone
    # is held to the bf16 rounding floor of a typical block, not to 2 % of
    # its own small norm.
    want_db = np.zeros(got_db.shape)
    got_in = np.zeros(got_db.shape)
    for s in range(len(sq)):
        a, z, c, e = cq[s], cq[s + 1], ck[s], ck[s + 1]
        for h in range(H):
            bb = bn[s, h, :sq[s], :sk[s]]
            eo[a:z, h], el[h, a:z] = ref.forward(qn[a:z, h], kn[c:e, h], vn[c:e, h], 0.11, *w,
                                                 bias=bb)
            g = ref.backward(qn[a:z, h], kn[c:e, h], vn[c:e, h], don[a:z, h], 0.11, *w, bias=bb)
            eg[0][a:z, h], eg[1][c:e, h], eg[2][c:e, h] = g[:3]
            want_db[s, h, :sq[s], :sk[s]] = g[3]
        got_in[s, :, :sq[s], :sk[s]] = got_db[s, :, :sq[s], :sk[s]]
        allowed = ref.allowed(sq[s], sk[s], *w)
        assert (got_db[s, :, :sq[s], :sk[s]][:, ~allowed] == 0).all(), f"seq {s}: masked pair"
        # past the sequence: never written
        assert np.isnan(got_db[s, :, sq[s]:, :]).all()
        assert np.isnan(got_db[s, :, :, sk[s]:]).all()
    assert torch.isnan(dbuf[..., Mk:].float()).all()
    assert np.isfinite(got_in).all()
    assert rel_fro(got_in, want_db) <= TOL_GRAD
    worst = max(local_errors(got_in, want_db), key=lambda t: t[1])
    assert worst[1] <= TOL_GRAD, f"dbias block {worst[0]} error {worst[1]}"
    assert_o_lse(f64(o), f64(lse), eo, el, dtype)
    assert_grads([f64(t) for t in (dq, dk, dv)], eg)


def test_bias_with_dropout():
    B = binding()
    Bn, H, Sq, Sk, D = 1, 2, 200, 304, 64
    dtype, p, seed, offset = torch.bfloat16, 0.2, 1234, 7
    q, k, v, do = synth.qkv_do((Bn, H, Sq, D), (Bn, H, Sk, D), seed_of("bias-drop"), dtype)
    bias = synth.bias((Bn, H, Sq, Sk), seed_of("bias-drop-b"), dtype, std=1.0)
    w = (CBR, 0, True)
    qd, kd, vd, bd = q.cuda(), k.cuda(), v.cuda(), bias.cuda()
    kw = dict(sm_scale=0.125, window=w[:2], bottom_right=w[2], bias=bd, dropout_p=p,
              philox_seed=seed, philox_offset=offset)
    o, lse = B.forward(qd, kd, vd, **kw)
    dbias = torch.full((Bn, H, Sq, Sk), NAN, dtype=dtype, device="cuda")
    dq, dk, dv, _ = B.backward(do.cuda(), qd, kd, vd, o, lse, dbias=dbias, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    qn, kn, vn, don, bn = f64(q), f64(k), f64(v), f64(do), f64(bias)
    for h in range(H):
        eo, el = dr.forward(qn[0, h], kn[0, h], vn[0, h], 0.125, *w, p, seed, offset, h,
                            bias=bn[0, h])
        g = dr.backward(qn[0, h], kn[0, h], vn[0, h], don[0, h], 0.125, *w, p, seed, offset, h,
                        bias=bn[0, h])
        assert_o_lse(f64(o[0, h]), f64(lse[0, h]), eo, el, dtype, what=f"head {h}")
        assert_grads([f64(t[0, h]) for t in (dq, dk, dv)], list(g[:3]), what=f"head {h}")
        assert_dbias(f64(dbias[0, h]), g[3], w, what=f"head {h}")


def test_deterministic_backward_with_bias_is_bit_identical():
    B = binding()
    Bn, H, Sq, Sk, D = 1, 4, 1024, 1024, 128
    dtype = torch.bfloat16
    q, k, v, do = (t.cuda() for t in synth.qkv_do((Bn, H, Sq, D), (Bn, H, Sk, D),
                                                  seed_of("bias-det"), dtype))
    bias = synth.bias((Bn, H, Sq, Sk), seed_of("bias-det-b"), dtype).cuda()
    o, lse = B.forward(q, k, v, sm_scale=0.088, bias=bias)
    outs = []
    for _ in range(3):
        dbias = torch.empty_like(bias)
        dq, dk, dv, _ = B.backward(do, q, k, v, o, lse, sm_scale=0.088, bias=bias, dbias=dbias,
                                   deterministic=True)
        outs.append((dq.clone(), dk.clone(), dv.clone(), dbias.clone()))
    torch.cuda.synchronize()
    assert B.device_status() == 0
    for other in outs[1:]:
        for a, b in zip(outs[0], other):
            assert torch.equal(a, b)

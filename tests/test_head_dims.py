"""Head dimensions that are not multiples of 16, prime ones included (AOTriton
0.10b release notes, "Known Problems": non-power-of-two head dims; 0.14b,
"Minor Changes from Release 0.13 Beta": test_prime_hdim; 0.15b, "Kernel Bug
Fixes": an early-exit store bounded by the padded head dim, not the real one).

Each tensor row is D values inside a row whose byte stride is a multiple of
16 (D rounded up to 8): the columns past D hold NaN in the inputs and act as
canaries in the outputs.  TMA zero-fills the columns past D on loads, the MMA
widths round up to 16, and every store stops at D."""

import numpy as np
import pytest
import torch

from attn_cases import (CBR, CTL, INF, assert_grads, assert_o_lse, binding, f64, oracle_dense,
                        oracle_packed, seed_of)
from scaled_dot_product_12_b200 import synth

pytestmark = pytest.mark.gpu
NAN = float("nan")


def _padded(t, D):
    """t [..., D] inside a NaN-filled [..., round8(D)] buffer (on the GPU)."""
    Dp = (D + 7) // 8 * 8
    buf = torch.full(t.shape[:-1] + (Dp,), NAN, dtype=t.dtype, device="cuda")
    buf[..., :D] = t.to("cuda")
    return buf, buf[..., :D]


def _out_like(t, D):
    Dp = (D + 7) // 8 * 8
    buf = torch.full(t.shape[:-1] + (Dp,), NAN, dtype=t.dtype, device="cuda")
    return buf, buf[..., :D]


@pytest.mark.parametrize("D", [1, 8, 24, 40, 67, 72, 100, 127])
@pytest.mark.parametrize("w", [(INF, INF, False), (CTL, 0, False), (-64, 128, True), (0, -1, False)],
                         ids=str)
def test_dense_head_dims(D, w):
    B = binding()
    dtype = torch.bfloat16 if D % 2 else torch.float16
    q, k, v, do = synth.qkv_do((2, 2, 300, D), (2, 2, 333, D), seed_of("hdim", D, w), dtype)
    (qb, qd), (kb, kd), (vb, vd), (dob, dod) = (_padded(t, D) for t in (q, k, v, do))
    (ob, o), (dqb, dq), (dkb, dk), (dvb, dv) = (_out_like(t, D) for t in (q, q, k, k))
    kw = dict(sm_scale=0.3, window=w[:2], bottom_right=w[2])
    _, lse = B.forward(qd, kd, vd, out=o, **kw)
    B.backward(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    for name, buf in (("O", ob), ("dQ", dqb), ("dK", dkb), ("dV", dvb)):
        assert torch.isnan(buf[..., D:].float()).all(), f"{name}: a column past D was written"
    want = oracle_dense(q, k, v, do, 0.3, *w)
    assert_o_lse(o.float().cpu().numpy(), lse.cpu().numpy(), want["o"], want["lse"], dtype)
    assert_grads([f64(t) for t in (dq, dk, dv)], [want["dq"], want["dk"], want["dv"]],
                 what=f"D={D}")


@pytest.mark.parametrize("D", [13, 56, 67, 120])
def test_packed_head_dims(D):
    B = binding()
    dev = torch.device("cuda")
    sq, sk = [300, 1, 129, 517], [310, 64, 129, 400]
    cu_q, cu_k = synth.cumsum0(sq), synth.cumsum0(sk)
    q, k, v, do = synth.qkv_do((sum(sq), 3, D), (sum(sk), 3, D), seed_of("hdimp", D),
                               torch.bfloat16)
    (qb, qd), (kb, kd), (vb, vd), (dob, dod) = (_padded(t, D) for t in (q, k, v, do))
    (ob, o), (dqb, dq), (dkb, dk), (dvb, dv) = (_out_like(t, D) for t in (q, q, k, k))
    kw = dict(sm_scale=D ** -0.5, window=(CBR, 0), bottom_right=True, cu_seqlens_q=cu_q.to(dev),
              cu_seqlens_k=cu_k.to(dev), max_seqlen_q=max(sq), max_seqlen_k=max(sk),
              lse_layout="TH")
    _, lse = B.forward(qd, kd, vd, out=o, **kw)
    B.backward(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    for name, buf in (("O", ob), ("dQ", dqb), ("dK", dkb), ("dV", dvb)):
        assert torch.isnan(buf[..., D:].float()).all(), f"{name}: a column past D was written"
    want = oracle_packed(q, k, v, do, cu_q, cu_k, D ** -0.5, CBR, 0, True)
    assert_o_lse(o.float().cpu().numpy(), lse.cpu().numpy().T, want["o"], want["lse_ht"],
                 torch.bfloat16)
    assert_grads([f64(t) for t in (dq, dk, dv)], [want["dq"], want["dk"], want["dv"]])


# Without a window, the pairs whose value head dim is a multiple of 16 and whose
# wider head dim is above 64 run on the CTA-pair forward: (64, 128), (128, 64),
# (48, 80), (128, 32), (80, 80), (96, 96), (112, 112), (88, 96), (72, 128).
@pytest.mark.parametrize("D,Dv", [(64, 128), (128, 64), (48, 80), (67, 13), (128, 32), (16, 120),
                                  (80, 80), (96, 96), (112, 112), (88, 96), (72, 128)])
@pytest.mark.parametrize("w", [(INF, INF, False), (CTL, 0, False), (256, 0, True)], ids=str)
def test_value_head_dim_of_its_own(D, Dv, w):
    # Hdim_vo != Hdim_qk (AOTriton 0.15b release notes, "Kernel Bug Fixes"):
    # V, O, dO and dV carry Dv columns, Q, K, dQ and dK carry D.
    B = binding()
    dtype = torch.bfloat16
    q, k, v, do = synth.qkv_do((2, 2, 300, D), (2, 2, 333, D), seed_of("dv", D, Dv, w), dtype,
                               dv=Dv)
    (_, qd), (_, kd), (vb, vd), (_, dod) = (_padded(q, D), _padded(k, D), _padded(v, Dv),
                                            _padded(do, Dv))
    (ob, o), (dqb, dq), (dkb, dk), (dvb, dv) = (_out_like(do, Dv), _out_like(q, D),
                                                _out_like(k, D), _out_like(v, Dv))
    kw = dict(sm_scale=D ** -0.5, window=w[:2], bottom_right=w[2])
    _, lse = B.forward(qd, kd, vd, out=o, **kw)
    B.backward(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    for name, buf, n in (("O", ob, Dv), ("dQ", dqb, D), ("dK", dkb, D), ("dV", dvb, Dv)):
        assert torch.isnan(buf[..., n:].float()).all(), f"{name}: a column past its head dim"
    want = oracle_dense(q, k, v, do, D ** -0.5, *w)
    assert want["o"].shape[-1] == Dv and want["dv"].shape[-1] == Dv
    assert_o_lse(o.float().cpu().numpy(), lse.cpu().numpy(), want["o"], want["lse"], dtype)
    assert_grads([f64(t) for t in (dq, dk, dv)], [want["dq"], want["dk"], want["dv"]],
                 what=f"D={D} Dv={Dv}")

"""Q and K sides addressed independently (AOTriton 0.14b release notes,
"VarlenBits supersedes VarlenType": one VarlenMode per side): every pairing of
dense BHSD, packed 1THD (cumulative lengths) and padded BHSD (per-batch
lengths) on the two sides, checked per sequence against the fp64 oracle on
the sliced tensors.  Padded sides hold NaN in their padding, which must stay
untouched and reach no result."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from attn_cases import CBR, INF, assert_grads, assert_o_lse, binding, f64, seed_of
from oracle import attn_ref as ref
from scaled_dot_product_12_b200 import synth

PAIRS = [("packed", "dense"), ("dense", "packed"), ("padded", "packed"), ("packed", "padded"),
         ("dense", "padded"), ("padded", "dense")]
WINDOWS = [(INF, INF, False), (CBR, 0, True), (256, 0, True), (-64, 128, False)]
H = 2
# per-sequence lengths of a varying side; a dense side uses its maximum for all
LQ, LK = [200, 1, 130], [257, 40, 0]


def _lengths(mode, lens):
    return [max(lens)] * len(lens) if mode == "dense" else list(lens)


def _side(mode, seqs, s_max, dev):
    """Per-sequence [H, L, D] tensors -> (tensor for `mode`, length array or None)."""
    if mode == "packed":
        t = torch.cat([x.transpose(0, 1) for x in seqs], dim=0).contiguous()
        cu = synth.cumsum0([x.shape[1] for x in seqs])
        return t.to(dev), cu.to(dev)
    D = seqs[0].shape[2]
    t = torch.full((len(seqs), H, s_max, D), float("nan"), dtype=seqs[0].dtype)
    for b, x in enumerate(seqs):
        t[b, :, :x.shape[1]] = x
    lens = torch.tensor([x.shape[1] for x in seqs], dtype=torch.int32)
    return t.to(dev), (lens.to(dev) if mode == "padded" else None)


def _rows(mode, t, b, n, cu):
    """Sequence b's first n rows of a side's output as [H, n, ...]."""
    if mode == "packed":
        r0 = int(cu[b])
        return t[r0:r0 + n].transpose(0, 1)
    return t[b, :, :n]


def _run(qmode, kmode, dtype, D, window):
    B = binding()
    wl, wr, br = window
    lq, lk = _lengths(qmode, LQ), _lengths(kmode, LK)
    sq_max, sk_max = max(lq), max(lk)
    seed = seed_of("mixed", qmode, kmode, str(dtype), D, window)
    qs, ks, vs, dos = [], [], [], []
    for b in range(len(lq)):
        q, k, v, do = synth.qkv_do((H, lq[b], D), (H, lk[b], D), seed + b, dtype)
        qs.append(q), ks.append(k), vs.append(v), dos.append(do)
    dev = torch.device("cuda")
    q, aq = _side(qmode, qs, sq_max, dev)
    do, _ = _side(qmode, dos, sq_max, dev)
    k, ak = _side(kmode, ks, sk_max, dev)
    v, _ = _side(kmode, vs, sk_max, dev)
    kw = dict(sm_scale=D ** -0.5, window=(wl, wr), bottom_right=br, lse_layout="HT")
    if qmode == "packed":
        kw.update(cu_seqlens_q=aq, max_seqlen_q=sq_max)
    elif qmode == "padded":
        kw.update(seqlens_q=aq)
    if kmode == "packed":
        kw.update(cu_seqlens_k=ak, max_seqlen_k=sk_max)
    elif kmode == "padded":
        kw.update(seqlens_k=ak)
    nan = float("nan")
    o = torch.full(q.shape, nan, dtype=dtype, device=dev)
    lse_shape = (H, q.shape[0]) if qmode == "packed" else (len(lq), H, sq_max)
    lse = torch.full(lse_shape, nan, dtype=torch.float32, device=dev)
    B.forward(q, k, v, out=o, lse=lse, **kw)
    dq, dk, dv = (torch.full_like(t, nan) for t in (q, k, v))
    B.backward(do, q, k, v, o, lse, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    got = {n: t.float().cpu() for n, t in dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()}
    cu_q = aq.cpu() if qmode == "packed" else None
    cu_k = ak.cpu() if kmode == "packed" else None
    return (qs, ks, vs, dos), got, (lq, lk, cu_q, cu_k), kw["sm_scale"]


@pytest.mark.gpu
@pytest.mark.parametrize("qmode,kmode", PAIRS, ids=lambda x: x)
@pytest.mark.parametrize("window", WINDOWS, ids=str)
@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128)], ids=["bf16-128"])
def test_mixed_addressing_parity(qmode, kmode, window, dtype, D):
    _check(qmode, kmode, window, dtype, D)


@pytest.mark.gpu
@pytest.mark.parametrize("qmode,kmode", [("packed", "padded"), ("padded", "dense")], ids=str)
def test_mixed_addressing_fp16_d64(qmode, kmode):
    _check(qmode, kmode, (256, 0, True), torch.float16, 64)


def _check(qmode, kmode, window, dtype, D):
    wl, wr, br = window
    (qs, ks, vs, dos), got, (lq, lk, cu_q, cu_k), scale = _run(qmode, kmode, dtype, D, window)
    for b in range(len(lq)):
        what = f"seq {b} ({lq[b]}, {lk[b]}) {qmode}/{kmode} w={window}"
        eo, el, eg = [], [], ([], [], [])
        for h in range(H):
            qn, kn, vn, don = f64(qs[b][h]), f64(ks[b][h]), f64(vs[b][h]), f64(dos[b][h])
            o_, l_ = ref.forward(qn, kn, vn, scale, wl, wr, br)
            eo.append(o_)
            el.append(l_)
            for acc, g in zip(eg, ref.backward(qn, kn, vn, don, scale, wl, wr, br)):
                acc.append(g)
        o = _rows(qmode, got["o"], b, lq[b], cu_q)
        lse = (got["lse"][:, int(cu_q[b]):int(cu_q[b]) + lq[b]] if qmode == "packed"
               else got["lse"][b, :, :lq[b]])
        assert_o_lse(o.numpy(), lse.numpy(), np.stack(eo), np.stack(el), dtype, what)
        assert_grads([_rows(qmode, got["dq"], b, lq[b], cu_q).numpy(),
                      _rows(kmode, got["dk"], b, lk[b], cu_k).numpy(),
                      _rows(kmode, got["dv"], b, lk[b], cu_k).numpy()],
                     [np.stack(g) for g in eg], what)
        if qmode == "padded":
            for name in ("o", "lse", "dq"):
                assert torch.isnan(got[name][b, :, lq[b]:]).all(), f"{what}: {name} padding"
        if kmode == "padded":
            for name in ("dk", "dv"):
                assert torch.isnan(got[name][b, :, lk[b]:]).all(), f"{what}: {name} padding"

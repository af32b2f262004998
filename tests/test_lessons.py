"""One GPU test per kernel lesson the release notes record.

* 0.14b notes, "Kernel Bug Fixes": an early-exit LSE write ran past a
  sequence under the stacked varlen layout -> canaries after the packed rows
  and around the head dimension stay untouched.
* the same lesson for a cumulative-lengths array that runs past the packed
  tensors (a caller's error): the sequences are clamped to the tensors, rows
  past them (canaries) stay untouched and the rest matches the oracle on the
  clamped lengths, forward and backward.
* 0.14b notes, "Kernel Bug Fixes": a backward addressed dO with O's strides
  -> dO with a layout of its own gives the same gradients.
* 0.15b notes, "Kernel Bug Fixes": the early-exit zero store was bounded by the
  padded head dim, not the real one -> a D = 48 output inside a 64-wide buffer
  keeps its last 16 columns.
* 0.15b notes, "Kernel Bug Fixes": truncating P to bf16 biased O low -> with
  V = 1, O averages to 1.
* 0.15b notes, "Known Problems": hardware that flushes fp16 subnormals fails
  window-(0, 0) varlen tests -> O is V exactly, subnormals included.
* 0.15b notes, "Minor Changes": test_null_logsumexp -> a NULL LSE pointer is
  accepted and O is unchanged.
* 0.14b notes, "Minor Changes": test_bottom_right_fully_masked_rows -> rows that
  see no key under a bottom-right window give O = 0, LSE = -inf, dQ = 0.
"""

import numpy as np
import pytest
import torch

from attn_cases import (CBR, CTL, INF, assert_grads, assert_o_lse, binding, dense_inputs, f64,
                        oracle_dense, packed_inputs, run_packed, oracle_packed, seed_of)
from oracle import attn_ref as ref
from scaled_dot_product_12_b200 import synth

pytestmark = pytest.mark.gpu
NAN16 = float("nan")


@pytest.mark.parametrize("lse_layout", ["HT", "TH"])
@pytest.mark.parametrize("w", [(CTL, 0, False), (CBR, 0, True), (256, 0, True), (-64, 128, False)],
                         ids=str)
def test_packed_rows_past_the_last_sequence_stay_untouched(lse_layout, w):
    B = binding()
    dev = torch.device("cuda")
    sq, sk = [130, 5, 257], [100, 300, 257]
    H, D, pad = 2, 64, 300
    q, k, v, do, cu_q, cu_k = packed_inputs(sq, sk, H, D, torch.bfloat16, 11)
    tq = sum(sq)
    # outputs live inside larger buffers filled with NaN canaries
    o_buf = torch.full((tq + pad, H, D), NAN16, dtype=torch.bfloat16, device=dev)
    # LSE is contiguous [T, H] or [H, T]; canaries follow it in one flat buffer
    lse_buf = torch.full((H * tq + pad,), float("nan"), device=dev)
    lse_c = lse_buf[:H * tq].view((tq, H) if lse_layout == "TH" else (H, tq))
    o = o_buf[:tq]
    B.forward(q.to(dev), k.to(dev), v.to(dev), sm_scale=0.125, window=w[:2], bottom_right=w[2],
              cu_seqlens_q=cu_q.to(dev), cu_seqlens_k=cu_k.to(dev), max_seqlen_q=max(sq),
              max_seqlen_k=max(sk), lse_layout=lse_layout, out=o, lse=lse_c)
    torch.cuda.synchronize()
    assert torch.isnan(o_buf[tq:].float()).all()
    assert torch.isnan(lse_buf[H * tq:]).all()
    want = ref.forward_packed(f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(), 0.125, *w)
    got_lse = lse_c.cpu().numpy()
    got_lse = got_lse.T if lse_layout == "TH" else got_lse
    assert_o_lse(o.float().cpu().numpy(), got_lse, want[0], want[1], torch.bfloat16)


@pytest.mark.parametrize("w", [(INF, INF, False), (CTL, 0, False), (256, 0, True), (-64, 128, True)],
                         ids=str)
def test_cumulative_lengths_past_the_tensors_are_clamped(w):
    B = binding()
    dev = torch.device("cuda")
    sq, sk = [130, 5, 257], [100, 300, 257]
    H, D, pad = 2, 64, 300
    q, k, v, do, cu_q, cu_k = packed_inputs(sq, sk, H, D, torch.bfloat16, 12)
    tq, tk = sum(sq), sum(sk)
    # the last entries claim 150 query rows and 200 key rows that do not exist
    bad_q = cu_q.clone()
    bad_q[-1] += 150
    bad_k = cu_k.clone()
    bad_k[-1] += 200
    kw = dict(sm_scale=0.125, window=w[:2], bottom_right=w[2], cu_seqlens_q=bad_q.to(dev),
              cu_seqlens_k=bad_k.to(dev), max_seqlen_q=257 + 150, max_seqlen_k=257 + 200,
              lse_layout="TH")

    def canary(rows):
        buf = torch.full((rows + pad, H, D), NAN16, dtype=torch.bfloat16, device=dev)
        return buf, buf[:rows]
    o_buf, o = canary(tq)
    dq_buf, dq = canary(tq)
    dk_buf, dk = canary(tk)
    dv_buf, dv = canary(tk)
    lse_buf = torch.full((H * tq + pad,), float("nan"), device=dev)
    lse = lse_buf[:H * tq].view(tq, H)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    B.forward(qd, kd, vd, out=o, lse=lse, **kw)
    B.backward(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert B.device_status(dev) == 0
    for buf, rows in ((o_buf, tq), (dq_buf, tq), (dk_buf, tk), (dv_buf, tk)):
        assert torch.isnan(buf[rows:].float()).all(), "a write ran past the tensor"
    assert torch.isnan(lse_buf[H * tq:]).all()
    want = oracle_packed(q, k, v, do, cu_q, cu_k, 0.125, *w)
    assert_o_lse(o.float().cpu().numpy(), lse.cpu().numpy().T, want["o"], want["lse_ht"],
                 torch.bfloat16)
    assert_grads([f64(t) for t in (dq, dk, dv)], [want["dq"], want["dk"], want["dv"]])


@pytest.mark.parametrize("w", [(INF, INF, False), (0, -1, False), (CBR, 0, True)], ids=str)
def test_head_dim_padding_columns_untouched(w):
    # D = 48 inside a 64-wide row: columns 48..63 are never written, in the
    # normal epilogue and in the fully-masked early exit ((0, -1) masks all).
    B = binding()
    dev = torch.device("cuda")
    q, k, v, do = dense_inputs(1, 2, 300, 200, 48, torch.float16, 21)
    o_buf = torch.full((1, 2, 300, 64), NAN16, dtype=torch.float16, device=dev)
    o = o_buf[..., :48]
    B.forward(q.to(dev), k.to(dev), v.to(dev), sm_scale=0.2, window=w[:2], bottom_right=w[2], out=o)
    torch.cuda.synchronize()
    assert torch.isnan(o_buf[..., 48:].float()).all()
    assert not torch.isnan(o.float()).any()
    want = ref.forward_dense(f64(q), f64(k), f64(v), 0.2, *w)[0]
    assert np.abs(o.float().cpu().numpy() - want).max() <= 1e-2


def test_dout_with_its_own_strides():
    B = binding()
    dev = torch.device("cuda")
    q, k, v, do = dense_inputs(2, 3, 300, 300, 128, torch.bfloat16, 31)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o, lse = B.forward(qd, kd, vd, sm_scale=0.1, window=(CTL, 0))
    do_c = do.to(dev)
    # the same values stored as [B, S, H, D] (strides differ from O's BHSD ones)
    do_t = do.permute(0, 2, 1, 3).contiguous().to(dev).permute(0, 2, 1, 3)
    assert do_t.stride() != o.stride()
    a = B.backward(do_c, qd, kd, vd, o, lse, sm_scale=0.1, window=(CTL, 0))
    b = B.backward(do_t, qd, kd, vd, o, lse, sm_scale=0.1, window=(CTL, 0))
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])  # dK, dV: same arithmetic
    diff = (a[0].float() - b[0].float()).norm() / a[0].float().norm()
    assert diff <= 1e-3  # dQ: fp32 reduction order may differ
    want = oracle_dense(q, k, v, do, 0.1, CTL, 0, False)
    assert_grads([t.float().cpu().numpy() for t in b[:3]], [want["dq"], want["dk"], want["dv"]])


def test_p_is_rounded_to_nearest_not_truncated():
    # V = 1: O_i = sum_j round(P_ij) / sum_j P_ij.  Round-to-nearest keeps the
    # mean at 1; truncating P to bf16 would pull it to about 1 - 2^-9.
    B = binding()
    dev = torch.device("cuda")
    q, k, _, _ = dense_inputs(1, 8, 1024, 1024, 128, torch.bfloat16, 41)
    v = torch.ones(1, 8, 1024, 128, dtype=torch.bfloat16)
    o, _ = B.forward(q.to(dev), k.to(dev), v.to(dev), sm_scale=128 ** -0.5)
    torch.cuda.synchronize()
    mean = o.float().mean().item()
    assert abs(mean - 1.0) < 5e-4, mean


@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("br", [False, True])
def test_window_zero_zero_keeps_fp16_subnormals(packed, br):
    B = binding()
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(51)
    H, D = 2, 64
    sq, sk = ([200, 77, 129], [230, 77, 100]) if packed else ([300], [330])
    tq, tk = sum(sq), sum(sk)
    q = torch.randn(tq, H, D, generator=g).half()
    k = torch.randn(tk, H, D, generator=g).half()
    v = (torch.randint(1, 1000, (tk, H, D), generator=g).float() * 2.0**-24).half()
    assert (v.float().abs() < 2.0**-14).all()  # subnormal fp16 values
    kw = dict(sm_scale=0.5, window=(0, 0), bottom_right=br)
    if packed:
        cu_q, cu_k = synth.cumsum0(sq), synth.cumsum0(sk)
        o, lse = B.forward(q.to(dev), k.to(dev), v.to(dev), cu_seqlens_q=cu_q.to(dev),
                           cu_seqlens_k=cu_k.to(dev), max_seqlen_q=max(sq), max_seqlen_k=max(sk),
                           **kw)
        o = o.cpu()
    else:
        cu_q, cu_k = synth.cumsum0(sq), synth.cumsum0(sk)
        o, lse = B.forward(q.permute(1, 0, 2)[None].to(dev), k.permute(1, 0, 2)[None].to(dev),
                           v.permute(1, 0, 2)[None].to(dev), **kw)
        o = o[0].permute(1, 0, 2).cpu()
    torch.cuda.synchronize()
    for s in range(len(sq)):
        d = sk[s] - sq[s] if br else 0
        for i in range(sq[s]):
            j = i + d
            row = o[cu_q[s] + i]
            if 0 <= j < sk[s]:
                assert torch.equal(row, v[cu_k[s] + j]), (s, i)
            else:
                assert (row == 0).all()


@pytest.mark.parametrize("wl,wr,br", [(256, 0, True), (INF, INF, False)])  # the latter: CTA pairs
def test_null_logsumexp_pointer(wl, wr, br):
    B = binding()
    dev = torch.device("cuda")
    q, k, v, _ = dense_inputs(2, 2, 300, 400, 128, torch.bfloat16, 61)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o1, lse = B.forward(qd, kd, vd, sm_scale=0.09, window=(wl, wr), bottom_right=br)
    o2, none = B.forward(qd, kd, vd, sm_scale=0.09, window=(wl, wr), bottom_right=br,
                         return_lse=False)
    torch.cuda.synchronize()
    assert none is None and torch.equal(o1, o2)


@pytest.mark.parametrize("packed", [False, True])
def test_bottom_right_fully_masked_rows(packed):
    # Sq > Sk with the bottom-right causal sentinel: rows i < Sq - Sk see nothing.
    if packed:
        sq, sk = [300, 130], [100, 129]
        q, k, v, do, cu_q, cu_k = packed_inputs(sq, sk, 2, 128, torch.bfloat16, 71)
        got = run_packed(q, k, v, do, cu_q, cu_k, 0.1, CBR, 0, False)
        want = oracle_packed(q, k, v, do, cu_q, cu_k, 0.1, CBR, 0, False)
        lse, want_lse = got["lse"].numpy().T, want["lse_ht"]
    else:
        from attn_cases import run_dense
        q, k, v, do = dense_inputs(1, 2, 300, 100, 128, torch.bfloat16, 72)
        got = run_dense(q, k, v, do, 0.1, CBR, 0, True)
        want = oracle_dense(q, k, v, do, 0.1, CBR, 0, True)
        lse, want_lse = got["lse"].numpy(), want["lse"]
    empty = np.isneginf(want_lse)
    assert empty.any()
    assert_o_lse(got["o"].float().numpy(), lse, want["o"], want_lse, torch.bfloat16)
    o = got["o"].float().numpy()
    dq = got["dq"].float().numpy()
    if packed:
        rows = np.nonzero(empty.any(0))[0]
        assert np.all(o[rows] == 0) and np.all(dq[rows] == 0)
    else:
        assert np.all(o[..., empty[0, 0], :] == 0) and np.all(dq[..., empty[0, 0], :] == 0)
    assert_grads([got[n].float().numpy() for n in ("dq", "dk", "dv")],
                 [want[n] for n in ("dq", "dk", "dv")])


@pytest.mark.parametrize("shape", [(512, 16, 384, 64), (4, 16, 384, 128), (2, 8, 2000, 128)])
def test_repeated_runs_never_time_out(shape):
    # Each query tile's softmax warps can run a step ahead of the MMA thread;
    # a barrier reused across steps once let a fast group lap its consumer and
    # stall it until the bounded wait gave up.  Repeat the shapes where that
    # showed up and require a clean device status after every run.
    B = binding()
    dev = torch.device("cuda")
    Bb, H, S, D = shape
    q, k, v, do = (t.to(dev) for t in dense_inputs(Bb, H, S, S, D, torch.bfloat16, 91))
    o, lse = B.forward(q, k, v)
    for _ in range(10):
        B.forward(q, k, v, out=o, lse=lse)
        B.backward(do, q, k, v, o, lse)
        torch.cuda.synchronize()
        assert B.device_status(dev) == 0

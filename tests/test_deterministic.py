"""Deterministic backward (ATTN_BWD_DETERMINISTIC): the dQ contributions of
the key tiles are added in key-tile order, so repeated calls give bit-equal
dQ (the AOTriton 0.15b release notes, "Known Problems", record run-to-run
differences of the backward, "even in deterministic mode").  Without the
flag the contributions are added in whatever order the CTAs reach them.
Every deterministic result also matches the fp64 oracle."""

import numpy as np
import pytest
import torch

from attn_cases import (CBR, CTL, INF, assert_grads, binding, dense_inputs, f64, oracle_dense,
                        oracle_packed, packed_inputs, run_packed)

pytestmark = pytest.mark.gpu


def _dense(D, w, B_=2, H=3, S=1100, seed=5):
    B = binding()
    dev = torch.device("cuda")
    host = dense_inputs(B_, H, S, S, D, torch.bfloat16, seed)
    q, k, v, do = (t.to(dev) for t in host)
    kw = dict(sm_scale=D ** -0.5, window=w[:2], bottom_right=w[2])
    o, lse = B.forward(q, k, v, **kw)
    return B, host, (q, k, v, do, o, lse), kw


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("w", [(INF, INF, False), (CTL, 0, False), (256, 0, True),
                               (-64, 128, False)], ids=str)
def test_deterministic_dq_is_bit_equal_across_runs(D, w):
    B, host, (q, k, v, do, o, lse), kw = _dense(D, w)
    runs = []
    for _ in range(4):
        dq, dk, dv, _ = B.backward(do, q, k, v, o, lse, deterministic=True, **kw)
        torch.cuda.synchronize()
        runs.append((dq.cpu(), dk.cpu(), dv.cpu()))
    assert B.device_status() == 0
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)
    want = oracle_dense(*host, kw["sm_scale"], *w)
    assert_grads([f64(t) for t in runs[0]], [want["dq"], want["dk"], want["dv"]])
    # the default mode agrees to within fp32 reduction order
    dq, dk, dv, _ = B.backward(do, q, k, v, o, lse, **kw)
    torch.cuda.synchronize()
    assert torch.equal(dk.cpu(), runs[0][1]) and torch.equal(dv.cpu(), runs[0][2])
    diff = (dq.float().cpu() - runs[0][0].float()).norm() / runs[0][0].float().norm()
    assert diff <= 1e-3


def test_deterministic_packed_varlen():
    B = binding()
    dev = torch.device("cuda")
    sq, sk = [300, 1, 700, 129, 0, 517], [310, 64, 650, 129, 33, 900]
    q, k, v, do, cu_q, cu_k = packed_inputs(sq, sk, 4, 128, torch.bfloat16, 9)
    kw = dict(sm_scale=128 ** -0.5, window=(CBR, 0), bottom_right=True,
              cu_seqlens_q=cu_q.to(dev), cu_seqlens_k=cu_k.to(dev), max_seqlen_q=max(sq),
              max_seqlen_k=max(sk), lse_layout="TH")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o, lse = B.forward(qd, kd, vd, **kw)
    first = None
    for _ in range(3):
        dq, dk, dv, _ = B.backward(dod, qd, kd, vd, o, lse, deterministic=True, **kw)
        torch.cuda.synchronize()
        cur = (dq.cpu(), dk.cpu(), dv.cpu())
        if first is None:
            first = cur
        else:
            assert all(torch.equal(a, b) for a, b in zip(first, cur))
    assert B.device_status() == 0
    want = oracle_packed(q, k, v, do, cu_q, cu_k, 128 ** -0.5, CBR, 0, True)
    assert_grads([f64(t) for t in first], [want["dq"], want["dk"], want["dv"]])


def test_deterministic_workspace_is_larger_by_the_counters():
    import ctypes
    B = binding()
    q = torch.empty((2, 3, 100, 64), dtype=torch.bfloat16)
    lse = torch.empty((2, 3, 100), dtype=torch.float32)
    pr = B.Problem(q, q, 0.1, (CTL, 0), False, None, None, None, None, "HT")
    p = B.bwd_params(q, q, q, q, q, lse, pr, q, q, q)
    base = B.workspace_bytes(p)
    p.flags = B.BWD_DETERMINISTIC
    assert B.workspace_bytes(p) == base + 2 * 3 * 100 * 16

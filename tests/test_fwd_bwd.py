"""GPU parity: the CUDA forward and backward (through the C ABI) against the
fp64 oracle on the same seeded inputs, element by element, at sizes that span
several 128-row tiles with ragged tails."""

import numpy as np
import pytest
import torch

from attn_cases import (CBR, CTL, INF, assert_grads, assert_o_lse, dense_inputs, oracle_dense,
                        oracle_packed, packed_inputs, run_dense, run_packed, seed_of)

pytestmark = pytest.mark.gpu

WINDOWS = [
    (INF, INF, False), (CTL, 0, False), (CTL, 0, True), (CBR, 0, False), (CBR, 0, True),
    (INF, 0, True), (256, 0, False), (256, 0, True), (-64, 128, False), (-64, 128, True),
    (100, -37, False), (0, 0, True), (3, -9, False),
]
SHAPES = [(200, 333), (333, 200), (256, 256), (1, 1), (129, 700)]


def _dense_case(dtype, D, sq, sk, w, scale=None, B=2, H=2, backward=True, lse_layout="HT"):
    seed = seed_of("dense", str(dtype), D, sq, sk, w, scale, B, H)
    q, k, v, do = dense_inputs(B, H, sq, sk, D, dtype, seed)
    scale = D ** -0.5 if scale is None else scale
    got = run_dense(q, k, v, do, scale, *w, lse_layout=lse_layout, backward=backward)
    want = oracle_dense(q, k, v, do, scale, *w, backward=backward)
    lse = got["lse"].numpy()
    if lse_layout == "TH":
        lse = np.swapaxes(lse, 1, 2)
    assert_o_lse(got["o"].float().numpy(), lse, want["o"], want["lse"], dtype,
                 what=f"D={D} {sq}x{sk} w={w}")
    if backward:
        assert_grads([got[n].float().numpy() for n in ("dq", "dk", "dv")],
                     [want[n] for n in ("dq", "dk", "dv")], what=f"D={D} {sq}x{sk} w={w}")


@pytest.mark.parametrize("w", WINDOWS, ids=str)
@pytest.mark.parametrize("sq,sk", SHAPES, ids=str)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16], ids=["bf16", "fp16"])
@pytest.mark.parametrize("D", [64, 128])
def test_dense_parity(D, dtype, sq, sk, w):
    _dense_case(dtype, D, sq, sk, w)


@pytest.mark.parametrize("D", [16, 32, 48, 80, 96, 112])
@pytest.mark.parametrize("w", [(INF, INF, False), (CTL, 0, False), (-64, 128, True)], ids=str)
def test_dense_other_head_dims(D, w):
    _dense_case(torch.bfloat16, D, 300, 271, w)


@pytest.mark.parametrize("scale", [0.0, -0.2, -1.0, 0.9])
@pytest.mark.parametrize("w", [(INF, INF, False), (CBR, 0, True), (256, 0, True)], ids=str)
def test_any_scale_sign(scale, w):
    # sm_scale <= 0 must work (0.15b release notes, "Kernel Bug Fixes": a fused
    # backward returned NaN or zero gradients for sm_scale <= 0).
    _dense_case(torch.bfloat16, 64, 257, 300, w, scale=scale)


def test_lse_th_dense():
    _dense_case(torch.bfloat16, 128, 300, 300, (CTL, 0, False), lse_layout="TH", H=3)


def test_tiny_causal_config():
    # fp16, B1 H2 S128 D64, causal top-left (window (INF, 0)), dense, LSE HT.
    _dense_case(torch.float16, 64, 128, 128, (INF, 0, False), B=1, H=2)


def test_many_heads_and_batches():
    _dense_case(torch.bfloat16, 64, 384, 384, (INF, INF, False), B=5, H=7)


@pytest.mark.parametrize("w", WINDOWS, ids=str)
@pytest.mark.parametrize("D", [128, 64, 48, 80])
def test_packed_parity(D, w):
    # Ragged sequences, one empty query sequence, seqlen_k >= or < seqlen_q.
    sq = [1, 300, 0, 129, 77, 513]
    sk = [5, 300, 40, 100, 200, 600]
    seed = seed_of("packed", D, w)
    q, k, v, do, cu_q, cu_k = packed_inputs(sq, sk, 3, D, torch.bfloat16, seed)
    scale = D ** -0.5
    got = run_packed(q, k, v, do, cu_q, cu_k, scale, *w, lse_layout="TH")
    want = oracle_packed(q, k, v, do, cu_q, cu_k, scale, *w)
    assert_o_lse(got["o"].float().numpy(), got["lse"].numpy().T, want["o"], want["lse_ht"],
                 torch.bfloat16, what=f"packed D={D} w={w}")
    assert_grads([got[n].float().numpy() for n in ("dq", "dk", "dv")],
                 [want[n] for n in ("dq", "dk", "dv")], what=f"packed D={D} w={w}")


def test_packed_lse_ht():
    sq, sk = [130, 3, 260], [200, 3, 100]
    q, k, v, do, cu_q, cu_k = packed_inputs(sq, sk, 2, 128, torch.float16, 77)
    got = run_packed(q, k, v, do, cu_q, cu_k, 0.1, 256, 0, True, lse_layout="HT")
    want = oracle_packed(q, k, v, do, cu_q, cu_k, 0.1, 256, 0, True)
    assert_o_lse(got["o"].float().numpy(), got["lse"].numpy(), want["o"], want["lse_ht"],
                 torch.float16)
    assert_grads([got[n].float().numpy() for n in ("dq", "dk", "dv")],
                 [want[n] for n in ("dq", "dk", "dv")])


def test_forward_is_deterministic():
    q, k, v, do = dense_inputs(2, 3, 700, 650, 128, torch.bfloat16, 5)
    a = run_dense(q, k, v, do, 0.1, CTL, 0, False, backward=False)
    b = run_dense(q, k, v, do, 0.1, CTL, 0, False, backward=False)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])

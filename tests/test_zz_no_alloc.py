"""attn_bwd_static_workspace: the backward for callers that cannot allocate
device memory (a host that owns all device memory and gives this library no
allocator, or a latency-critical path that cannot afford cudaMalloc's implicit
synchronisation).  It takes its scratch memory from an array compiled into the
library instead of a caller-provided workspace.

Checked here through the C ABI, on a dense causal problem and on a packed
variable-length one (LSE in TH layout, whose scratch is sized by the packed
token count): two calls in a row give the dK and dV of attn_bwd with its own
workspace bit for bit (each key tile's gradients are computed by one CTA in a
fixed order) and its dQ to within fp32 reduction order (the dQ tiles are
added in whatever order the CTAs finish); the first result also matches the
fp64 oracle within the parity tolerance; a problem too large for the array is
refused with cudaErrorMemoryAllocation.  This file is named so that pytest
collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from attn_cases import (CTL, assert_grads, dense_inputs, f64, oracle_dense, oracle_packed,
                        packed_inputs)

pytestmark = pytest.mark.gpu


def _dense_setup(B_, H, S, D, seed):
    from scaled_dot_product_12_b200 import binding as Bd
    dev = torch.device("cuda")
    host = dense_inputs(B_, H, S, S, D, torch.bfloat16, seed)
    q, k, v, do = (t.to(dev) for t in host)
    scale = D ** -0.5
    o, lse = Bd.forward(q, k, v, sm_scale=scale, window=(CTL, 0))
    pr = Bd.Problem(q, k, scale, (CTL, 0), False, None, None, None, None, "HT")
    want = oracle_dense(*host, scale, CTL, 0, False)
    return Bd, dev, (q, k, v, do, o, lse), pr, want


def _packed_setup(seed):
    from scaled_dot_product_12_b200 import binding as Bd
    dev = torch.device("cuda")
    sq, sk = [300, 1, 129, 517], [310, 64, 129, 400]
    host = packed_inputs(sq, sk, 3, 128, torch.bfloat16, seed)
    q, k, v, do = (t.to(dev) for t in host[:4])
    cu_q, cu_k = host[4].to(dev), host[5].to(dev)
    w = (256, 0)
    scale = 128 ** -0.5
    kw = dict(cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, max_seqlen_q=max(sq), max_seqlen_k=max(sk),
              lse_layout="TH")
    o, lse = Bd.forward(q, k, v, sm_scale=scale, window=w, bottom_right=True, **kw)
    pr = Bd.Problem(q, k, scale, w, True, cu_q, cu_k, max(sq), max(sk), "TH")
    want = oracle_packed(*host, scale, *w, True)
    return Bd, dev, (q, k, v, do, o, lse), pr, want


def _grads(Bd, tensors, pr, entry, stream):
    q, k, v, do, o, lse = tensors
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    p = Bd.bwd_params(do, q, k, v, o, lse, pr, dq, dk, dv)
    if entry == "attn_bwd":
        ws = torch.empty(Bd.workspace_bytes(p), dtype=torch.uint8, device=q.device)
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    code = getattr(Bd.lib(), entry)(ctypes.byref(p), stream.cuda_stream)
    assert code == 0, f"{entry} returned {code}"
    torch.cuda.synchronize()
    return dq.cpu(), dk.cpu(), dv.cpu()


@pytest.mark.parametrize("case", ["dense_causal", "packed_window_TH"])
def test_static_workspace_matches_attn_bwd_twice_in_a_row(case):
    if case == "dense_causal":
        Bd, dev, tensors, pr, want = _dense_setup(2, 3, 333, 64, seed=2024)
    else:
        Bd, dev, tensors, pr, want = _packed_setup(seed=2025)
    stream = torch.cuda.current_stream(dev)
    ref_dq, ref_dk, ref_dv = _grads(Bd, tensors, pr, "attn_bwd", stream)
    for call in range(2):  # the second call reuses the array the first one left behind
        dq, dk, dv = _grads(Bd, tensors, pr, "attn_bwd_static_workspace", stream)
        assert torch.equal(dk, ref_dk) and torch.equal(dv, ref_dv), f"call {call}: dK / dV"
        diff = (dq.float() - ref_dq.float()).norm() / ref_dq.float().norm()
        assert diff <= 1e-3, f"call {call}: dQ differs by {diff}"
        if call == 0:
            assert_grads([f64(t) for t in (dq, dk, dv)], [want["dq"], want["dk"], want["dv"]],
                         what=case)
    assert Bd.device_status(dev) == 0


def test_static_workspace_refuses_problems_larger_than_the_array():
    from scaled_dot_product_12_b200 import binding as Bd
    dev = torch.device("cuda")
    # 1 x 64 heads x 8192 rows x (128 + 1) fp32 values is about 270 MB > 64 MiB.
    q = torch.empty((1, 64, 8192, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, 64, 8192), dtype=torch.float32, device=dev)
    pr = Bd.Problem(q, q, 0.1, (CTL, 0), False, None, None, None, None, "HT")
    p = Bd.bwd_params(q, q, q, q, q, lse, pr, q, q, q)
    assert Bd.workspace_bytes(p) > Bd.STATIC_WORKSPACE_BYTES
    code = Bd.lib().attn_bwd_static_workspace(ctypes.byref(p), None)
    assert code == Bd.ERROR_MEMORY_ALLOCATION

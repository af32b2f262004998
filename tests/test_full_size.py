"""Parity at the full workload sizes, in the launch configuration bench.py times
(the same tensors, the same two C-ABI calls), on seeded samples the oracle can
afford: whole heads of dense workloads, and whole heads of every sequence of
the packed Generalized-SWA workload.  The count probe (sm_scale = 0) checks
the mask of every packed case exactly."""

import numpy as np
import pytest
import torch

from attn_cases import assert_grads, assert_o_lse, binding, f64
from oracle import attn_ref as ref
from scaled_dot_product_12_b200 import synth

pytestmark = pytest.mark.gpu


def _sample_heads(w, n, seed):
    g = np.random.default_rng(seed)
    pairs = [(int(g.integers(w.B)), int(g.integers(w.H))) for _ in range(n)]
    return sorted(set(pairs))


@pytest.mark.parametrize("name", ["tiny_causal", "bert_large", "roberta_large", "gpt2",
                                  "ltx_6630", "ltx_15300", "long_8192"])
def test_dense_workload_sampled_heads(name):
    B = binding()
    w = synth.WORKLOADS[name]
    dtype = synth.DTYPES[w.dtype]
    dev = torch.device("cuda")
    q, k, v, do = synth.qkv_do((w.B, w.H, w.Sq, w.D), (w.B, w.H, w.Sk, w.D), w.seed, dtype)
    scale = w.D ** -0.5
    win = (w.window_left, w.window_right)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = B.forward(qd, kd, vd, sm_scale=scale, window=win, bottom_right=w.bottom_right)
    dq, dk, dv, _ = B.backward(dod, qd, kd, vd, o, lse, sm_scale=scale, window=win,
                               bottom_right=w.bottom_right)
    torch.cuda.synchronize()
    assert B.device_status(dev) == 0
    heads = _sample_heads(w, 2 if w.B * w.H > 2 else w.B * w.H, w.seed)
    for b, h in heads:
        eo, el = ref.forward(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), scale, *win, w.bottom_right)
        eg = ref.backward(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), f64(do[b, h]), scale, *win,
                          w.bottom_right)
        assert_o_lse(o[b, h].float().cpu().numpy(), lse[b, h].cpu().numpy(), eo, el, dtype,
                     what=f"{name} head {(b, h)}")
        assert_grads([t[b, h].float().cpu().numpy() for t in (dq, dk, dv)], eg,
                     what=f"{name} head {(b, h)}")


_SQ, _SK = synth.varlen_seqlens(synth.VARLEN_SEQLEN_SEED)
_CASES = synth.varlen_cases()


def _packed_setup(D, seed, dev):
    H = 16
    cu_q, cu_k = synth.cumsum0(_SQ), synth.cumsum0(_SK)
    q, k, v, do = synth.qkv_do((int(cu_q[-1]), H, D), (int(cu_k[-1]), H, D), seed, torch.bfloat16)
    kw = dict(cu_seqlens_q=cu_q.to(dev), cu_seqlens_k=cu_k.to(dev), max_seqlen_q=max(_SQ),
              max_seqlen_k=max(_SK), lse_layout="TH")
    return q, k, v, do, cu_q, cu_k, kw


@pytest.mark.parametrize("case", _CASES, ids=[c[0] for c in _CASES])
def test_packed_workload_sampled_heads(case):
    name, D, wl, wr, br, seed = case
    B = binding()
    dev = torch.device("cuda")
    q, k, v, do, cu_q, cu_k, kw = _packed_setup(D, seed, dev)
    scale = D ** -0.5
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o, lse = B.forward(qd, kd, vd, sm_scale=scale, window=(wl, wr), bottom_right=br, **kw)
    dq, dk, dv, _ = B.backward(do.to(dev), qd, kd, vd, o, lse, sm_scale=scale, window=(wl, wr),
                               bottom_right=br, **kw)
    torch.cuda.synchronize()
    assert B.device_status(dev) == 0
    g = np.random.default_rng(seed)
    heads = sorted(set(int(x) for x in g.integers(0, 16, 2 if D == 128 else 1)))
    o, lse, dq, dk, dv = (t.float().cpu() for t in (o, lse, dq, dk, dv))
    for h in heads:
        sl = (slice(None), slice(h, h + 1))
        eo, el = ref.forward_packed(f64(q[sl]), f64(k[sl]), f64(v[sl]), cu_q.numpy(), cu_k.numpy(),
                                    scale, wl, wr, br)
        eg = ref.backward_packed(f64(q[sl]), f64(k[sl]), f64(v[sl]), f64(do[sl]), cu_q.numpy(),
                                 cu_k.numpy(), scale, wl, wr, br)
        assert_o_lse(o[sl].numpy(), lse[:, h:h + 1].numpy().T, eo, el, torch.bfloat16,
                     what=f"{name} head {h}")
        assert_grads([t[sl].numpy() for t in (dq, dk, dv)], eg, what=f"{name} head {h}")


@pytest.mark.parametrize("case", [c for c in _CASES if c[1] == 128], ids=lambda c: c[0])
def test_packed_workload_count_probe(case):
    name, D, wl, wr, br, seed = case
    B = binding()
    dev = torch.device("cuda")
    q, k, v, do, cu_q, cu_k, kw = _packed_setup(D, seed, dev)
    _, lse = B.forward(q.to(dev), k.to(dev), v.to(dev), sm_scale=0.0, window=(wl, wr),
                       bottom_right=br, **kw)
    torch.cuda.synchronize()
    lse = lse.cpu().numpy().astype(np.float64)  # [T, H]
    for s in range(len(_SQ)):
        _, _, cnt = ref.row_extent(_SQ[s], _SK[s], wl, wr, br)
        rows = lse[int(cu_q[s]):int(cu_q[s + 1])]
        empty = cnt == 0
        assert np.array_equal(np.isneginf(rows), np.broadcast_to(empty[:, None], rows.shape))
        got = np.rint(np.exp(rows[~empty]))
        assert np.array_equal(got, np.broadcast_to(cnt[~empty, None], got.shape).astype(float))


@pytest.mark.parametrize("name,shared", [("bert_large", False), ("gpt2", False),
                                         ("ltx_6630", True)])
def test_dense_workload_with_bias_sampled_heads(name, shared):
    """The additive bias and its gradient at full size: a bias per (batch,
    head) for the D = 64 shapes (staged by TMA in both kernels), one bias
    shared by every batch and head at LTX 6630 (D = 128: staged in the
    forward, loaded per thread in the backward)."""
    B = binding()
    w = synth.WORKLOADS[name]
    dtype = synth.DTYPES[w.dtype]
    dev = torch.device("cuda")
    q, k, v, do = synth.qkv_do((w.B, w.H, w.Sq, w.D), (w.B, w.H, w.Sk, w.D), w.seed, dtype)
    pitch = (w.Sk + 7) // 8 * 8  # 16-byte rows
    shape = (1, 1) if shared else (w.B, w.H)
    host_bias = synth.bias(shape + (w.Sq, w.Sk), w.seed + 101, dtype, std=1.0)
    bias_buf = torch.zeros(shape + (w.Sq, pitch), dtype=dtype, device=dev)
    bias_buf[..., :w.Sk] = host_bias.to(dev)
    bias = bias_buf[..., :w.Sk].expand(w.B, w.H, w.Sq, w.Sk)
    dbias = torch.empty((w.B, w.H, w.Sq, pitch), dtype=dtype, device=dev)[..., :w.Sk]
    scale = w.D ** -0.5
    win = (w.window_left, w.window_right)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    kw = dict(sm_scale=scale, window=win, bottom_right=w.bottom_right, bias=bias)
    o, lse = B.forward(qd, kd, vd, **kw)
    dq, dk, dv, _ = B.backward(dod, qd, kd, vd, o, lse, dbias=dbias, **kw)
    torch.cuda.synchronize()
    assert B.device_status(dev) == 0
    for b, h in _sample_heads(w, 1, w.seed + 7):
        bb = f64(host_bias[0, 0] if shared else host_bias[b, h])
        eo, el = ref.forward(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), scale, *win, w.bottom_right,
                             bias=bb)
        eg = ref.backward(f64(q[b, h]), f64(k[b, h]), f64(v[b, h]), f64(do[b, h]), scale, *win,
                          w.bottom_right, bias=bb)
        what = f"{name} bias head {(b, h)}"
        assert_o_lse(o[b, h].float().cpu().numpy(), lse[b, h].cpu().numpy(), eo, el, dtype, what=what)
        assert_grads([t[b, h].float().cpu().numpy() for t in (dq, dk, dv)], eg[:3], what=what)
        got_db = dbias[b, h].float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got_db).all()
        assert_grads([got_db], [eg[3]], what=what + " dbias")
        allowed = ref.allowed(w.Sq, w.Sk, *win, w.bottom_right)
        assert (got_db[~allowed] == 0).all()

"""Padded varlen mode: BHSD tensors with a per-batch length array (VarlenMode
not stacked, length = per-sequence array, uniform positions; AOTriton 0.14b
release notes, "VarlenBits supersedes VarlenType").  Batch b attends over its
first seqlen_q[b] queries and seqlen_k[b] keys, with d = seqlen_k[b] -
seqlen_q[b] for the bottom-right diagonal.  The padding rows here hold NaN:
they must not reach any result, and no output row past a batch's lengths may
be written."""

from __future__ import annotations

import ctypes
import os

import numpy as np
import pytest
import torch

from attn_cases import CBR, CTL, INF, assert_grads, assert_o_lse, binding, f64, seed_of
from oracle import attn_ref as ref
from scaled_dot_product_12_b200 import synth

# (seqlen_q, seqlen_k) per batch: a full batch, one query, no keys, no
# queries, and lengths one past / at a tile edge.
LENS = [(300, 357), (1, 40), (177, 0), (0, 5), (129, 128)]
WINDOWS = [(INF, INF, False), (CTL, 0, False), (CBR, 0, True), (256, 0, True), (-64, 128, False),
           (0, 0, True)]
CASES = [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float16, 80)]


def test_padded_mode_encoding_matches_header():
    B = binding()
    text = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                             "include", "attn.h")).read()
    assert "#define ATTN_VARLEN_MODE_PADDED ATTN_VARLEN_MODE(0, 2, 0)" in text
    assert B.MODE_PADDED == B.varlen_mode(0, 2, 0) == 0b00100


def _fwd_params(B, bits, with_lengths):
    p = B.FwdParams()
    p.struct_size = ctypes.sizeof(p)
    p.version = B.PARAMS_VERSION
    p.dtype = B.DTYPE_BF16
    p.B, p.H, p.Sq, p.Sk, p.D = 2, 3, 100, 90, 64
    fake = 0x7F0000000000  # never dereferenced: validation fails first
    p.q = p.k = p.v = p.o = p.lse = fake
    for name in ("q_stride", "k_stride", "v_stride", "o_stride"):
        setattr(p, name, (3 * 128 * 64, 128 * 64, 64))
    p.sm_scale = 0.125
    p.window_left, p.window_right = B.WINDOW_INF, B.WINDOW_INF
    p.varlen_bits = bits
    if with_lengths:
        p.cu_seqlens_q = p.cu_seqlens_k = fake
    return p


def test_padded_mode_needs_both_length_arrays():
    B = binding()
    bits = B.varlen_bits(B.MODE_PADDED, B.MODE_PADDED, 0, 0)
    p = _fwd_params(B, bits, with_lengths=False)
    assert B.lib().attn_fwd(ctypes.byref(p), None) == B.ERROR_INVALID_VALUE
    p.cu_seqlens_q = 0x7F0000000000
    assert B.lib().attn_fwd(ctypes.byref(p), None) == B.ERROR_INVALID_VALUE


def test_each_side_needs_its_own_length_array():
    B = binding()
    fake = 0x7F0000000000
    for qm, km, have_q, have_k in ((B.MODE_PADDED, B.MODE_DENSE, False, True),
                                   (B.MODE_DENSE, B.MODE_PADDED, True, False),
                                   (B.MODE_PACKED, B.MODE_PADDED, False, True),
                                   (B.MODE_PADDED, B.MODE_PACKED, True, False)):
        p = _fwd_params(B, B.varlen_bits(qm, km, 0, 0), with_lengths=False)
        p.total_q = p.total_k = 100
        p.cu_seqlens_q = fake if have_q else 0
        p.cu_seqlens_k = fake if have_k else 0
        assert B.lib().attn_fwd(ctypes.byref(p), None) == B.ERROR_INVALID_VALUE, (qm, km)


@pytest.mark.parametrize("mode", [B_mode for B_mode in (0x05, 0x06, 0x10, 0x12, 0x0D)])
def test_unknown_modes_rejected(mode):
    B = binding()
    for qm, km in ((mode, B.MODE_DENSE), (B.MODE_PADDED, mode)):
        p = _fwd_params(B, B.varlen_bits(qm, km, 0, 0), with_lengths=True)
        assert B.lib().attn_fwd(ctypes.byref(p), None) == B.ERROR_INVALID_VALUE


def test_padded_workspace_matches_dense():
    B = binding()
    for mode in (B.MODE_DENSE, B.MODE_PADDED):
        p = B.BwdParams()
        p.struct_size = ctypes.sizeof(p)
        p.version = B.PARAMS_VERSION
        p.dtype = B.DTYPE_BF16
        p.B, p.H, p.Sq, p.Sk, p.D = 3, 2, 300, 357, 128
        p.sm_scale = 0.1
        p.window_left, p.window_right = B.WINDOW_INF, B.WINDOW_INF
        p.varlen_bits = B.varlen_bits(mode, mode, 0, 0)
        rows = 3 * 300
        want_delta = (2 * rows * 4 + 255) // 256 * 256
        assert B.workspace_bytes(p) == want_delta + 2 * rows * 128 * 4


def _run(dtype, D, window, lse_layout):
    B = binding()
    wl, wr, br = window
    nb, H = len(LENS), 2
    sq_max, sk_max = max(l[0] for l in LENS), max(l[1] for l in LENS)
    q, k, v, do = synth.qkv_do((nb, H, sq_max, D), (nb, H, sk_max, D),
                               seed_of("padded", str(dtype), D, window, lse_layout), dtype)
    nan = float("nan")
    for b, (lq, lk) in enumerate(LENS):
        q[b, :, lq:] = nan
        do[b, :, lq:] = nan
        k[b, :, lk:] = nan
        v[b, :, lk:] = nan
    dev = torch.device("cuda")
    lens_q = torch.tensor([l[0] for l in LENS], dtype=torch.int32, device=dev)
    lens_k = torch.tensor([l[1] for l in LENS], dtype=torch.int32, device=dev)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    scale = D ** -0.5
    th = lse_layout == "TH"
    o = torch.full(qd.shape, nan, dtype=dtype, device=dev)
    lse = torch.full((nb, sq_max, H) if th else (nb, H, sq_max), nan, dtype=torch.float32,
                     device=dev)
    kw = dict(sm_scale=scale, window=(wl, wr), bottom_right=br, lse_layout=lse_layout,
              seqlens_q=lens_q, seqlens_k=lens_k)
    B.forward(qd, kd, vd, out=o, lse=lse, **kw)
    dq, dk, dv = (torch.full_like(t, nan) for t in (qd, kd, vd))
    B.backward(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    o, lse, dq, dk, dv = (t.float().cpu() for t in (o, lse, dq, dk, dv))
    if th:
        lse = lse.transpose(1, 2)
    return (q, k, v, do), dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv), scale


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,D", CASES, ids=lambda x: str(x))
@pytest.mark.parametrize("window", WINDOWS, ids=str)
def test_padded_parity_and_untouched_padding(dtype, D, window):
    wl, wr, br = window
    (q, k, v, do), got, scale = _run(dtype, D, window, "HT")
    for b, (lq, lk) in enumerate(LENS):
        what = f"batch {b} lens ({lq}, {lk}) D={D} w={window}"
        want_o, want_l, want_g = [], [], ([], [], [])
        for h in range(q.shape[1]):
            qb, kb, vb, dob = (f64(t[b, h, :n]) for t, n in ((q, lq), (k, lk), (v, lk), (do, lq)))
            eo, el = ref.forward(qb, kb, vb, scale, wl, wr, br)
            want_o.append(eo)
            want_l.append(el)
            for acc, g in zip(want_g, ref.backward(qb, kb, vb, dob, scale, wl, wr, br)):
                acc.append(g)
        assert_o_lse(got["o"][b, :, :lq].numpy(), got["lse"][b, :, :lq].numpy(),
                     np.stack(want_o), np.stack(want_l), dtype, what)
        assert_grads([got["dq"][b, :, :lq].numpy(), got["dk"][b, :, :lk].numpy(),
                      got["dv"][b, :, :lk].numpy()], [np.stack(g) for g in want_g], what)
        # rows past the lengths are padding: left as they were (NaN)
        for name, n in (("o", lq), ("lse", lq), ("dq", lq), ("dk", lk), ("dv", lk)):
            assert torch.isnan(got[name][b, :, n:]).all(), f"{what}: {name} padding written"


@pytest.mark.gpu
def test_padded_lse_th_layout():
    window = (CBR, 0, True)
    (q, k, v, do), got, scale = _run(torch.bfloat16, 128, window, "TH")
    for b, (lq, lk) in enumerate(LENS):
        for h in range(q.shape[1]):
            _, el = ref.forward(f64(q[b, h, :lq]), f64(k[b, h, :lk]), f64(v[b, h, :lk]), scale,
                                *window)
            g = got["lse"][b, h, :lq].numpy()
            assert np.array_equal(np.isneginf(g), np.isneginf(el))
            fin = ~np.isneginf(el)
            assert np.abs(g[fin] - el[fin]).max(initial=0.0) <= 1e-3
            assert torch.isnan(got["lse"][b, h, lq:]).all()

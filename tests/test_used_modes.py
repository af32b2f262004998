"""The two stacked VarlenModes with a length array (AOTriton 0.14b release
notes, "VarlenBits supersedes VarlenType": a length field that names an array
and a position field that reuses the cumulative sums or names a second
array):

* PACKED_USED: sequence b owns the slot [cu[b], cu[b + 1]) of the packed
  tensor and uses its first seqused[b] rows -- a packed KV cache whose slots
  are longer than their contents;
* PACKED_OFFSETS: sequence b starts at row start[b] (any order, gaps allowed)
  and has seqused[b] rows.

Rows outside every used range hold NaN: they must not reach any result and
must not be written (O, LSE, dQ on the Q side; dK, dV on the K side).  Each
sequence matches the fp64 oracle run on its own used rows, with its own
seqlen_q / seqlen_k (so bottom-right windows shift by the used lengths)."""

import numpy as np
import pytest
import torch

from attn_cases import CBR, CTL, INF, assert_grads, assert_o_lse, binding, f64, seed_of
from oracle import attn_ref as ref
from scaled_dot_product_12_b200 import synth

pytestmark = pytest.mark.gpu
NAN = float("nan")


def _layout(used, slack, seed, offsets):
    """Row ranges of the used parts inside a packed tensor with NaN gaps:
    (positions array, B starts, total rows).  Cumulative slots when not
    `offsets`, else sequences in a shuffled order."""
    g = np.random.default_rng(seed)
    n = len(used)
    extra = [int(g.integers(0, slack + 1)) for _ in range(n)]
    order = g.permutation(n) if offsets else np.arange(n)
    start = [0] * n
    row = int(g.integers(0, 5)) if offsets else 0
    for b in order:
        start[b] = row
        row += used[b] + extra[b]
    if offsets:
        return torch.tensor(start, dtype=torch.int32), start, row
    cu = [0]
    for b in range(n):
        cu.append(cu[-1] + used[b] + extra[b])
    return torch.tensor(cu, dtype=torch.int32), cu[:-1], cu[-1]


def _packed(total, H, D, starts, used, dtype, seed):
    """[total, H, D] N(0,1) values on the used rows and NaN elsewhere."""
    t = torch.full((total, H, D), NAN, dtype=torch.float32)
    g = torch.Generator().manual_seed(seed)
    for s, n in zip(starts, used):
        t[s:s + n] = torch.randn(n, H, D, generator=g)
    return t.to(dtype)


CASES = [
    # (Q mode, K mode, window)
    ("packed", "used", (CTL, 0, False)),
    ("packed", "used", (INF, INF, False)),
    ("packed", "used", (256, 0, True)),
    ("packed", "used", (CBR, 0, True)),
    ("offsets", "packed", (-64, 128, False)),
    ("offsets", "offsets", (CBR, 0, False)),
    ("used", "offsets", (100, 30, True)),
    ("used", "used", (INF, INF, False)),
]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("qmode,kmode,w", CASES, ids=[f"{a}-{b}-{w}" for a, b, w in CASES])
def test_used_length_modes_match_the_oracle_and_leave_gaps_alone(qmode, kmode, w, D):
    B = binding()
    dev = torch.device("cuda")
    H = 2
    used_q = [130, 0, 257, 1, 300]
    used_k = [200, 40, 257, 64, 129]
    seed = seed_of("used-modes", qmode, kmode, w, D) & 0xFFFF
    dtype = torch.bfloat16

    def side(mode, used, s):
        if mode == "packed":
            arr = synth.cumsum0(used)
            return arr, arr[:-1].tolist(), int(arr[-1]), None
        arr, starts, total = _layout(used, 50, s, offsets=(mode == "offsets"))
        return arr, starts, total, torch.tensor(used, dtype=torch.int32)
    arr_q, st_q, tq, sused_q = side(qmode, used_q, seed)
    arr_k, st_k, tk, sused_k = side(kmode, used_k, seed + 1)
    q = _packed(tq, H, D, st_q, used_q, dtype, seed + 2)
    do = _packed(tq, H, D, st_q, used_q, dtype, seed + 3)
    k = _packed(tk, H, D, st_k, used_k, dtype, seed + 4)
    v = _packed(tk, H, D, st_k, used_k, dtype, seed + 5)

    kw = dict(sm_scale=D ** -0.5, window=w[:2], bottom_right=w[2], lse_layout="TH",
              max_seqlen_q=max(used_q), max_seqlen_k=max(used_k))
    for name, mode, arr, used in (("q", qmode, arr_q, sused_q), ("k", kmode, arr_k, sused_k)):
        if mode == "offsets":
            kw[f"seqstart_{name}"] = arr.to(dev)
        else:
            kw[f"cu_seqlens_{name}"] = arr.to(dev)
        if used is not None:
            kw[f"seqused_{name}"] = used.to(dev)

    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    o = torch.full_like(qd, NAN)
    lse = torch.full((tq, H), NAN, device=dev)
    dq, dk, dv = torch.full_like(qd, NAN), torch.full_like(kd, NAN), torch.full_like(vd, NAN)
    B.forward(qd, kd, vd, out=o, lse=lse, **kw)
    B.backward(dod, qd, kd, vd, o, lse, dq=dq, dk=dk, dv=dv, **kw)
    torch.cuda.synchronize()
    assert B.device_status(dev) == 0
    o, lse, dq, dk, dv = (t.float().cpu() for t in (o, lse, dq, dk, dv))

    def gaps(total, starts, used):
        m = torch.ones(total, dtype=torch.bool)
        for s, n in zip(starts, used):
            m[s:s + n] = False
        return m
    gq, gk = gaps(tq, st_q, used_q), gaps(tk, st_k, used_k)
    for name, t, gmask in (("O", o, gq), ("LSE", lse, gq), ("dQ", dq, gq), ("dK", dk, gk),
                           ("dV", dv, gk)):
        assert torch.isnan(t[gmask]).all(), f"{name}: a row outside every sequence was written"

    for b in range(len(used_q)):
        rq = slice(st_q[b], st_q[b] + used_q[b])
        rk = slice(st_k[b], st_k[b] + used_k[b])
        if used_q[b] == 0:
            continue
        for h in range(H):
            a = (f64(q[rq, h]), f64(k[rk, h]), f64(v[rk, h]))
            eo, el = ref.forward(*a, D ** -0.5, *w)
            assert_o_lse(o[rq, h].numpy(), lse[rq, h].numpy(), eo, el, dtype,
                         what=f"seq {b} head {h}")
            if used_k[b] == 0:
                continue
            eg = ref.backward(*a, f64(do[rq, h]), D ** -0.5, *w)
            assert_grads([dq[rq, h].numpy(), dk[rk, h].numpy(), dv[rk, h].numpy()], eg,
                         what=f"seq {b} head {h}")


def test_used_length_is_clamped_to_its_slot():
    # seqused larger than the slot: the sequence is the whole slot, nothing past it
    B = binding()
    dev = torch.device("cuda")
    H, D = 2, 64
    slots_k = [100, 150]
    cu_k = synth.cumsum0(slots_k)
    used_k = torch.tensor([1000, 20], dtype=torch.int32)
    sq = [90, 80]
    cu_q = synth.cumsum0(sq)
    q, k, v, do = synth.qkv_do((sum(sq), H, D), (sum(slots_k), H, D), 77, torch.bfloat16)
    o, lse = B.forward(q.to(dev), k.to(dev), v.to(dev), cu_seqlens_q=cu_q.to(dev),
                       cu_seqlens_k=cu_k.to(dev), seqused_k=used_k.to(dev), max_seqlen_q=90,
                       max_seqlen_k=1000, lse_layout="TH")
    torch.cuda.synchronize()
    o, lse = o.float().cpu(), lse.cpu()
    for b, (ks, kn) in enumerate(((0, 100), (100, 20))):
        rq = slice(int(cu_q[b]), int(cu_q[b + 1]))
        for h in range(H):
            eo, el = ref.forward(f64(q[rq, h]), f64(k[ks:ks + kn, h]), f64(v[ks:ks + kn, h]),
                                 D ** -0.5, INF, INF)
            assert_o_lse(o[rq, h].numpy(), lse[rq, h].numpy(), eo, el, torch.bfloat16)

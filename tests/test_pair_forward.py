"""GPU parity of the CTA-pair forward (dense inputs, no window, bias or
dropout, head dims above 64: the calls the library routes to the two-SM
kernel; here D = 128, the other head dims are in test_head_dims.py) against
the fp64 oracle, on shapes that stress what that kernel adds: many
512-row units per CTA pair (persistent loop, Q buffers reused across units),
a last round split into 256-row half units,
units whose second CTA has no valid rows, ragged key tiles, a single query
row, fp16 with a negative scale and the TH LSE layout, and strided views."""

import pytest
import torch

from attn_cases import INF, assert_o_lse, dense_inputs, oracle_dense, run_dense, seed_of

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, Sq, Sk, dtype, scale, lse layout
    (3, 50, 700, 333, torch.bfloat16, None, "HT"),     # 300 units: several per pair
    (2, 40, 1030, 1025, torch.float16, -0.07, "TH"),   # last unit: CTA 1 has no rows
    (1, 3, 1, 5000, torch.bfloat16, None, "HT"),       # one query row
    (2, 2, 4096, 129, torch.bfloat16, 0.3, "HT"),      # second key tile holds one key
    (1, 1, 512, 512, torch.float16, None, "HT"),       # exactly one unit
    (1, 80, 1000, 300, torch.bfloat16, None, "HT"),    # 160 units: last round in half units
]


@pytest.mark.parametrize("B,H,sq,sk,dtype,scale,layout", CASES)
def test_pair_forward_matches_oracle(B, H, sq, sk, dtype, scale, layout):
    seed = seed_of("pair", B, H, sq, sk, str(dtype), scale, layout)
    q, k, v, do = dense_inputs(B, H, sq, sk, 128, dtype, seed)
    scale = 128 ** -0.5 if scale is None else scale
    got = run_dense(q, k, v, do, scale, INF, INF, False, lse_layout=layout, backward=False)
    want = oracle_dense(q, k, v, do, scale, INF, INF, False, backward=False)
    lse = got["lse"].numpy()
    if layout == "TH":
        lse = lse.transpose(0, 2, 1)
    assert_o_lse(got["o"].float().numpy(), lse, want["o"], want["lse"], dtype,
                 what=f"pair B{B} H{H} {sq}x{sk}")


def test_pair_forward_strided_views():
    """Q, K, V and O as [B, S, H, D] storage seen through [B, H, S, D] views."""
    B, H, sq, sk = 2, 6, 777, 901
    seed = seed_of("pair-strided", B, H, sq, sk)
    q, k, v, do = dense_inputs(B, H, sq, sk, 128, torch.bfloat16, seed)
    qs, ks, vs = (t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v))
    assert not qs.is_contiguous()
    got = run_dense(qs, ks, vs, do, 128 ** -0.5, INF, INF, False, backward=False)
    want = oracle_dense(q, k, v, do, 128 ** -0.5, INF, INF, False, backward=False)
    assert_o_lse(got["o"].float().numpy(), got["lse"].numpy(), want["o"], want["lse"],
                 torch.bfloat16, what="pair strided")

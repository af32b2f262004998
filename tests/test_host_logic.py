"""Host-side logic that needs no GPU: how the binding derives sizes and
VarlenBits from the tensors it is given (each side dense, packed or padded),
and the bench's choice of roofline denominator and helper-kernel bandwidth."""

from __future__ import annotations

import pytest
import torch

import bench
from scaled_dot_product_12_b200 import binding as B
from scaled_dot_product_12_b200 import synth


def _t(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _problem(q, k, **kw):
    args = dict(cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None, max_seqlen_k=None)
    args.update(kw)
    return B.Problem(q, k, None, (B.WINDOW_INF, B.WINDOW_INF), False, args["cu_seqlens_q"],
                     args["cu_seqlens_k"], args["max_seqlen_q"], args["max_seqlen_k"], "HT",
                     kw.get("seqlens_q"), kw.get("seqlens_k"))


def test_dense_sizes_and_bits():
    pr = _problem(_t(2, 3, 100, 64), _t(2, 3, 90, 64))
    assert (pr.B, pr.H, pr.Sq, pr.Sk, pr.D) == (2, 3, 100, 90, 64)
    assert pr.bits == 0 and pr.lse_shape() == (2, 3, 100)


def test_packed_q_dense_k():
    cu = synth.cumsum0([5, 7])
    pr = _problem(_t(12, 3, 64), _t(2, 3, 90, 64), cu_seqlens_q=cu, max_seqlen_q=7)
    assert (pr.B, pr.Sq, pr.Sk, pr.total_q, pr.total_k) == (2, 7, 90, 12, 0)
    assert pr.bits == B.varlen_bits(B.MODE_PACKED, B.MODE_DENSE, 0, 0)
    assert pr.lse_shape() == (3, 12)
    assert pr.cu_q is cu and pr.cu_k is None


def test_padded_q_packed_k():
    lens = torch.tensor([3, 9], dtype=torch.int32)
    cu_k = synth.cumsum0([4, 0])
    pr = _problem(_t(2, 3, 9, 64), _t(4, 3, 64), seqlens_q=lens, cu_seqlens_k=cu_k,
                  max_seqlen_k=4)
    assert (pr.B, pr.Sq, pr.Sk, pr.total_q, pr.total_k) == (2, 9, 4, 0, 4)
    assert pr.bits == B.varlen_bits(B.MODE_PADDED, B.MODE_PACKED, 0, 0)
    assert pr.cu_q is lens and pr.cu_k is cu_k


@pytest.mark.parametrize("kw,q,k", [
    (dict(seqlens_q=torch.tensor([1, 2], dtype=torch.int32),
          cu_seqlens_q=synth.cumsum0([1, 2]), max_seqlen_q=2), (3, 3, 64), (2, 3, 5, 64)),
    (dict(cu_seqlens_q=synth.cumsum0([1, 2])), (3, 3, 64), (2, 3, 5, 64)),          # no max_seqlen
    (dict(cu_seqlens_q=synth.cumsum0([1, 2, 3]), max_seqlen_q=3), (6, 3, 64), (2, 3, 5, 64)),
    (dict(seqlens_k=torch.tensor([1, 2, 3], dtype=torch.int32)), (2, 3, 5, 64), (2, 3, 5, 64)),
    (dict(), (3, 3, 64), (2, 3, 5, 64)),                                             # 3-D dense
])
def test_inconsistent_calls_rejected(kw, q, k):
    with pytest.raises(ValueError):
        _problem(_t(*q), _t(*k), **kw)


def test_roofline_denominator_follows_the_clocks():
    # a throttle flag with the clock still at its maximum: burst figure
    assert not bench.clock_lowered({"reasons": ["sw_power_cap"], "sm_mhz": 1965,
                                    "sm_max_mhz": 1965})
    assert bench.clock_lowered({"reasons": ["sw_power_cap"], "sm_mhz": 1755, "sm_max_mhz": 1965})
    assert bench.clock_lowered({"reasons": [], "sm_mhz": 1700, "sm_max_mhz": 1965})
    assert not bench.clock_lowered({"reasons": [], "sm_mhz": 1950, "sm_max_mhz": 1965})
    assert not bench.clock_lowered({"reasons": ["clocks not sampled"], "sm_mhz": None,
                                    "sm_max_mhz": None})
    # the recorded source names the reasons that were actually seen
    src = bench.peak_source("measured", True, {"sm_mhz": 1700, "sm_max_mhz": 1965,
                                               "reasons": ["sw_thermal_slowdown"]})
    assert "sw_thermal_slowdown" in src and "power cap" not in src
    assert "none" in bench.peak_source("measured", True, {"sm_mhz": 1700, "sm_max_mhz": 1965,
                                                          "reasons": []})


def test_helper_kernel_bytes():
    w = synth.WORKLOADS["ltx_15300"]
    nb = bench.workload_bytes(w)
    rows = 15300 * 32
    assert nb["bwd_other"] == rows * (14 * 128 + 4)
    assert nb["attn_fwd_kernel"] == rows * (4 * 128 + 4) + rows * 4 * 128
    assert nb["attn_bwd_kernel"] == rows * (12 * 128 + 8) + rows * 8 * 128
    d = bench.other_bandwidth(nb["bwd_other"], 0.2, 6542.1)
    assert d["gbs"] == pytest.approx(d["bytes"] / 0.2e-3 / 1e9, rel=1e-3)
    assert d["frac"] == pytest.approx(d["gbs"] / 6542.1, rel=1e-3)
    assert bench.other_bandwidth(nb["bwd_other"], 0.0, 6542.1)["gbs"] is None
    # packed workloads count their tokens, not B * max_seqlen
    wv = synth.VARLEN_WORKLOADS["varlen_D128_w256_0_TL"]
    sq, sk = synth.varlen_seqlens(synth.VARLEN_SEQLEN_SEED)
    assert bench.workload_bytes(wv)["bwd_other"] == 16 * sum(sq) * (14 * 128 + 4)
    assert bench.workload_bytes(wv)["attn_fwd_kernel"] == \
        16 * sum(sq) * (4 * 128 + 4) + 16 * sum(sk) * 4 * 128


def test_kernel_roofline_picks_the_binding_resource():
    r = bench.kernel_roofline("k", 1e12, 1e6, 1.0, 1000.0, 6000.0)   # AI 1e6: tensor
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(1000.0) and r["frac"] == pytest.approx(1.0)
    r = bench.kernel_roofline("k", 1e9, 6e9, 1.0, 1000.0, 6000.0)    # AI 0.17: HBM
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(6000.0) and r["frac"] == pytest.approx(1.0)


INF, CTL, CBR = synth.WINDOW_INF, synth.CAUSAL_TOP_LEFT, synth.CAUSAL_BOTTOM_RIGHT


@pytest.mark.parametrize("w", [(INF, INF, 0), (CTL, 0, 0), (CTL, 0, 1), (CBR, 0, 0), (CBR, 0, 1),
                               (INF, 0, 1), (256, 0, 0), (256, 0, 1), (-64, 128, 0),
                               (-64, 128, 1), (3, -5, 0), (0, 0, 1), (-300, 200, 1),
                               (130, INF, 1), (INF, -7, 0)])
@pytest.mark.parametrize("sq,sk", [(1, 1), (5, 9), (128, 128), (200, 333), (333, 200),
                                   (700, 513)])
def test_bench_pair_count_matches_the_oracle_mask(w, sq, sk):
    from oracle import attn_ref as ref
    assert bench.pair_count(sq, sk, *w) == ref.allowed_count(sq, sk, *w)


def test_bench_flops_of_the_packed_workload():
    from oracle import attn_ref as ref
    wv = synth.VARLEN_WORKLOADS["varlen_D128_w-64_128_BR"]
    sq, sk = synth.varlen_seqlens(synth.VARLEN_SEQLEN_SEED)
    want = 16 * sum(ref.allowed_count(a, b, -64, 128, True) for a, b in zip(sq, sk))
    f, b, n = bench.workload_flops(wv)
    assert n == want and f == 4 * 128 * n and b == 10 * 128 * n


def test_traffic_is_null_for_other_kernel_builds(tmp_path, monkeypatch):
    import json
    root = tmp_path
    (root / "profiles").mkdir()
    src = root / "scaled_dot_product_12_b200" / "csrc"
    src.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES:
        (src / name).write_text(name)
    monkeypatch.setattr(bench, "ROOT", str(root))
    hashes = {k: bench.kernels_sha256(k) for k in ("attn_bwd_kernel", "attn_fwd_pair_kernel")}
    table = {"attn_bwd_kernel:ltx_15300": 123, "attn_fwd_pair_kernel:ltx_15300": 45}
    (root / "profiles" / "traffic.json").write_text(
        json.dumps({"kernels_sha256": hashes, "bytes_per_launch": table}))
    assert bench.load_traffic("attn_bwd_kernel", "ltx_15300") == 123
    assert bench.load_traffic("attn_fwd_pair_kernel", "ltx_15300") == 45
    assert bench.load_traffic("attn_fwd_kernel", "ltx_15300") is None  # no record
    # a change to one kernel's source voids its counters, not another's
    (src / "fwd_pair.cu").write_text("changed")
    assert bench.load_traffic("attn_fwd_pair_kernel", "ltx_15300") is None
    assert bench.load_traffic("attn_bwd_kernel", "ltx_15300") == 123
    (src / "common.cuh").write_text("changed")
    assert bench.load_traffic("attn_bwd_kernel", "ltx_15300") is None


def test_forward_kernel_name_follows_the_dispatch_rule():
    """Dense calls at D = 128 without a window or bias run the CTA-pair kernel."""
    w = synth.ALL_WORKLOADS
    assert bench.fwd_kernel_name(w["ltx_15300"], False) == "attn_fwd_pair_kernel"
    assert bench.fwd_kernel_name(w["ltx_15300"], True) == "attn_fwd_kernel"
    assert bench.fwd_kernel_name(w["bert_large"], False) == "attn_fwd_kernel"
    assert bench.fwd_kernel_name(w["gpt2"], False) == "attn_fwd_kernel"
    assert bench.fwd_kernel_name(w["varlen_D128_w256_0_TL"], False) == "attn_fwd_kernel"


def test_end_to_end_groups_cover_the_workload_once():
    for name, w in synth.ALL_WORKLOADS.items():
        dim, groups = bench.e2e_groups(w, 4)
        if w.packed or name == "tiny_causal":
            assert dim is None and groups == [slice(None)]
            continue
        size = w.B if dim == 0 else w.H
        assert dim == (0 if w.B > 1 else 1)
        covered = [i for g in groups for i in range(size)[g]]
        assert covered == list(range(size)), name
        assert 1 <= len(groups) <= 4


def test_kernel_hash_ignores_comments_but_not_code():
    import bench
    base = 'int f(int a) { return a + 1; }  // one\n/* two */ const char* s = "// x";\n'
    same = '// header\nint f(int a)   {\n  return a + 1;  /* changed */ }\nconst char* s = "// x";'
    other = 'int f(int a) { return a + 2; }  // one\n/* two */ const char* s = "// x";\n'
    lit = 'int f(int a) { return a + 1; }  // one\n/* two */ const char* s = "// y";\n'
    assert bench._code_only(base) == bench._code_only(same)
    assert bench._code_only(base) != bench._code_only(other)
    assert bench._code_only(base) != bench._code_only(lit)  # string contents are code

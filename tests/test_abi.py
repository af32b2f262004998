"""Host-side checks of the C ABI (CPU only: no call here reaches a kernel).

* the library loads and exports every function include/attn.h declares;
* the header's constants match the binding's;
* parameter validation rejects what the header says it rejects;
* the kernels' tile plan and the FLOP-count helper, run on the host, agree
  with the fp64 oracle's mask.
"""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import attn_ref as ref

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def B(lib_path):
    from scaled_dot_product_12_b200 import binding
    binding.lib()
    return binding


def _declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib_path):
    names = _declared_functions()
    assert {"attn_fwd", "attn_bwd", "attn_bwd_workspace_size"} <= set(names)
    handle = ctypes.CDLL(lib_path)
    for n in names:
        assert hasattr(handle, n), n


def test_binding_covers_every_export(B):
    assert set(_declared_functions()) == set(B.EXPORTS)


def test_header_constants_match_binding(B):
    text = open(HEADER).read()
    def macro(name):
        m = re.search(rf"#define {name}\s+\(?(-?\d+)\s*(-\s*1)?\)?", text)
        val = int(m.group(1))
        return val - 1 if m.group(2) else val
    assert macro("ATTN_WINDOW_INF") == B.WINDOW_INF
    assert macro("ATTN_CAUSAL_TOP_LEFT") == B.CAUSAL_TOP_LEFT
    assert macro("ATTN_CAUSAL_BOTTOM_RIGHT") == B.CAUSAL_BOTTOM_RIGHT
    assert macro("ATTN_ERROR_INVALID_VALUE") == B.ERROR_INVALID_VALUE
    assert B.MODE_PACKED == 0b01011 and B.MODE_DENSE == 0
    assert B.varlen_bits(B.MODE_PACKED, B.MODE_PACKED, 1, 1) == (0x0B | 0x0B00 | 0x10000 | 0x40000)
    # the oracle and the input generator restate the same encodings
    from scaled_dot_product_12_b200 import synth
    assert (ref.WINDOW_INF, ref.CAUSAL_TOP_LEFT, ref.CAUSAL_BOTTOM_RIGHT) == \
        (B.WINDOW_INF, B.CAUSAL_TOP_LEFT, B.CAUSAL_BOTTOM_RIGHT) == \
        (synth.WINDOW_INF, synth.CAUSAL_TOP_LEFT, synth.CAUSAL_BOTTOM_RIGHT)


FAKE = 0x7F0000000000  # never dereferenced: every case below fails validation first


def _fwd(lib_b, **kw):
    B = lib_b
    p = B.FwdParams()
    p.struct_size = ctypes.sizeof(p)
    p.version = B.PARAMS_VERSION
    p.dtype = B.DTYPE_BF16
    p.B, p.H, p.Sq, p.Sk, p.D = 2, 3, 100, 90, 64
    p.q = p.k = p.v = p.o = p.lse = FAKE
    for name in ("q_stride", "k_stride", "v_stride", "o_stride"):
        setattr(p, name, (3 * 128 * 64, 128 * 64, 64))
    p.sm_scale = 0.125
    p.window_left, p.window_right = B.WINDOW_INF, B.WINDOW_INF
    p.varlen_bits = 0
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _call_fwd(B, p):
    return B.lib().attn_fwd(ctypes.byref(p), None)


@pytest.mark.parametrize("field,value", [
    ("struct_size", 8), ("version", 4), ("version", 2), ("version", 1), ("dtype", 2), ("D", 144), ("D", 0),
    ("D", -3),
    ("B", -1), ("Sq", 1 << 30), ("sm_scale", float("nan")), ("sm_scale", float("inf")),
    ("varlen_bits", 1 << 19), ("varlen_bits", 1 << 31), ("varlen_bits", 0x20),
    ("varlen_bits", 0x2000), ("varlen_bits", 2 << 16), ("varlen_bits", 3 << 16),
    ("varlen_bits", 0x0B),                       # packed Q without cu_seqlens_q
    ("varlen_bits", 0x0505),                     # stacked, length array, uniform positions
    ("varlen_bits", 0x1313),                     # stacked, cumulative lengths, position array
    ("flags", 1), ("flags", 2), ("Dv", -1), ("Dv", 129), ("dropout_p", -0.1), ("dropout_p", 1.0),
    ("dropout_p", float("nan")),
    ("q", 0), ("o", 0), ("k", 0), ("q", FAKE + 8), ("o", FAKE + 2),
    ("q_stride", (3 * 128 * 64, 128 * 64, 60)),  # row stride of 120 bytes
    ("k_stride", (3 * 128 * 64, 0, 64)),         # zero head stride with H > 1
    ("bias", FAKE + 8),                          # bias base not 16-byte aligned
])
def test_forward_rejects_invalid_parameters(B, field, value):
    assert _call_fwd(B, _fwd(B, **{field: value})) == B.ERROR_INVALID_VALUE


def test_empty_head_dim_128_problems_succeed_without_a_device(B):
    # dense D = 128 calls go to the CTA-pair kernel: an empty batch or head
    # count returns before any launch, as for every other kernel
    st = (3 * 128 * 128, 128 * 128, 128)
    for kw in ({"B": 0}, {"H": 0}, {"B": 0, "H": 0}):
        p = _fwd(B, D=128, q_stride=st, k_stride=st, v_stride=st, o_stride=st, **kw)
        assert _call_fwd(B, p) == 0


def test_version_one_callers_are_accepted(B):
    # a caller built against version 1 passes version 1 and the version-1 size:
    # the call validates (an empty problem succeeds without a device) ...
    p = _fwd(B, B=0, version=1, struct_size=B.FWD_PARAMS_V1_SIZE)
    assert _call_fwd(B, p) == 0
    # ... and the version-2 fields it cannot know are not read
    p = _fwd(B, B=0, version=1, struct_size=B.FWD_PARAMS_V1_SIZE, flags=7, Dv=-5)
    assert _call_fwd(B, p) == 0
    q = _bwd(B, B=0, version=1, struct_size=B.BWD_PARAMS_V1_SIZE)
    assert B.lib().attn_bwd(ctypes.byref(q), None) == 0
    assert B.lib().attn_bwd_workspace_size(ctypes.byref(_bwd(B, version=1,
                                                            struct_size=B.BWD_PARAMS_V1_SIZE))) \
        == B.lib().attn_bwd_workspace_size(ctypes.byref(_bwd(B)))


def test_version_two_callers_are_accepted(B):
    # version 2 (no bias fields): validated without reading past its size
    p = _fwd(B, B=0, version=2, struct_size=B.FWD_PARAMS_V2_SIZE, bias=FAKE + 2)
    assert _call_fwd(B, p) == 0
    q = _bwd(B, B=0, version=2, struct_size=B.BWD_PARAMS_V2_SIZE, dbias=FAKE + 2)
    assert B.lib().attn_bwd(ctypes.byref(q), None) == 0
    assert B.lib().attn_bwd_workspace_size(ctypes.byref(_bwd(B, version=2,
                                                            struct_size=B.BWD_PARAMS_V2_SIZE))) \
        == B.lib().attn_bwd_workspace_size(ctypes.byref(_bwd(B)))
    # a version-2 number with the current size (or the reverse) is refused
    assert _call_fwd(B, _fwd(B, B=0, version=2)) == B.ERROR_INVALID_VALUE
    assert _call_fwd(B, _fwd(B, B=0, struct_size=B.FWD_PARAMS_V2_SIZE)) == B.ERROR_INVALID_VALUE


def test_header_older_struct_sizes_match_the_binding(B):
    text = open(HEADER).read()
    assert "offsetof(attn_fwd_params, seqused_q)" in text
    assert "offsetof(attn_bwd_params, seqused_q)" in text
    assert "offsetof(attn_fwd_params, bias)" in text
    assert "offsetof(attn_bwd_params, bias)" in text
    assert B.FwdParams.seqused_q.offset == B.FWD_PARAMS_V1_SIZE
    assert B.BwdParams.seqused_q.offset == B.BWD_PARAMS_V1_SIZE
    assert B.FwdParams.bias.offset == B.FWD_PARAMS_V2_SIZE
    assert B.BwdParams.bias.offset == B.BWD_PARAMS_V2_SIZE


BIAS_STRIDES = (3 * 100 * 96, 100 * 96, 96)   # [B=2, H=3, Sq=100, Sk=90] rows padded to 96


@pytest.mark.parametrize("strides", [
    (3 * 100 * 96, 100 * 96, 90),     # row stride of 180 bytes
    (3 * 100 * 96, 100 * 96, 0),      # every query row on one row
    (3 * 100 * 96, 100 * 96 + 4, 96), # head stride of odd 8-byte multiple
    (-96, 100 * 96, 96),              # negative batch stride
])
def test_bias_strides_rejected(B, strides):
    p = _fwd(B, bias=FAKE, bias_stride=strides)
    assert _call_fwd(B, p) == B.ERROR_INVALID_VALUE
    q = _bwd(B, workspace_bytes=1 << 30, bias=FAKE, bias_stride=strides)
    assert B.lib().attn_bwd(ctypes.byref(q), None) == B.ERROR_INVALID_VALUE


@pytest.mark.parametrize("strides", [(0, 100 * 96, 96), (3 * 100 * 96, 0, 96), (0, 0, 96)])
def test_bias_broadcast_passes_validation_but_dbias_broadcast_does_not(B, strides):
    # validation passes (the call then fails only for want of a device here)
    p = _fwd(B, bias=FAKE, bias_stride=strides)
    assert _call_fwd(B, p) != B.ERROR_INVALID_VALUE
    q = _bwd(B, workspace_bytes=1 << 30, bias=FAKE, bias_stride=strides)
    assert B.lib().attn_bwd(ctypes.byref(q), None) != B.ERROR_INVALID_VALUE
    q = _bwd(B, workspace_bytes=1 << 30, dbias=FAKE, dbias_stride=strides)
    assert B.lib().attn_bwd(ctypes.byref(q), None) == B.ERROR_INVALID_VALUE
    q = _bwd(B, workspace_bytes=1 << 30, dbias=FAKE + 8, dbias_stride=BIAS_STRIDES)
    assert B.lib().attn_bwd(ctypes.byref(q), None) == B.ERROR_INVALID_VALUE


@pytest.mark.parametrize("mode_name", ["MODE_PACKED_USED", "MODE_PACKED_OFFSETS"])
def test_used_length_modes_need_their_arrays(B, mode_name):
    mode = getattr(B, mode_name)
    bits = B.varlen_bits(mode, B.MODE_DENSE, 0, 0)
    p = _fwd(B, varlen_bits=bits, total_q=100, cu_seqlens_q=FAKE)   # no seqused_q
    p.q_stride = p.o_stride = (0, 64, 3 * 64)
    assert _call_fwd(B, p) == B.ERROR_INVALID_VALUE
    p = _fwd(B, varlen_bits=bits, total_q=100, seqused_q=FAKE)      # no positions
    p.q_stride = p.o_stride = (0, 64, 3 * 64)
    assert _call_fwd(B, p) == B.ERROR_INVALID_VALUE


def test_reserved_diagonal_bits_rejected_but_diagonal_accepted_in_validation(B):
    # bit 18 is the diagonal (valid); bits 19..31 are reserved.
    for bit in range(19, 32):
        assert _call_fwd(B, _fwd(B, varlen_bits=1 << bit)) == B.ERROR_INVALID_VALUE


def test_packed_needs_cu_seqlens(B):
    bits = B.varlen_bits(B.MODE_PACKED, B.MODE_PACKED, 0, 0)
    p = _fwd(B, varlen_bits=bits, total_q=100, total_k=90)
    p.q_stride = p.o_stride = p.k_stride = p.v_stride = (0, 64, 3 * 64)
    assert _call_fwd(B, p) == B.ERROR_INVALID_VALUE


@pytest.mark.parametrize("field", ["B", "H", "Sq"])
def test_empty_problems_succeed_without_a_device(B, field):
    p = _fwd(B, **{field: 0})
    assert _call_fwd(B, p) == 0


def _bwd(lib_b, **kw):
    B = lib_b
    p = B.BwdParams()
    p.struct_size = ctypes.sizeof(p)
    p.version = B.PARAMS_VERSION
    p.dtype = B.DTYPE_FP16
    p.B, p.H, p.Sq, p.Sk, p.D = 2, 3, 100, 90, 128
    for n in ("q", "k", "v", "o", "dout", "lse", "dq", "dk", "dv", "workspace"):
        setattr(p, n, FAKE)
    for n in ("q", "k", "v", "o", "do", "dq", "dk", "dv"):
        setattr(p, n + "_stride", (3 * 128 * 128, 128 * 128, 128))
    p.sm_scale = 0.1
    p.window_left, p.window_right = B.CAUSAL_TOP_LEFT, 0
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("kw", [
    dict(H=3, B=1 << 20, Sq=1024),                                    # dense: 3 * 2^30 rows
    dict(H=4, total_q=(1 << 29) + 64, total_k=300, cu_seqlens_q=FAKE, cu_seqlens_k=FAKE),
])
def test_backward_rejects_rows_past_the_tma_coordinate_range(B, kw):
    # H * rows_q rows of the fp32 dQ accumulator are addressed by a signed
    # 32-bit TMA coordinate: 2^31 - 256 or more is refused before any launch.
    if "total_q" in kw:
        kw = dict(kw, varlen_bits=B.varlen_bits(B.MODE_PACKED, B.MODE_PACKED, 0, 0))
    p = _bwd(B, workspace_bytes=1 << 62, **kw)  # the workspace check alone would pass
    assert B.lib().attn_bwd(ctypes.byref(p), None) == B.ERROR_INVALID_VALUE


def test_workspace_size_formula(B):
    p = _bwd(B)
    n = 3 * 2 * 100
    want = ((n * 4 + 255) // 256) * 256 + n * 128 * 4
    assert B.lib().attn_bwd_workspace_size(ctypes.byref(p)) == want
    pk = _bwd(B, varlen_bits=B.varlen_bits(B.MODE_PACKED, B.MODE_PACKED, 1, 0), total_q=333,
              total_k=300)
    n = 3 * 333
    assert B.lib().attn_bwd_workspace_size(ctypes.byref(pk)) == ((n * 4 + 255) // 256) * 256 + n * 128 * 4
    assert B.lib().attn_bwd_workspace_size(ctypes.byref(_bwd(B, version=7))) == 0


@pytest.mark.parametrize("field,value", [
    ("workspace_bytes", 100), ("workspace", 0), ("workspace", FAKE + 16), ("lse", 0),
    ("dout", 0), ("dq", 0), ("dk", FAKE + 4), ("do_stride", (3 * 128 * 128, 128 * 128, 100)),
    ("varlen_bits", 1 << 20),
])
def test_backward_rejects_invalid_parameters(B, field, value):
    p = _bwd(B, workspace_bytes=1 << 30)
    setattr(p, field, value)
    assert B.lib().attn_bwd(ctypes.byref(p), None) == B.ERROR_INVALID_VALUE


INF, CTL, CBR = ref.WINDOW_INF, ref.CAUSAL_TOP_LEFT, ref.CAUSAL_BOTTOM_RIGHT
PLAN_WINDOWS = [(INF, INF, 0), (CTL, 0, 0), (CTL, 0, 1), (CBR, 0, 0), (INF, 0, 1),
                (256, 0, 0), (256, 0, 1), (-64, 128, 0), (-64, 128, 1), (3, -5, 0),
                (0, 0, 1), (-300, 200, 1), (130, INF, 1)]
PLAN_SIZES = [(1, 1), (128, 128), (200, 333), (333, 200), (513, 700), (129, 5)]


@pytest.mark.parametrize("w", PLAN_WINDOWS)
@pytest.mark.parametrize("sq,sk", PLAN_SIZES)
def test_tile_plan_covers_exactly_the_allowed_pairs(B, w, sq, sk):
    mask = ref.allowed(sq, sk, *w)
    for m0 in range(0, sq, 128):
        nb, ne, full = B.tile_plan(sq, sk, w[0], w[1], w[2], m0)
        rows = mask[m0:m0 + 128]
        cols = np.nonzero(rows.any(0))[0]
        if len(cols):
            assert nb <= cols[0] // 128 and cols[-1] // 128 < ne
        for n in range(nb, ne):
            tile = mask[m0:m0 + 128, n * 128:(n + 1) * 128]
            is_full = tile.shape == (128, 128) and tile.all()
            assert bool(full[n - nb]) == is_full, (m0, n)
        if rows.any(1).all() and ne > nb:
            # when no row is empty the range is tight at both ends
            assert mask[m0:m0 + 128, nb * 128:(nb + 1) * 128].any()
            assert mask[m0:m0 + 128, (ne - 1) * 128:ne * 128].any()


@pytest.mark.parametrize("w", PLAN_WINDOWS)
@pytest.mark.parametrize("sq,sk", PLAN_SIZES)
def test_backward_tile_plan_covers_every_query_of_a_key_tile(B, w, sq, sk):
    mask = ref.allowed(sq, sk, *w)
    for n0 in range(0, sk, 128):
        mb, me = B.tile_plan_bwd(sq, sk, w[0], w[1], w[2], n0)
        qs = np.nonzero(mask[:, n0:n0 + 128].any(1))[0]
        if len(qs):
            assert mb <= qs[0] // 128 and qs[-1] // 128 < me
        else:
            assert me <= mb or not mask[mb * 128:me * 128, n0:n0 + 128].any()


@pytest.mark.parametrize("w", PLAN_WINDOWS)
@pytest.mark.parametrize("sq,sk", PLAN_SIZES + [(6630, 6630), (15300, 15300)])
def test_allowed_pairs_matches_oracle_count(B, w, sq, sk):
    if sq * sk > 2e7 and w[0] not in (INF, CTL):
        pytest.skip("large sizes only for the two common windows")
    assert B.allowed_pairs(sq, sk, *w) == ref.allowed_count(sq, sk, *w)


@pytest.mark.parametrize("w", PLAN_WINDOWS + [(-500, 600, 0), (-130, 2, 1), (700, -650, 0)])
@pytest.mark.parametrize("sq,sk", PLAN_SIZES + [(1000, 300), (300, 1000)])
def test_key_tiles_visiting_a_query_tile_are_contiguous(B, w, sq, sk):
    # The deterministic backward orders the dQ contributions of one query tile
    # by key tile and gives each key tile the rank n - n_lo, n_lo found by
    # bisection on "m < m_end(n)": that needs the visiting key tiles to form
    # one run, and every key tile below a visiting one to have m_end <= m or
    # to visit too.
    plans = [B.tile_plan_bwd(sq, sk, w[0], w[1], w[2], n0) for n0 in range(0, sk, 128)]
    for m in range(0, (sq + 127) // 128):
        visit = [mb <= m < me for mb, me in plans]
        ns = [n for n, v in enumerate(visit) if v]
        if not ns:
            continue
        assert ns == list(range(ns[0], ns[-1] + 1)), (m, ns)
        for n in range(ns[0]):
            assert plans[n][1] <= m, (m, n, plans[n])
        for n in ns:
            assert plans[n][1] > m

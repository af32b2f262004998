"""Python binding of libattn.so (include/attn.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
builds the parameter structs from torch tensors (pointers, strides, sizes),
allocates outputs with torch on the tensors' device and passes the current
CUDA stream.  If the library is missing or a call fails, it raises: there is
no fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn.so")

# Constants of include/attn.h
PARAMS_VERSION = 3
BWD_DETERMINISTIC = 1
DTYPE_FP16, DTYPE_BF16 = 0, 1
WINDOW_INF = 2**31 - 1
CAUSAL_TOP_LEFT = -(2**31)
CAUSAL_BOTTOM_RIGHT = -(2**31) + 1
LSE_HT, LSE_TH = 0, 1
DIAGONAL_TOP_LEFT, DIAGONAL_BOTTOM_RIGHT = 0, 1
ERROR_INVALID_VALUE = 1
ERROR_NO_KERNEL_IMAGE = 209
ERROR_MEMORY_ALLOCATION = 2
STATIC_WORKSPACE_BYTES = 64 << 20


def varlen_mode(stacked: int, length: int, position: int) -> int:
    return (stacked & 1) | ((length & 3) << 1) | ((position & 3) << 3)


MODE_DENSE = varlen_mode(0, 0, 0)
MODE_PACKED = varlen_mode(1, 1, 1)
MODE_PADDED = varlen_mode(0, 2, 0)
MODE_PACKED_USED = varlen_mode(1, 2, 1)
MODE_PACKED_OFFSETS = varlen_mode(1, 2, 2)


def varlen_bits(qmode: int, kmode: int, lse_layout: int, diagonal: int) -> int:
    return (qmode & 0xFF) | ((kmode & 0xFF) << 8) | ((lse_layout & 3) << 16) | ((diagonal & 1) << 18)


_i64x3 = ctypes.c_int64 * 3


class FwdParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("version", ctypes.c_uint32), ("dtype", ctypes.c_int32),
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("Sq", ctypes.c_int32), ("Sk", ctypes.c_int32),
        ("D", ctypes.c_int32), ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("q_stride", _i64x3), ("k_stride", _i64x3), ("v_stride", _i64x3), ("o_stride", _i64x3),
        ("sm_scale", ctypes.c_float), ("window_left", ctypes.c_int32),
        ("window_right", ctypes.c_int32), ("varlen_bits", ctypes.c_uint32),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        # version 2
        ("seqused_q", ctypes.c_void_p), ("seqused_k", ctypes.c_void_p), ("Dv", ctypes.c_int32),
        ("dropout_p", ctypes.c_float), ("philox_seed", ctypes.c_uint64),
        ("philox_offset", ctypes.c_uint32), ("flags", ctypes.c_uint32),
        # version 3
        ("bias", ctypes.c_void_p), ("bias_stride", _i64x3),
    ]


class BwdParams(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("version", ctypes.c_uint32), ("dtype", ctypes.c_int32),
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("Sq", ctypes.c_int32), ("Sk", ctypes.c_int32),
        ("D", ctypes.c_int32), ("total_q", ctypes.c_int64), ("total_k", ctypes.c_int64),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("o", ctypes.c_void_p), ("dout", ctypes.c_void_p), ("lse", ctypes.c_void_p),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("q_stride", _i64x3), ("k_stride", _i64x3), ("v_stride", _i64x3), ("o_stride", _i64x3),
        ("do_stride", _i64x3), ("dq_stride", _i64x3), ("dk_stride", _i64x3), ("dv_stride", _i64x3),
        ("sm_scale", ctypes.c_float), ("window_left", ctypes.c_int32),
        ("window_right", ctypes.c_int32), ("varlen_bits", ctypes.c_uint32),
        ("cu_seqlens_q", ctypes.c_void_p), ("cu_seqlens_k", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("main_kernel_events", ctypes.c_void_p * 2),
        # version 2
        ("seqused_q", ctypes.c_void_p), ("seqused_k", ctypes.c_void_p), ("Dv", ctypes.c_int32),
        ("dropout_p", ctypes.c_float), ("philox_seed", ctypes.c_uint64),
        ("philox_offset", ctypes.c_uint32), ("flags", ctypes.c_uint32),
        # version 3
        ("bias", ctypes.c_void_p), ("dbias", ctypes.c_void_p),
        ("bias_stride", _i64x3), ("dbias_stride", _i64x3),
    ]


# Sizes of the older structs: version 1 ends before seqused_q, version 2
# before bias.
FWD_PARAMS_V1_SIZE = FwdParams.seqused_q.offset
BWD_PARAMS_V1_SIZE = BwdParams.seqused_q.offset
FWD_PARAMS_V2_SIZE = FwdParams.bias.offset
BWD_PARAMS_V2_SIZE = BwdParams.bias.offset


EXPORTS = {
    "attn_fwd": (ctypes.c_int, [ctypes.POINTER(FwdParams), ctypes.c_void_p]),
    "attn_bwd": (ctypes.c_int, [ctypes.POINTER(BwdParams), ctypes.c_void_p]),
    "attn_bwd_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(BwdParams)]),
    "attn_bwd_static_workspace": (ctypes.c_int, [ctypes.POINTER(BwdParams), ctypes.c_void_p]),
    "attn_allowed_pairs": (ctypes.c_int64, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_int32, ctypes.c_uint32]),
    "attn_tile_plan": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_uint32, ctypes.c_int32,
                                      ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                      ctypes.POINTER(ctypes.c_uint8)]),
    "attn_tile_plan_bwd": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_uint32, ctypes.c_int32,
                                          ctypes.POINTER(ctypes.c_int32),
                                          ctypes.POINTER(ctypes.c_int32)]),
    "attn_device_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint32)]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m scaled_dot_product_12_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class AttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned cudaError_t {code}")
        self.code = code


def _check(fn: str, code: int) -> None:
    if code != 0:
        raise AttnError(fn, code)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return DTYPE_FP16
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: fp16 or bf16 only")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _strides(t: torch.Tensor, packed: bool):
    if t.stride(-1) != 1:
        raise ValueError("the head dimension must be contiguous (stride 1)")
    s = t.stride()
    return _i64x3(0, s[1], s[0]) if packed else _i64x3(s[0], s[1], s[2])


def _stream_handle(device: torch.device, stream) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Problem:
    """Sizes, window and layout of one call, shared by forward and backward.

    Each side on its own: dense (4-D [B, H, S, D]), padded (4-D with
    ``seqlens``: B lengths), packed (3-D [T, H, D] with ``cu_seqlens``: B + 1
    cumulative lengths), packed with used lengths (``cu_seqlens`` as slots
    plus ``seqused``: B lengths) or packed at positions (``seqstart``: B
    start rows plus ``seqused``).
    """

    def __init__(self, q, k, sm_scale, window, bottom_right, cu_seqlens_q, cu_seqlens_k,
                 max_seqlen_q, max_seqlen_k, lse_layout, seqlens_q=None, seqlens_k=None,
                 seqused_q=None, seqused_k=None, seqstart_q=None, seqstart_k=None):
        sides = {}
        for name, cu, lens, used, start in (("q", cu_seqlens_q, seqlens_q, seqused_q, seqstart_q),
                                            ("k", cu_seqlens_k, seqlens_k, seqused_k, seqstart_k)):
            given = [x is not None for x in (cu, lens, start)]
            if sum(given) > 1:
                raise ValueError(f"{name}: give one of cu_seqlens, seqlens or seqstart")
            if used is not None and cu is None and start is None:
                raise ValueError(f"{name}: seqused needs cu_seqlens (slots) or seqstart (positions)")
            if start is not None and used is None:
                raise ValueError(f"{name}: seqstart needs seqused")
            if cu is not None:
                mode = MODE_PACKED_USED if used is not None else MODE_PACKED
                count, ptr = cu.numel() - 1, cu
            elif start is not None:
                mode, count, ptr = MODE_PACKED_OFFSETS, start.numel(), start
            elif lens is not None:
                mode, count, ptr = MODE_PADDED, lens.numel(), lens
            else:
                mode, count, ptr = MODE_DENSE, None, None
            if used is not None and used.numel() != count:
                raise ValueError(f"{name}: seqused needs one entry per sequence")
            sides[name] = (mode, count, ptr, used)
        (qmode, qcount, self.cu_q, self.used_q) = sides["q"]
        (kmode, kcount, self.cu_k, self.used_k) = sides["k"]
        self.q_packed, self.k_packed = bool(qmode & 1), bool(kmode & 1)
        self.q_padded, self.k_padded = qmode == MODE_PADDED, kmode == MODE_PADDED
        for name, packed, t in (("q", self.q_packed, q), ("k", self.k_packed, k)):
            if t.dim() != (3 if packed else 4):
                raise ValueError(f"{name}: packed inputs are [tokens, H, D], others [B, H, S, D]")
        sizes = set()
        for count in (qcount, kcount):
            if count is not None:
                sizes.add(count)
        if not self.q_packed:
            sizes.add(q.shape[0])
        if not self.k_packed:
            sizes.add(k.shape[0])
        if len(sizes) != 1:
            raise ValueError(f"inconsistent batch / sequence counts {sorted(sizes)}")
        self.B = sizes.pop()
        self.H, self.D = (q.shape[1], q.shape[2]) if self.q_packed else (q.shape[1], q.shape[3])
        if (self.q_packed and max_seqlen_q is None) or (self.k_packed and max_seqlen_k is None):
            raise ValueError("a packed side needs its max_seqlen")
        self.Sq = int(max_seqlen_q) if self.q_packed else q.shape[2]
        self.Sk = int(max_seqlen_k) if self.k_packed else k.shape[2]
        self.total_q = q.shape[0] if self.q_packed else 0
        self.total_k = k.shape[0] if self.k_packed else 0
        self.sm_scale = float(sm_scale) if sm_scale is not None else self.D ** -0.5
        self.window = (int(window[0]), int(window[1]))
        self.bottom_right = bool(bottom_right)
        self.lse_th = (lse_layout.upper() == "TH")
        self.bits = varlen_bits(qmode, kmode, LSE_TH if self.lse_th else LSE_HT,
                                DIAGONAL_BOTTOM_RIGHT if self.bottom_right else DIAGONAL_TOP_LEFT)
        self.dropout_p, self.philox_seed, self.philox_offset = 0.0, 0, 0
        self.flags = 0

    def lse_shape(self):
        if self.q_packed:
            return (self.total_q, self.H) if self.lse_th else (self.H, self.total_q)
        return (self.B, self.Sq, self.H) if self.lse_th else (self.B, self.H, self.Sq)

    def set_dropout(self, p, seed, offset):
        self.dropout_p, self.philox_seed, self.philox_offset = float(p), int(seed), int(offset)

    def fill(self, p, dtype_code):
        p.struct_size = ctypes.sizeof(p)
        p.version = PARAMS_VERSION
        p.dtype = dtype_code
        p.B, p.H, p.Sq, p.Sk, p.D = self.B, self.H, self.Sq, self.Sk, self.D
        p.total_q, p.total_k = self.total_q, self.total_k
        p.sm_scale = self.sm_scale
        p.window_left, p.window_right = self.window
        p.varlen_bits = self.bits
        p.cu_seqlens_q = _ptr(self.cu_q)
        p.cu_seqlens_k = _ptr(self.cu_k)
        p.seqused_q = _ptr(self.used_q)
        p.seqused_k = _ptr(self.used_k)
        p.dropout_p = self.dropout_p
        p.philox_seed = self.philox_seed & (2**64 - 1)
        p.philox_offset = self.philox_offset & 0xFFFFFFFF
        p.flags = self.flags


def _bias_strides(t: Optional[torch.Tensor], q: torch.Tensor, name: str):
    """Strides of a [B, H, Sq, Sk] bias (or its gradient), checked for shape
    rank, dtype and a contiguous key dimension; the library checks the rest."""
    if t is None:
        return _i64x3(0, 0, 0)
    if t.dim() != 4:
        raise ValueError(f"{name}: a [B, H, Sq, Sk] tensor is expected")
    if t.dtype != q.dtype:
        raise ValueError(f"{name}: dtype {t.dtype} differs from q's {q.dtype}")
    if t.shape[3] > 1 and t.stride(3) != 1:
        raise ValueError(f"{name}: the key dimension must be contiguous")
    s = t.stride()
    return _i64x3(s[0] if t.shape[0] > 1 else 0, s[1] if t.shape[1] > 1 else 0,
                  s[2] if t.shape[2] > 1 else 0)


def forward(q, k, v, sm_scale=None, window=(WINDOW_INF, WINDOW_INF), bottom_right=False,
            cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None, max_seqlen_k=None,
            lse_layout="HT", out=None, lse=None, return_lse=True, stream=None,
            seqlens_q=None, seqlens_k=None, seqused_q=None, seqused_k=None, seqstart_q=None,
            seqstart_k=None, dropout_p=0.0, philox_seed=0,
            philox_offset=0, bias=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """O (and LSE) of FlashAttention through attn_fwd.

    Dense: q [B,H,Sq,D], k/v [B,H,Sk,D].  Packed: q [Tq,H,D], k/v [Tk,H,D] with
    int32 cu_seqlens on the device and the largest sequence lengths; with
    seqused as well, sequence b uses the first seqused[b] rows of its slot;
    seqstart (B start rows) with seqused places the sequences anywhere in the
    packed tensor.  Padded: dense shapes plus int32 seqlens_q / seqlens_k [B]
    on the device.  Rows outside every sequence are left untouched.  dropout_p
    > 0 drops elements of P with the Philox generator keyed by philox_seed.
    ``bias`` [B, H, Sq, Sk] (q's dtype; batch and head may be broadcast with
    ``expand``) is added to the scaled scores, (i, j) counted within each
    sequence.
    """
    pr = Problem(q, k, sm_scale, window, bottom_right, cu_seqlens_q, cu_seqlens_k,
                 max_seqlen_q, max_seqlen_k, lse_layout, seqlens_q, seqlens_k, seqused_q,
                 seqused_k, seqstart_q, seqstart_k)
    pr.set_dropout(dropout_p, philox_seed, philox_offset)
    if out is None:
        out = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=q.device)
    if lse is None and return_lse:
        lse = torch.empty(pr.lse_shape(), dtype=torch.float32, device=q.device)
    p = FwdParams()
    pr.fill(p, _dtype_code(q))
    p.q, p.k, p.v, p.o, p.lse = _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse)
    p.Dv = v.shape[-1]
    p.q_stride = _strides(q, pr.q_packed)
    p.k_stride = _strides(k, pr.k_packed)
    p.v_stride = _strides(v, pr.k_packed)
    p.o_stride = _strides(out, pr.q_packed)
    p.bias, p.bias_stride = _ptr(bias), _bias_strides(bias, q, "bias")
    _check("attn_fwd", lib().attn_fwd(ctypes.byref(p), _stream_handle(q.device, stream)))
    return out, lse


def bwd_params(dout, q, k, v, o, lse, pr: Problem, dq, dk, dv, workspace=None, bias=None,
               dbias=None) -> BwdParams:
    p = BwdParams()
    pr.fill(p, _dtype_code(q))
    p.q, p.k, p.v, p.o, p.dout, p.lse = _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse)
    p.dq, p.dk, p.dv = _ptr(dq), _ptr(dk), _ptr(dv)
    p.Dv = v.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", dout), ("dq", dq), ("dk", dk),
                    ("dv", dv)):
        setattr(p, name + "_stride", _strides(t, pr.k_packed if name in ("k", "v", "dk", "dv")
                                              else pr.q_packed))
    p.bias, p.bias_stride = _ptr(bias), _bias_strides(bias, q, "bias")
    p.dbias, p.dbias_stride = _ptr(dbias), _bias_strides(dbias, q, "dbias")
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    return p


def workspace_bytes(p: BwdParams) -> int:
    return int(lib().attn_bwd_workspace_size(ctypes.byref(p)))


def backward(dout, q, k, v, o, lse, sm_scale=None, window=(WINDOW_INF, WINDOW_INF),
             bottom_right=False, cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None,
             max_seqlen_k=None, lse_layout="HT", dq=None, dk=None, dv=None, workspace=None,
             stream=None, seqlens_q=None, seqlens_k=None, seqused_q=None, seqused_k=None,
             seqstart_q=None, seqstart_k=None, dropout_p=0.0, philox_seed=0, philox_offset=0,
             deterministic=False, bias=None, dbias=None):
    """(dQ, dK, dV) through attn_bwd; the workspace is allocated if not given.
    ``deterministic`` adds the dQ contributions in a fixed order.  ``bias`` is
    the forward's bias; ``dbias`` (a [B, H, Sq, Sk] tensor, not broadcast)
    receives the gradient with respect to the bias."""
    pr = Problem(q, k, sm_scale, window, bottom_right, cu_seqlens_q, cu_seqlens_k,
                 max_seqlen_q, max_seqlen_k, lse_layout, seqlens_q, seqlens_k, seqused_q,
                 seqused_k, seqstart_q, seqstart_k)
    pr.set_dropout(dropout_p, philox_seed, philox_offset)
    pr.flags = BWD_DETERMINISTIC if deterministic else 0
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    p = bwd_params(dout, q, k, v, o, lse, pr, dq, dk, dv, bias=bias, dbias=dbias)
    need = workspace_bytes(p)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    p.workspace = workspace.data_ptr()
    p.workspace_bytes = workspace.numel() * workspace.element_size()
    _check("attn_bwd", lib().attn_bwd(ctypes.byref(p), _stream_handle(q.device, stream)))
    return dq, dk, dv, workspace


def allowed_pairs(seqlen_q: int, seqlen_k: int, window_left: int, window_right: int,
                  bottom_right: bool) -> int:
    return int(lib().attn_allowed_pairs(seqlen_q, seqlen_k, window_left, window_right,
                                        1 if bottom_right else 0))


def tile_plan(seqlen_q, seqlen_k, window_left, window_right, bottom_right, m0):
    nb, ne = ctypes.c_int32(), ctypes.c_int32()
    buf = (ctypes.c_uint8 * max(1, (seqlen_k + 127) // 128))()
    _check("attn_tile_plan", lib().attn_tile_plan(seqlen_q, seqlen_k, window_left, window_right,
                                                  1 if bottom_right else 0, m0,
                                                  ctypes.byref(nb), ctypes.byref(ne), buf))
    return nb.value, ne.value, [buf[i] for i in range(max(0, ne.value - nb.value))]


def tile_plan_bwd(seqlen_q, seqlen_k, window_left, window_right, bottom_right, n0):
    mb, me = ctypes.c_int32(), ctypes.c_int32()
    _check("attn_tile_plan_bwd", lib().attn_tile_plan_bwd(seqlen_q, seqlen_k, window_left,
                                                          window_right, 1 if bottom_right else 0,
                                                          n0, ctypes.byref(mb), ctypes.byref(me)))
    return mb.value, me.value


def device_status(device=None, stream=None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_uint32()
    _check("attn_device_status", lib().attn_device_status(_stream_handle(dev, stream),
                                                          ctypes.byref(st)))
    return st.value

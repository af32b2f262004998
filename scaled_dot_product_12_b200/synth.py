"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws numbers and names
shapes, so the tests, the benchmark and the fp64 oracle can all be fed the same
tensors.  Values are i.i.d. N(0, 1) drawn in fp32 on the CPU from
``torch.Generator().manual_seed(seed)`` and rounded to the compute dtype
(round-to-nearest-even by ``Tensor.to``).

The shapes stand in for the regression workloads the AOTriton 0.15b release
notes time (github.com releases, section "Performance Regression Fixes":
roberta-large, bert-large-uncased, gpt2, LTX at 6630 / 15300 and hdim 128 at
8192) plus the packed variable-length case of the 0.14b notes ("VarlenBits
supersedes VarlenType").  No dataset is involved.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch

# Window encodings of include/attn.h (kept in step by tests/test_abi.py).
WINDOW_INF = 2**31 - 1
CAUSAL_TOP_LEFT = -(2**31)
CAUSAL_BOTTOM_RIGHT = -(2**31) + 1

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


def normal(shape, seed: int, dtype=torch.bfloat16, generator: Optional[torch.Generator] = None):
    """i.i.d. N(0,1) in fp32 on the CPU, rounded to ``dtype``."""
    g = generator if generator is not None else torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)


def qkv_do(q_shape, k_shape, seed: int, dtype=torch.bfloat16, dv: Optional[int] = None):
    """Q, K, V, dO drawn in that order from one generator seeded with ``seed``."""
    g = torch.Generator().manual_seed(seed)
    v_shape = tuple(k_shape[:-1]) + ((dv if dv is not None else k_shape[-1]),)
    do_shape = tuple(q_shape[:-1]) + (v_shape[-1],)
    q = normal(q_shape, seed, dtype, g)
    k = normal(k_shape, seed, dtype, g)
    v = normal(v_shape, seed, dtype, g)
    do = normal(do_shape, seed, dtype, g)
    return q, k, v, do


def bias(shape, seed: int, dtype=torch.bfloat16, std: float = 1.0):
    """An additive attention bias: i.i.d. N(0, std^2) drawn in fp32 on the CPU
    from its own generator, rounded to ``dtype``."""
    return (normal(shape, seed, torch.float32) * std).to(dtype)


def varlen_seqlens(seed: int, n_seqs: int = 16, max_q: int = 4096, max_extra_k: int = 512):
    """seqlen_q ~ U[1, max_q], seqlen_k = seqlen_q + U[0, max_extra_k] (int64 lists)."""
    g = torch.Generator().manual_seed(seed)
    sq = torch.randint(1, max_q + 1, (n_seqs,), generator=g)
    sk = sq + torch.randint(0, max_extra_k + 1, (n_seqs,), generator=g)
    return sq.tolist(), sk.tolist()


def cumsum0(lengths):
    """[0, l0, l0+l1, ...] as int32 (the cu_seqlens layout)."""
    out = [0]
    for x in lengths:
        out.append(out[-1] + int(x))
    return torch.tensor(out, dtype=torch.int32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str
    B: int
    H: int
    Sq: int
    Sk: int
    D: int
    window_left: int
    window_right: int
    bottom_right: bool
    seed: int
    packed: bool = False
    lse_th: bool = False
    describe: str = ""


NO_MASK = (WINDOW_INF, WINDOW_INF)

WORKLOADS = {
    "tiny_causal": Workload("tiny_causal", "fp16", 1, 2, 128, 128, 64, WINDOW_INF, 0, False, 1,
                            describe="tiny causal MHA, fp16 B1 H2 S128 D64, causal top-left"),
    "bert_large": Workload("bert_large", "bf16", 192, 16, 512, 512, 64, *NO_MASK, False, 2,
                           describe="BERT-large shape, bf16 B192 H16 S512 D64, no mask"),
    "roberta_large": Workload("roberta_large", "bf16", 512, 16, 384, 384, 64, *NO_MASK, False, 3,
                              describe="roberta-large shape, bf16 B512 H16 S384 D64, no mask"),
    "gpt2": Workload("gpt2", "fp16", 72, 12, 1024, 1024, 64, WINDOW_INF, 0, False, 4,
                     describe="GPT-2 shape, fp16 B72 H12 S1024 D64, causal top-left"),
    "ltx_6630": Workload("ltx_6630", "bf16", 1, 32, 6630, 6630, 128, *NO_MASK, False, 5,
                         describe="LTX diffusion shape, bf16 B1 H32 S6630 D128, no mask"),
    "ltx_15300": Workload("ltx_15300", "bf16", 1, 32, 15300, 15300, 128, *NO_MASK, False, 6,
                          describe="LTX diffusion shape, bf16 B1 H32 S15300 D128, no mask"),
    "long_8192": Workload("long_8192", "bf16", 1, 16, 8192, 8192, 128, *NO_MASK, False, 7,
                          describe="long sequence, bf16 B1 H16 S8192 D128, no mask"),
}

# Packed variable-length cases: 16 sequences, seqlens from seed 8, windows
# (256, 0), (-64, 128) and both causal sentinels, each under both diagonals.
VARLEN_SEQLEN_SEED = 8
VARLEN_WINDOWS = [
    (256, 0),
    (-64, 128),
    (CAUSAL_TOP_LEFT, 0),
    (CAUSAL_BOTTOM_RIGHT, 0),
]


def varlen_cases(dims=(128, 48, 80)):
    """(name, D, window_left, window_right, bottom_right, seed) of every packed case."""
    cases = []
    k = 0
    for D in dims:
        for wl, wr in VARLEN_WINDOWS:
            for br in (False, True):
                tag = {CAUSAL_TOP_LEFT: "causalTL", CAUSAL_BOTTOM_RIGHT: "causalBR"}.get(wl, f"w{wl}_{wr}")
                cases.append((f"varlen_D{D}_{tag}_{'BR' if br else 'TL'}", D, wl, wr, br, 9 + k))
                k += 1
    return cases


def varlen_workloads(dims=(128,)):
    """The packed cases as named workloads: 16 sequences (lengths from
    VARLEN_SEQLEN_SEED), H = 16, bf16, LSE in TH layout; Sq / Sk hold the
    largest seqlen_q / seqlen_k."""
    sq, sk = varlen_seqlens(VARLEN_SEQLEN_SEED)
    out = {}
    for name, D, wl, wr, br, seed in varlen_cases(dims):
        win = {CAUSAL_TOP_LEFT: "causal top-left sentinel",
               CAUSAL_BOTTOM_RIGHT: "causal bottom-right sentinel"}.get(wl, f"window ({wl}, {wr})")
        out[name] = Workload(name, "bf16", len(sq), 16, max(sq), max(sk), D, wl, wr, br, seed,
                             packed=True, lse_th=True,
                             describe=(f"packed 1THD varlen, bf16 16 seqs (seqlen_q ~ U[1,4096], "
                                       f"seqlen_k = seqlen_q + U[0,512]) H16 D{D}, {win}, "
                                       f"{'bottom-right' if br else 'top-left'} diagonal, LSE TH"))
    return out


VARLEN_WORKLOADS = varlen_workloads()
ALL_WORKLOADS = {**WORKLOADS, **VARLEN_WORKLOADS}

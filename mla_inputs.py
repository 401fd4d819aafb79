"""Seeded synthetic inputs for absorbed-form MLA decode.

Shared by the tests, the smoke check and the benchmark, for both the GPU
library and the CPU oracle.  This module draws random numbers and lays out
pages; it holds none of the attention arithmetic.

Recipe (torch CPU generator, ``manual_seed(seed)``, draws in this order):
  1. per-sequence lengths, when the workload draws them: uniform integers in
     [lo, hi] inclusive (``torch.randint``);
  2. outlier channels, when the workload has them: ``randperm(512)[:count]``;
  3. q: ``randn(B, s_q, H, 576)`` in fp32;
  4. the cache: one ``randn(64, 576)`` page per physical block, in block
     order, drawn in chunks of 1024 pages;
  5. the page permutation (shuffled tables only): ``randperm(num_blocks)``.
Outlier channels are latent columns (so V carries them too): they are
multiplied by the factor in fp32, in q and in every cache row, before the
values are rounded to bf16 (round to nearest even, the torch conversion).
Page tables: sequence b owns ceil(L_b / 64) pages.  "identity" gives sequence b
the consecutive physical blocks that follow sequence b-1's; "shuffled" hands
out the same slices of a random permutation of the physical blocks.  Unused
table entries are -1.  Cache rows past a sequence's length, in its last page,
are randn like the rest unless ``tail_fill`` replaces them (NaN in tests, to
show they never reach the result).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Sequence

import torch

D_QK = 576
D_V = 512
PAGE = 64
DEFAULT_SCALE = 1.0 / math.sqrt(192.0)


@dataclass(frozen=True)
class Workload:
    """One decode call's shape and input distribution."""
    name: str
    B: int
    s_q: int
    H: int
    seqlen: int = 0                      # fixed length for every sequence
    seqlen_range: Optional[tuple] = None  # (lo, hi) inclusive, drawn per sequence
    seqlens: Optional[tuple] = None      # explicit per-sequence lengths
    table: str = "shuffled"              # "identity" or "shuffled"
    outliers: int = 0                    # number of latent channels scaled up
    outlier_factor: float = 20.0
    scale: float = DEFAULT_SCALE
    extra_table_cols: int = 0            # unused (-1) columns appended to the table


# The five decode workloads, named by what they are.
WORKLOADS: Dict[str, Workload] = {
    "b1_h16_l1k_identity": Workload("b1_h16_l1k_identity", B=1, s_q=1, H=16, seqlen=1024,
                                    table="identity"),
    "b16_h16_l4k": Workload("b16_h16_l4k", B=16, s_q=1, H=16, seqlen=4096),
    "b32_sq2_h16_l16k_outliers": Workload("b32_sq2_h16_l16k_outliers", B=32, s_q=2, H=16,
                                          seqlen=16384, outliers=4),
    "b64_h128_lvar1k32k": Workload("b64_h128_lvar1k32k", B=64, s_q=1, H=128,
                                   seqlen_range=(1024, 32768)),
    "b8_h16_l64k": Workload("b8_h16_l64k", B=8, s_q=1, H=16, seqlen=65536),
}

HEADLINE = "b8_h16_l64k"


def workload(name: str, **overrides) -> Workload:
    return replace(WORKLOADS[name], **overrides) if overrides else WORKLOADS[name]


def pages_for(L: int) -> int:
    return (L + PAGE - 1) // PAGE


@dataclass
class Inputs:
    """CPU tensors of one decode call."""
    q: torch.Tensor              # [B, s_q, H, 576] bf16
    kv_cache: torch.Tensor       # [num_blocks, 64, 576] bf16
    block_table: torch.Tensor    # [B, max_blocks] int32
    cache_seqlens: torch.Tensor  # [B] int32
    scale: float
    outlier_channels: List[int] = field(default_factory=list)

    @property
    def B(self) -> int:
        return self.q.shape[0]

    @property
    def s_q(self) -> int:
        return self.q.shape[1]

    @property
    def H(self) -> int:
        return self.q.shape[2]


def _lengths(w: Workload, g: torch.Generator) -> List[int]:
    if w.seqlens is not None:
        assert len(w.seqlens) == w.B
        return [int(x) for x in w.seqlens]
    if w.seqlen_range is not None:
        lo, hi = w.seqlen_range
        return [int(x) for x in torch.randint(lo, hi + 1, (w.B,), generator=g)]
    return [w.seqlen] * w.B


def make_inputs(w: Workload, seed: int = 0, tail_fill: Optional[float] = None) -> Inputs:
    g = torch.Generator().manual_seed(seed)
    lengths = _lengths(w, g)
    outlier_channels: List[int] = []
    if w.outliers:
        outlier_channels = sorted(int(x) for x in torch.randperm(D_V, generator=g)[: w.outliers])
    idx = torch.tensor(outlier_channels, dtype=torch.long)

    q32 = torch.randn(w.B, w.s_q, w.H, D_QK, generator=g)
    if w.outliers:
        q32[..., idx] *= w.outlier_factor
    q = q32.to(torch.bfloat16)

    n_pages = [pages_for(L) for L in lengths]
    num_blocks = max(1, sum(n_pages))
    kv = torch.empty(num_blocks, PAGE, D_QK, dtype=torch.bfloat16)
    chunk = 1024
    for c0 in range(0, num_blocks, chunk):
        c1 = min(num_blocks, c0 + chunk)
        t = torch.randn(c1 - c0, PAGE, D_QK, generator=g)
        if w.outliers:
            t[..., idx] *= w.outlier_factor
        kv[c0:c1] = t.to(torch.bfloat16)

    if w.table == "shuffled":
        perm = torch.randperm(num_blocks, generator=g)
    elif w.table == "identity":
        perm = torch.arange(num_blocks)
    else:
        raise ValueError(f"unknown table kind {w.table!r}")

    max_blocks = max(1, max(n_pages) if n_pages else 1) + w.extra_table_cols
    table = torch.full((w.B, max_blocks), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[off: off + n].to(torch.int32)
        off += n

    if tail_fill is not None:
        for b, L in enumerate(lengths):
            if L % PAGE:
                last = int(table[b, L // PAGE])
                kv[last, L % PAGE:, :] = tail_fill

    return Inputs(q=q, kv_cache=kv, block_table=table,
                  cache_seqlens=torch.tensor(lengths, dtype=torch.int32),
                  scale=w.scale, outlier_channels=outlier_channels)


def small(B: int, s_q: int, H: int, seqlens: Sequence[int], table: str = "shuffled",
          scale: float = DEFAULT_SCALE, outliers: int = 0, extra_table_cols: int = 0,
          seed: int = 0, tail_fill: Optional[float] = None) -> Inputs:
    """Ad-hoc inputs for tests (explicit lengths, same recipe)."""
    w = Workload(name="adhoc", B=B, s_q=s_q, H=H, seqlens=tuple(int(x) for x in seqlens),
                 table=table, scale=scale, outliers=outliers, extra_table_cols=extra_table_cols)
    return make_inputs(w, seed=seed, tail_fill=tail_fill)


@dataclass
class Fp8Cache:
    """An e4m3 cache with one fp32 scale per cached token (CPU tensors)."""
    codes: torch.Tensor  # [num_blocks, 64, 576] uint8: e4m3 bit patterns
    scale: torch.Tensor  # [num_blocks, 64] fp32


def fp8_cache(num_blocks: int, seed: int = 0, pow2_scales: bool = False) -> Fp8Cache:
    """Seeded random e4m3 cache, drawn field by field rather than rounded from
    real values: sign bits uniform; exponent fields round(N(7, 1.5)) clipped to
    [0, 14] (magnitudes around 1, subnormals included, no NaN); mantissa fields
    uniform on 0..7.  Token scales are 2^k, k uniform on {-3, -2, -1}, with
    ``pow2_scales``, else uniform on [0.05, 0.3).  Draw order: signs,
    exponents, mantissas, scales."""
    g = torch.Generator().manual_seed(seed)
    shape = (num_blocks, PAGE, D_QK)
    sign = torch.randint(0, 2, shape, generator=g)
    expo = torch.round(torch.randn(shape, generator=g) * 1.5 + 7.0).clamp(0, 14).to(torch.int64)
    mant = torch.randint(0, 8, shape, generator=g)
    codes = ((sign << 7) | (expo << 3) | mant).to(torch.uint8)
    if pow2_scales:
        scale = torch.exp2(torch.randint(-3, 0, (num_blocks, PAGE), generator=g).to(torch.float32))
    else:
        scale = 0.05 + 0.25 * torch.rand(num_blocks, PAGE, generator=g)
    return Fp8Cache(codes=codes, scale=scale.to(torch.float32))


def algorithmic_bytes(inp: Inputs) -> int:
    """Bytes a decode call must move at minimum: every visible cache row once
    (shared by all heads and query positions), q, out (bf16), lse (fp32) and
    the page-table entries in use."""
    B, s_q, H = inp.B, inp.s_q, inp.H
    Ls = [int(x) for x in inp.cache_seqlens]
    kv = sum(Ls) * D_QK * 2
    q = B * s_q * H * D_QK * 2
    out = B * s_q * H * D_V * 2
    lse = B * s_q * H * 4
    table = sum(pages_for(L) for L in Ls) * 4 + B * 4
    return kv + q + out + lse + table


def algorithmic_flops(inp: Inputs) -> int:
    """2 * H * s_q * L * (576 + 512) summed over sequences."""
    return sum(2 * inp.H * inp.s_q * int(L) * (D_QK + D_V) for L in inp.cache_seqlens)


# ------------------------------------------------- non-absorbed form inputs
D_NOPE = 128   # decompressed key / value width per head
D_ROPE = 64    # rope columns, the last 64 of a cached latent row


@dataclass
class NaiveInputs:
    """Extra inputs of the non-absorbed form over the same latent cache: the
    queries in the decompressed space and the per-head up-projections."""
    q: torch.Tensor     # [B, s_q, H, 192] bf16: 128 key columns, then 64 rope
    w_uk: torch.Tensor  # [H, 128, 512] bf16: row e of head h = latent coefficients of key dim e
    w_uv: torch.Tensor  # [H, 128, 512] bf16: the same for value dim e


def naive_inputs(B: int, s_q: int, H: int, seed: int = 0) -> NaiveInputs:
    """Seeded queries and up-projection matrices (torch CPU generator, drawn in
    the order q, w_uk, w_uv): q ~ N(0, 1); the matrices ~ N(0, 1/512), so a
    decompressed key or value of an N(0, 1) latent row is again about N(0, 1).
    Every value is drawn in fp32 and rounded to bf16."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, s_q, H, D_NOPE + D_ROPE, generator=g).to(torch.bfloat16)
    w_uk = (torch.randn(H, D_NOPE, D_V, generator=g) / math.sqrt(D_V)).to(torch.bfloat16)
    w_uv = (torch.randn(H, D_NOPE, D_V, generator=g) / math.sqrt(D_V)).to(torch.bfloat16)
    return NaiveInputs(q=q, w_uk=w_uk, w_uv=w_uv)


def naive_algorithmic_flops(inp: Inputs) -> int:
    """FLOPs of the non-absorbed form per call: per visible token and head the
    two up-projections (2 x 2 x 512 x 128), then the 192-wide score and the
    128-wide value accumulation per query position."""
    H, s_q = inp.H, inp.s_q
    tokens = sum(int(L) for L in inp.cache_seqlens)
    return tokens * H * (2 * 2 * D_V * D_NOPE + s_q * 2 * (D_NOPE + D_ROPE + D_NOPE))

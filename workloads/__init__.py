"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the CUDA path (tests, bench, smoke) and the
float64 oracle consume the tensors produced here, so that both sides see
bit-identical inputs.

Recipe (one ``torch.Generator`` per call, seeded by the caller):

* prefill: q, k, v drawn in that order, fp32 N(0, 1), cast round-to-nearest-even
  to bf16, contiguous ``[B, H, L, D]`` (v ``[B, H, L, Dv]`` where the value
  width differs) (the ``(batch, num_heads, seqlen,
  head_dim)`` layout of the HF-Llama ``view(...).transpose(1, 2)`` code on the
  zeeklog page "LLM 中的 Attention 实现及优化", GQA section).
* FP8 prefill: the same fp32 draws, each tensor quantised to ``float8_e4m3fn``
  with one per-tensor scale ``s = amax(|x|) / 448`` (the largest finite e4m3
  value), ``x8 = cast(x / s)``.  This is the input preparation of the
  long-context FP8 workload; the kernel and the oracle both receive ``x8`` and
  ``s``.
* FP8 e5m2 prefill: the same draws quantised to ``float8_e5m2`` with
  ``s = amax(|x|) / 57344`` (the largest finite e5m2 value).
* paged decode: q ``[B, Hq, D]``, then per-sequence lengths uniform in
  ``[len_lo, len_hi]`` (so that the pool can be sized from them), then the K
  pool, then the V pool (pools are ``[num_pages, page_size, Hkv, D]``), then a
  random permutation of page ids that becomes the block table
  (``int32 [B, max_pages]``, unused slots 0).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

FP8_E4M3_MAX = 448.0
FP8_E5M2_MAX = 57344.0
PAGE_SIZE = 16


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    D: int
    causal: bool
    window: int = 0          # 0 = no window
    fp8: bool = False
    Dv: int = 0              # value width; 0 = D (queries and keys have width D)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def dv(self) -> int:
        return self.Dv or self.D


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    len_lo: int
    len_hi: int
    page_size: int = PAGE_SIZE
    Dv: int = 0              # value width; 0 = D (queries and keys have width D)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def dv(self) -> int:
        return self.Dv or self.D


# The five workloads of the build, indexed 0..4.  The seed of workload i is
# 1000 + i.
TINY_MHA = PrefillShape("tiny_mha_L128_D64", B=1, Hq=2, Hkv=2, Lq=128, Lk=128, D=64, causal=False)
GQA_CAUSAL = PrefillShape("gqa_causal_B4_H32_G4_L4096_D128", B=4, Hq=32, Hkv=8, Lq=4096, Lk=4096, D=128, causal=True)
MQA_DECODE = DecodeShape("mqa_paged_decode_B64_H32_Hkv1_D128_len512_8192", B=64, Hq=32, Hkv=1, D=128, len_lo=512, len_hi=8192)
SWA_CAUSAL = PrefillShape("swa_causal_B2_H32_G4_L16384_W4096_D128", B=2, Hq=32, Hkv=8, Lq=16384, Lk=16384, D=128, causal=True, window=4096)
FP8_CAUSAL = PrefillShape("fp8_causal_B1_H32_L32768_D128", B=1, Hq=32, Hkv=32, Lq=32768, Lk=32768, D=128, causal=True, fp8=True)

WORKLOADS = [TINY_MHA, GQA_CAUSAL, MQA_DECODE, SWA_CAUSAL, FP8_CAUSAL]

# Latent-space shapes (queries and keys of width 64-256, values of their own
# width: the latent projection of the Flash MLA page, §2.1), measured beside
# the five workloads above with the seeds of workloads 1 and 3.
LATENT_192_128 = PrefillShape("latent_causal_B4_H32_G4_L4096_Dqk192_Dv128", B=4, Hq=32, Hkv=8, Lq=4096, Lk=4096,
                              D=192, causal=True, Dv=128)
LATENT_256 = PrefillShape("latent_causal_B4_H32_G4_L4096_D256", B=4, Hq=32, Hkv=8, Lq=4096, Lk=4096, D=256,
                          causal=True)


def seed_of(index: int) -> int:
    return 1000 + index


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _normal(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def prefill_inputs(shape: PrefillShape, seed: int):
    """bf16 q, k, v on the host, contiguous [B, H, L, D]."""
    g = _gen(seed)
    q = _normal(g, (shape.B, shape.Hq, shape.Lq, shape.D)).to(torch.bfloat16)
    k = _normal(g, (shape.B, shape.Hkv, shape.Lk, shape.D)).to(torch.bfloat16)
    v = _normal(g, (shape.B, shape.Hkv, shape.Lk, shape.dv)).to(torch.bfloat16)
    return q, k, v


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor e4m3 quantisation of an fp32 tensor: (x8, scale).

    ``scale = amax/448`` in fp32 and ``x8 = float8_e4m3fn(x / scale)`` (torch's
    round-to-nearest-even cast; |x/scale| <= 448 so nothing saturates).
    """
    amax = x.abs().max().to(torch.float32)
    scale = (amax / FP8_E4M3_MAX).item() if amax > 0 else 1.0
    x8 = (x / scale).to(torch.float8_e4m3fn)
    return x8, float(scale)


def quantize_e5m2(x: torch.Tensor):
    """Per-tensor e5m2 quantisation of an fp32 tensor: (x8, scale), with
    ``scale = amax/57344`` (the largest finite e5m2 value) and torch's
    round-to-nearest-even cast to ``float8_e5m2``."""
    amax = x.abs().max().to(torch.float32)
    scale = (amax / FP8_E5M2_MAX).item() if amax > 0 else 1.0
    x8 = (x / scale).to(torch.float8_e5m2)
    return x8, float(scale)


def prefill_inputs_fp8(shape: PrefillShape, seed: int, fmt: str = "e4m3"):
    """(q8, k8, v8, q_scale, k_scale, v_scale); tensors float8_e4m3fn (or,
    with ``fmt="e5m2"``, float8_e5m2) [B, H, L, D], from the same fp32 draws
    as ``prefill_inputs``."""
    g = _gen(seed)
    q = _normal(g, (shape.B, shape.Hq, shape.Lq, shape.D))
    k = _normal(g, (shape.B, shape.Hkv, shape.Lk, shape.D))
    v = _normal(g, (shape.B, shape.Hkv, shape.Lk, shape.D))
    quant = {"e4m3": quantize_e4m3, "e5m2": quantize_e5m2}[fmt]
    q8, sq = quant(q)
    k8, sk = quant(k)
    v8, sv = quant(v)
    return q8, k8, v8, sq, sk, sv


@dataclasses.dataclass
class PagedKV:
    q: torch.Tensor            # [B, Hq, D] bf16
    k_pages: torch.Tensor      # [num_pages, page_size, Hkv, D] bf16
    v_pages: torch.Tensor      # [num_pages, page_size, Hkv, Dv] bf16
    block_table: torch.Tensor  # [B, max_pages] int32
    seq_lens: torch.Tensor     # [B] int32

    @property
    def num_pages(self) -> int:
        return int(self.k_pages.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])


def decode_inputs(shape: DecodeShape, seed: int, seq_lens: Optional[list] = None,
                  extra_pages: int = 0) -> PagedKV:
    """Paged decode inputs.  ``seq_lens`` overrides the drawn lengths (edge
    cases); the pool holds exactly the pages the sequences need plus
    ``extra_pages`` unused ones, in a random order."""
    g = _gen(seed)
    ps = shape.page_size
    q = _normal(g, (shape.B, shape.Hq, shape.D)).to(torch.bfloat16)
    if seq_lens is None:
        # lengths are drawn before the pools are sized, but after q; the pools
        # are drawn afterwards so that their size can follow the lengths.
        lens = torch.randint(shape.len_lo, shape.len_hi + 1, (shape.B,), generator=g, dtype=torch.int64)
    else:
        assert len(seq_lens) == shape.B
        lens = torch.tensor(seq_lens, dtype=torch.int64)
    pages_per_seq = [(int(n) + ps - 1) // ps for n in lens]
    max_pages = max(1, max(pages_per_seq) if pages_per_seq else 1)
    need = sum(pages_per_seq)
    num_pages = max(1, need + extra_pages)
    k_pages = _normal(g, (num_pages, ps, shape.Hkv, shape.D)).to(torch.bfloat16)
    v_pages = _normal(g, (num_pages, ps, shape.Hkv, shape.dv)).to(torch.bfloat16)
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    table = torch.zeros((shape.B, max_pages), dtype=torch.int32)
    cursor = 0
    for b, npg in enumerate(pages_per_seq):
        table[b, :npg] = perm[cursor:cursor + npg]
        cursor += npg
    return PagedKV(q=q, k_pages=k_pages, v_pages=v_pages, block_table=table,
                   seq_lens=lens.to(torch.int32))


def decode_queries(shape: DecodeShape, q_len: int, seed: int) -> torch.Tensor:
    """Queries of a q_len-token decode (the last q_len cached tokens of each
    sequence), [B, Hq, q_len, D] bf16, N(0,1) from their own seed."""
    g = _gen(seed)
    return _normal(g, (shape.B, shape.Hq, q_len, shape.D)).to(torch.bfloat16)

"""Work accounting for the measured metric: required FLOPs and algorithmic
HBM bytes of each workload.  Used by the benchmark to turn times into TFLOP/s
and GB/s; neither the kernels nor the oracle use it."""
from __future__ import annotations

import torch

from . import DecodeShape, PrefillShape


def prefill_flops(shape: PrefillShape) -> float:
    """FLOPs as actually required: 2*D + 2*Dv per visible (query, key) pair
    per head (2*D for Q.K^T, 2*Dv for P.V; 4*D when the widths agree)."""
    return 2.0 * (shape.D + shape.dv) * shape.B * shape.Hq * visible_pairs(shape.Lq, shape.Lk, shape.causal,
                                                                          shape.window)


def visible_pairs(Lq: int, Lk: int, causal: bool, window: int) -> int:
    """Number of (query, key) pairs a causal/window mask lets through.
    Counting only: bottom-right aligned causal, window of W keys incl. self."""
    if not causal:
        return Lq * Lk
    total = 0
    off = Lk - Lq
    # closed form per row would do, but a vectorised count keeps this obvious
    i = torch.arange(Lq, dtype=torch.int64)
    hi = torch.clamp(i + off + 1, 0, Lk)
    lo = torch.clamp(hi - window, min=0) if window > 0 else torch.zeros_like(hi)
    total = int((hi - lo).clamp(min=0).sum())
    return total


def prefill_bytes(shape: PrefillShape) -> float:
    """Algorithmic HBM bytes: read Q, K, V once, write O and LSE once."""
    el = 1 if shape.fp8 else 2
    q = shape.B * shape.Hq * shape.Lq * shape.D * el
    kv = shape.B * shape.Hkv * shape.Lk * (shape.D + shape.dv) * el
    o = shape.B * shape.Hq * shape.Lq * shape.dv * 2
    lse = shape.B * shape.Hq * shape.Lq * 4
    return float(q + kv + o + lse)


def decode_bytes(shape: DecodeShape, seq_lens, q_len: int = 1) -> float:
    """Algorithmic HBM bytes of one paged decode of q_len tokens per sequence:
    every cached K and V element of every sequence once, plus q, o, lse, the
    used block-table entries and seq_lens."""
    ps = shape.page_size
    lens = [int(x) for x in seq_lens]
    kv = sum(lens) * shape.Hkv * shape.D * 2 * 2
    q = shape.B * shape.Hq * q_len * shape.D * 2
    o = shape.B * shape.Hq * q_len * shape.D * 2
    lse = shape.B * shape.Hq * q_len * 4
    table = sum((n + ps - 1) // ps for n in lens) * 4 + shape.B * 4
    return float(kv + q + o + lse + table)


def decode_flops(shape: DecodeShape, seq_lens) -> float:
    return 4.0 * shape.D * shape.Hq * float(sum(int(x) for x in seq_lens))

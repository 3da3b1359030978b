"""The work accounting behind every TFLOP/s and GB/s figure, pinned to the
closed forms of the five workloads and to brute-force mask counts."""
import itertools

from workloads import (FP8_CAUSAL, GQA_CAUSAL, MQA_DECODE, SWA_CAUSAL, TINY_MHA, DecodeShape,
                       PrefillShape)
from workloads.accounting import decode_bytes, decode_flops, prefill_bytes, prefill_flops, visible_pairs


def test_workload_flops_closed_forms():
    # 4*D FLOP per visible (query, key) pair per head; causal rows i see i + 1 keys
    assert prefill_flops(TINY_MHA) == 4 * 64 * 1 * 2 * 128 * 128
    assert prefill_flops(GQA_CAUSAL) == 4 * 128 * 4 * 32 * (4096 * 4097 // 2)
    assert round(prefill_flops(GQA_CAUSAL) / 1e11, 3) == 5.499
    W, L = 4096, 16384  # window of W keys including the query's own
    assert prefill_flops(SWA_CAUSAL) == 4 * 128 * 2 * 32 * (W * (W + 1) // 2 + (L - W) * W)
    assert round(prefill_flops(SWA_CAUSAL) / 1e12, 3) == 1.924
    assert prefill_flops(FP8_CAUSAL) == 4 * 128 * 1 * 32 * (32768 * 32769 // 2)
    assert round(prefill_flops(FP8_CAUSAL) / 1e12, 3) == 8.796


def test_visible_pairs_brute_force():
    for Lq, Lk, causal, window in itertools.product((1, 3, 7, 20), (1, 5, 20, 33), (False, True), (0, 1, 2, 6, 50)):
        if Lq > Lk or (window and not causal):
            continue
        off = Lk - Lq  # bottom-right alignment
        n = 0
        for i in range(Lq):
            for j in range(Lk):
                if causal and j > i + off:
                    continue
                if window and j < i + off - window + 1:
                    continue
                n += 1
        assert visible_pairs(Lq, Lk, causal, window) == n, (Lq, Lk, causal, window)


def test_prefill_bytes():
    # bf16: Q, K, V read once, O written once (bf16), LSE (fp32)
    q = 4 * 32 * 4096 * 128 * 2
    kv = 2 * 4 * 8 * 4096 * 128 * 2
    assert prefill_bytes(GQA_CAUSAL) == q + kv + q + 4 * 32 * 4096 * 4
    assert round(prefill_bytes(GQA_CAUSAL) / 1e6, 1) == 337.6
    # e4m3 inputs are one byte, O stays bf16
    el8 = 32 * 32768 * 128
    assert prefill_bytes(FP8_CAUSAL) == el8 * 3 + el8 * 2 + 32 * 32768 * 4
    assert round(prefill_bytes(FP8_CAUSAL) / 1e6, 1) == 675.3


def test_decode_accounting():
    sh = DecodeShape("t", B=3, Hq=8, Hkv=2, D=128, len_lo=1, len_hi=100)
    lens = [17, 1, 32]
    pages = 2 + 1 + 2
    kv = sum(lens) * 2 * 128 * 2 * 2
    for q_len in (1, 4):
        qo = 2 * 3 * 8 * q_len * 128 * 2
        assert decode_bytes(sh, lens, q_len) == kv + qo + 3 * 8 * q_len * 4 + pages * 4 + 3 * 4
    assert decode_flops(sh, lens) == 4 * 128 * 8 * sum(lens)
    # the MQA workload's K/V bytes at the mean length 4352: ~142.6 MB
    assert round(64 * 4352 * 1 * 128 * 2 * 2 / 1e6, 1) == 142.6
    assert MQA_DECODE.Hkv == 1 and MQA_DECODE.page_size == 16


def test_prefill_shape_fields():
    assert isinstance(GQA_CAUSAL, PrefillShape) and GQA_CAUSAL.Hq // GQA_CAUSAL.Hkv == 4


def test_latent_shapes_count_both_widths():
    """D_qk != D_v: Q.K^T costs 2*D_qk per visible pair and P.V 2*D_v; K is
    read at width D_qk, V at D_v, O written at D_v."""
    from workloads import LATENT_192_128
    s = LATENT_192_128
    pairs = 4096 * 4097 // 2
    assert prefill_flops(s) == 2 * (192 + 128) * 4 * 32 * pairs
    q = 4 * 32 * 4096 * 192 * 2
    kv = 4 * 8 * 4096 * (192 + 128) * 2
    o = 4 * 32 * 4096 * 128 * 2
    assert prefill_bytes(s) == q + kv + o + 4 * 32 * 4096 * 4

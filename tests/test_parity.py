"""GPU parity: the CUDA kernels (through the C ABI) against the float64 oracle
on the same seeded inputs.

Tolerances (bf16 output): max |O - O_ref| <= 1e-2, mean <= 1e-3, and
|LSE - LSE_ref| <= 1e-3; FP8 inputs: 5e-2 / 5e-3 on O, 1e-3 on LSE.  The
bf16 rounding of O alone contributes up to half an ulp (3.9e-3 for |O| in
[1, 2)); the rest comes from fp32 accumulation and the bf16 (or e4m3)
rounding of P before the P.V product.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import (FP8_CAUSAL, GQA_CAUSAL, MQA_DECODE, SWA_CAUSAL, TINY_MHA, DecodeShape,
                       PrefillShape, decode_inputs, decode_queries, prefill_inputs, prefill_inputs_fp8,
                       seed_of)

pytestmark = pytest.mark.gpu

BF16_TOL = (1e-2, 1e-3)
FP8_TOL = (5e-2, 5e-3)
LSE_TOL = 1e-3


def _errs(o_gpu, o_ref, lse_gpu, lse_ref):
    o_gpu = o_gpu.double().cpu().numpy()
    lse_gpu = lse_gpu.double().cpu().numpy()
    d = np.abs(o_gpu - o_ref)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin), "LSE finiteness differs (empty rows)"
    dl = np.abs(lse_gpu[fin] - lse_ref[fin]) if fin.any() else np.zeros(1)
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0, float(dl.max())


def _check(o_gpu, o_ref, lse_gpu, lse_ref, tol=BF16_TOL, what=""):
    mx, mean, dl = _errs(o_gpu, o_ref, lse_gpu, lse_ref)
    assert mx <= tol[0] and mean <= tol[1] and dl <= LSE_TOL, \
        f"{what}: max {mx:.3e} mean {mean:.3e} lse {dl:.3e}"
    # rows with no visible key must be exactly zero
    empty = ~np.isfinite(lse_ref)
    if empty.any():
        assert np.all(o_gpu.float().cpu().numpy()[empty] == 0)
    return mx, mean, dl


def _run_prefill(lib, shape: PrefillShape, seed: int):
    q, k, v = prefill_inputs(shape, seed)
    o, lse = lib.attn_fwd(q.cuda(), k.cuda(), v.cuda(), shape.scale, shape.causal, shape.window)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    return q, k, v, o, lse


def test_tiny_mha_exact_definition(lib):
    shape = TINY_MHA
    q, k, v, o, lse = _run_prefill(lib, shape, seed_of(0))
    o_ref, l_ref = oracle.attention(q, k, v, shape.scale, shape.causal, shape.window)
    _check(o, o_ref, lse, l_ref, what=shape.name)


SWEEP = []
for D in (64, 128):
    for (Hq, Hkv) in ((2, 2), (4, 1), (8, 2), (3, 1)):
        for L in (1, 17, 127, 128, 129, 300):
            for causal in (False, True):
                SWEEP.append((1, Hq, Hkv, L, L, D, causal, 0))
SWEEP += [
    (3, 4, 4, 1000, 1000, 128, True, 0),
    (1, 8, 1, 257, 257, 128, False, 0),
    (2, 32, 1, 200, 200, 128, True, 0),     # MQA, group 32
    (1, 4, 2, 100, 300, 128, True, 0),      # Lq < Lk, bottom-right causal
    (1, 4, 2, 100, 300, 64, False, 0),
    (1, 4, 2, 300, 100, 128, True, 0),      # Lq > Lk: first rows see no key
    (1, 2, 2, 50, 0, 128, False, 0),        # no keys at all
]
for W in (1, 2, 127, 128, 129, 300, 5000):
    SWEEP.append((1, 4, 2, 600, 600, 128, True, W))
    SWEEP.append((1, 3, 3, 300, 300, 64, True, W))
SWEEP.append((2, 8, 2, 1000, 1300, 128, True, 200))


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,D,causal,window", SWEEP)
def test_prefill_sweep(lib, B, Hq, Hkv, Lq, Lk, D, causal, window):
    shape = PrefillShape("sweep", B, Hq, Hkv, Lq, Lk, D, causal, window)
    q, k, v, o, lse = _run_prefill(lib, shape, 7 + Lq + 3 * Lk + D + window)
    o_ref, l_ref = oracle.attention(q, k, v, shape.scale, causal, window)
    _check(o, o_ref, lse, l_ref, what=str(shape))


def test_window_at_least_length_equals_causal_on_gpu(lib):
    shape = PrefillShape("w", 1, 4, 2, 333, 333, 128, True, 0)
    q, k, v = prefill_inputs(shape, 5)
    a = lib.attn_fwd(q.cuda(), k.cuda(), v.cuda(), shape.scale, True, 0)
    b = lib.attn_fwd(q.cuda(), k.cuda(), v.cuda(), shape.scale, True, 333)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_causal_row_zero_and_window_one_are_exact(lib):
    """Row 0 under a causal mask (and every row with W = 1) sees one key, so
    O equals that bf16 V row exactly."""
    shape = PrefillShape("w1", 1, 4, 2, 256, 256, 128, True, 1)
    q, k, v = prefill_inputs(shape, 6)
    o, lse = lib.attn_fwd(q.cuda(), k.cuda(), v.cuda(), shape.scale, True, 1)
    torch.cuda.synchronize()
    vr = v.repeat_interleave(2, dim=1)
    assert torch.equal(o.cpu(), vr)
    o2, _ = lib.attn_fwd(q.cuda(), k.cuda(), v.cuda(), shape.scale, True, 0)
    torch.cuda.synchronize()
    assert torch.equal(o2[:, :, 0].cpu(), vr[:, :, 0])


def _sampled_rows(L, n, seed):
    g = np.random.default_rng(seed)
    rows = set(g.choice(L, size=n, replace=False).tolist())
    rows |= {0, 1, 127, 128, L - 1}
    return sorted(r for r in rows if r < L)


@pytest.mark.parametrize("idx,shape", [(1, GQA_CAUSAL), (3, SWA_CAUSAL)])
def test_full_size_prefill_sampled_rows(lib, idx, shape):
    """Full workload on the GPU; the oracle computes sampled rows of a few
    (batch, head) pairs, one by one."""
    q, k, v, o, lse = _run_prefill(lib, shape, seed_of(idx))
    rows = _sampled_rows(shape.Lq, 24, idx)
    for b, heads in ((0, [0, 1, 5]), (shape.B - 1, [shape.Hq - 1, shape.Hq - 4])):
        o_ref, l_ref = oracle.attention(q, k, v, shape.scale, shape.causal, shape.window,
                                        rows=rows, heads=heads, batches=[b])
        _check(o[b][heads][:, rows], o_ref[0], lse[b][heads][:, rows], l_ref[0], what=shape.name)


def test_fp8_small(lib):
    shape = PrefillShape("fp8_small", 1, 4, 4, 700, 700, 128, True, fp8=True)
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, 11)
    o, lse = lib.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, shape.scale, True, 0)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    o_ref, l_ref = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, shape.scale, True)
    _check(o, o_ref, lse, l_ref, FP8_TOL, what="fp8 small")


@pytest.mark.parametrize("window", [2, 3])
def test_fp8_few_key_rows(lib, window):
    """FP8 with a window of 2 or 3 keys: every row averages a handful of V
    rows, where the rounding of the weights to e4m3 does not average out.
    Tiles whose rows see fewer than 512 keys multiply V by the e4m3 weights
    and by their e4m3 rounding residual, so these rows meet the same
    5e-2 / 5e-3 bound as the FP8 workload."""
    shape = PrefillShape("fp8_w", 1, 2, 2, 600, 600, 128, True, window=window, fp8=True)
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, 12)
    o, lse = lib.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, shape.scale, True, window)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    o_ref, l_ref = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, shape.scale, True, window)
    _check(o, o_ref, lse, l_ref, FP8_TOL, what=f"fp8 window {window}")


FP8_SWEEP = [
    (1, 4, 2, 1100, 1100, True, 0),     # GQA pairs; tiles before and after row 512
    (1, 3, 3, 1100, 1100, True, 0),     # MHA pairs of row blocks across row 512
    (1, 4, 2, 700, 700, True, 300),     # every row sees <= 300 keys
    (1, 4, 2, 900, 900, True, 600),     # window wider than 512
    (1, 4, 4, 100, 900, True, 0),       # Lq < Lk: every row sees > 800 keys
    (1, 2, 2, 300, 100, True, 0),       # Lq > Lk: first rows see no key
    (2, 2, 1, 77, 200, False, 0),       # non-causal, short key range
    (1, 8, 1, 600, 600, True, 0),       # MQA, group 8
    (1, 2, 2, 17, 17, True, 0),         # one ragged tile
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,causal,window", FP8_SWEEP)
def test_fp8_sweep(lib, B, Hq, Hkv, Lq, Lk, causal, window):
    shape = PrefillShape("fp8_sweep", B, Hq, Hkv, Lq, Lk, 128, causal, window=window, fp8=True)
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, 13 + Lq + Lk + window)
    o, lse = lib.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, shape.scale, causal, window)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    o_ref, l_ref = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, shape.scale, causal, window)
    _check(o, o_ref, lse, l_ref, FP8_TOL, what=str(shape))


def test_fp8_full_size_rows(lib):
    """The FP8 workload (B1 Hq32 L32768, causal): rows 0..255 of all 32 heads
    (the rows with the fewest keys, row 1 of each head sees two), plus sampled
    rows of three heads across the whole length."""
    shape = FP8_CAUSAL
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, seed_of(4))
    o, lse = lib.attn_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, shape.scale, True, 0)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    first = list(range(256))
    o_ref, l_ref = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, shape.scale, True, rows=first, batches=[0])
    _check(o[0][:, first], o_ref[0], lse[0][:, first], l_ref[0], FP8_TOL, what=shape.name + " rows 0-255")
    rows = _sampled_rows(shape.Lq, 16, 4)
    heads = [0, 13, 31]
    o_ref, l_ref = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, shape.scale, True,
                                        rows=rows, heads=heads, batches=[0])
    _check(o[0][heads][:, rows], o_ref[0], lse[0][heads][:, rows], l_ref[0], FP8_TOL, what=shape.name)


E5M2_SWEEP = [
    (1, 4, 2, 1100, 1100, True, 0),
    (1, 3, 3, 300, 300, True, 2),       # rows of two keys
    (1, 4, 2, 700, 700, True, 300),
    (1, 4, 4, 100, 900, True, 0),       # Lq < Lk
    (1, 2, 2, 300, 100, True, 0),       # Lq > Lk: first rows see no key
    (2, 2, 1, 77, 200, False, 0),
]


def _run_e5m2(lib, shape, seed):
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, seed, fmt="e5m2")
    o, lse = lib.attn_fwd_e5m2(q8.cuda(), k8.cuda(), v8.cuda(), sq, sk, sv, shape.scale, shape.causal,
                               shape.window)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    return (q8, k8, v8, sq, sk, sv), o, lse


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,causal,window", E5M2_SWEEP)
def test_e5m2_sweep(lib, B, Hq, Hkv, Lq, Lk, causal, window):
    """float8_e5m2 inputs (kler.cn §四.2): e5m2 products, P multiplied with V
    as e5m2 and its e5m2 residual; the FP8 bound."""
    shape = PrefillShape("e5m2", B, Hq, Hkv, Lq, Lk, 128, causal, window=window, fp8=True)
    ins, o, lse = _run_e5m2(lib, shape, 17 + Lq + Lk + window)
    o_ref, l_ref = oracle.attention_fp8(*ins, shape.scale, causal, window)
    _check(o, o_ref, lse, l_ref, FP8_TOL, what=f"e5m2 {shape}")


def test_e5m2_full_size_rows(lib):
    """The long-context FP8 workload's shape (B1 Hq32 L32768, causal) with
    e5m2 inputs: rows 0..127 of all heads and sampled rows of three heads."""
    shape = FP8_CAUSAL
    ins, o, lse = _run_e5m2(lib, shape, seed_of(4))
    first = list(range(128))
    o_ref, l_ref = oracle.attention_fp8(*ins, shape.scale, True, rows=first, batches=[0])
    _check(o[0][:, first], o_ref[0], lse[0][:, first], l_ref[0], FP8_TOL, what="e5m2 rows 0-127")
    rows = _sampled_rows(shape.Lq, 12, 5)
    heads = [2, 17, 30]
    o_ref, l_ref = oracle.attention_fp8(*ins, shape.scale, True, rows=rows, heads=heads, batches=[0])
    _check(o[0][heads][:, rows], o_ref[0], lse[0][heads][:, rows], l_ref[0], FP8_TOL, what="e5m2 sampled")


def _whole_heads(q, k, v, shape, b, heads, o, lse, tol=BF16_TOL, chunk=2048):
    """Every row of the given heads of batch b against the oracle, in row
    chunks (each chunk's score block spans only its visible keys)."""
    for r0 in range(0, shape.Lq, chunk):
        rows = list(range(r0, min(r0 + chunk, shape.Lq)))
        o_ref, l_ref = oracle.attention(q, k, v, shape.scale, shape.causal, shape.window,
                                        rows=rows, heads=heads, batches=[b])
        _check(o[b][heads][:, rows], o_ref[0], lse[b][heads][:, rows], l_ref[0], tol,
               what=f"{shape.name} b{b} heads {heads} rows {r0}..")


def test_full_size_gqa_causal_whole_groups(lib):
    """The GQA causal workload (B4 Hq32 Hkv8 L4096): every row of the first
    K/V group of batch 0 (query heads 0-3) and of the last group of batch 3
    (heads 28-31), i.e. all (head, row-block) work units of those groups."""
    shape = GQA_CAUSAL
    q, k, v, o, lse = _run_prefill(lib, shape, seed_of(1))
    _whole_heads(q, k, v, shape, 0, [0, 1, 2, 3], o, lse)
    _whole_heads(q, k, v, shape, shape.B - 1, [28, 29, 30, 31], o, lse)


def test_full_size_sliding_window_whole_heads(lib):
    """The sliding-window workload (B2 Hq32 Hkv8 L16384 W4096): every row of
    head 0 of batch 0 and of head 31 of batch 1."""
    shape = SWA_CAUSAL
    q, k, v, o, lse = _run_prefill(lib, shape, seed_of(3))
    _whole_heads(q, k, v, shape, 0, [0], o, lse)
    _whole_heads(q, k, v, shape, 1, [31], o, lse)


# Keys that no query row can see are never loaded or multiplied: they hold
# NaN here, and since P = 0 times NaN is still NaN, one multiplied NaN key
# would reach O.  Lq = 300 queries over Lk = 1000 keys with a window of 189:
# row 0 sees keys 512..700 (bottom-right alignment), so keys 0..511 -- four
# whole 128-key blocks -- are invisible to every row.
NAN_CASES = [(1, 4, 2, 300, 1000, 189), (2, 3, 1, 300, 1000, 189), (1, 2, 2, 44, 556, 1)]


def _nan_prefix(shape):
    lo0, _ = oracle.visible_key_range(0, shape.Lq, shape.Lk, True, shape.window)
    assert lo0 % 128 == 0 and lo0 > 0
    return lo0


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,W", NAN_CASES)
def test_never_visible_blocks_are_not_read(lib, B, Hq, Hkv, Lq, Lk, W):
    shape = PrefillShape("nan", B, Hq, Hkv, Lq, Lk, 128, True, window=W)
    q, k, v = prefill_inputs(shape, 31 + Lq + W)
    n0 = _nan_prefix(shape)
    kn, vn = k.clone(), v.clone()
    kn[:, :, :n0] = float("nan")
    vn[:, :, :n0] = float("nan")
    o, lse = lib.attn_fwd(q.cuda(), kn.cuda(), vn.cuda(), shape.scale, True, W)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    o_ref, l_ref = oracle.attention(q, k, v, shape.scale, True, W)   # the NaN keys do not enter the definition
    _check(o, o_ref, lse, l_ref, what=f"nan prefix {shape}")
    # backward: the invisible keys get exactly zero gradients, the rest match
    g = torch.Generator().manual_seed(32 + Lq)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    dq, dk, dv = lib.attn_bwd(q.cuda(), kn.cuda(), vn.cuda(), o, do.cuda(), lse, shape.scale, True, W)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    assert (dk[:, :, :n0] == 0).all() and (dv[:, :, :n0] == 0).all()
    dq_r, dk_r, dv_r = oracle.attention_backward(q, k, v, o_ref, do, l_ref, shape.scale, True, W)
    # relative to each gradient's scale, as in the backward tests; with W = 1
    # the exact dQ is 0 (one weight of 1: dP - rowsum(dO * O) vanishes) and the
    # kernel leaves fp32 rounding of that difference, hence the 1e-5 floor
    for name, got, ref in (("dq", dq, dq_r), ("dk", dk, dk_r), ("dv", dv, dv_r)):
        err = np.abs(got.double().cpu().numpy() - ref)
        assert err.max() <= 2e-2 * np.abs(ref).max() + 1e-5, name


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,W", NAN_CASES[:2])
def test_never_visible_blocks_are_not_read_fp8(lib, B, Hq, Hkv, Lq, Lk, W):
    shape = PrefillShape("nan8", B, Hq, Hkv, Lq, Lk, 128, True, window=W, fp8=True)
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, 33 + Lq)
    n0 = _nan_prefix(shape)
    kn, vn = k8.clone(), v8.clone()
    nan8 = torch.tensor(float("nan")).to(torch.float8_e4m3fn)
    kn[:, :, :n0] = nan8
    vn[:, :, :n0] = nan8
    o, lse = lib.attn_fwd_fp8(q8.cuda(), kn.cuda(), vn.cuda(), sq, sk, sv, shape.scale, True, W)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    o_ref, l_ref = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, shape.scale, True, W)
    _check(o, o_ref, lse, l_ref, FP8_TOL, what=f"nan prefix fp8 {shape}")


# ------------------------------------------------------------------ decode
def _run_decode(lib, kv, scale):
    d = {n: getattr(kv, n).cuda() for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
    o, lse = lib.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], scale)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    return o, lse


def test_decode_full_workload(lib):
    shape = MQA_DECODE
    kv = decode_inputs(shape, seed_of(2))
    o, lse = _run_decode(lib, kv, shape.scale)
    o_ref, l_ref = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    _check(o, o_ref, lse, l_ref, what=shape.name)


@pytest.mark.parametrize("lens,Hq,Hkv", [
    ([1, 15, 16, 17, 512, 513, 8192, 0], 32, 1),
    ([3, 100, 1000, 2049], 32, 4),
    ([700, 1, 64], 16, 2),
    ([5000, 31], 8, 8),
    ([0, 0], 32, 1),
    ([300, 77, 1], 64, 1),       # two softmax warps per K/V group
    ([129, 4000], 128, 1),       # four
    ([50, 33, 16], 12, 4),       # group of 3 (query rows padded to 8)
])
def test_decode_edge_lengths(lib, lens, Hq, Hkv):
    shape = DecodeShape("edge", B=len(lens), Hq=Hq, Hkv=Hkv, D=128, len_lo=1, len_hi=1)
    kv = decode_inputs(shape, 99 + sum(lens), seq_lens=lens, extra_pages=5)
    o, lse = _run_decode(lib, kv, shape.scale)
    o_ref, l_ref = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    _check(o, o_ref, lse, l_ref, what=str(lens))


def test_decode_ignores_cache_slots_past_the_end(lib):
    # Slots of the last page beyond a sequence's length (and pages no table
    # entry reaches) hold NaN: attention over the first `len` tokens must not
    # see them.
    shape = DecodeShape("nan-tail", B=4, Hq=32, Hkv=2, D=128, len_lo=1, len_hi=1)
    lens = [17, 100, 1, 250]
    kv = decode_inputs(shape, 11, seq_lens=lens, extra_pages=3)
    used = torch.zeros(kv.num_pages, dtype=torch.bool)
    for b, n in enumerate(lens):
        npg = (n + 15) // 16
        used[kv.block_table[b, :npg].long()] = True
        last = int(kv.block_table[b, npg - 1])
        kv.k_pages[last, n - (npg - 1) * 16:] = float("nan")
        kv.v_pages[last, n - (npg - 1) * 16:] = float("nan")
    kv.k_pages[~used] = float("nan")
    kv.v_pages[~used] = float("nan")
    o, lse = _run_decode(lib, kv, shape.scale)
    o_ref, l_ref = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    _check(o, o_ref, lse, l_ref, what="nan-tail")


# ------------------------------------------------------- multi-token decode
def _run_decode_multi(lib, kv, qm, scale):
    d = {n: getattr(kv, n).cuda() for n in ("k_pages", "v_pages", "block_table", "seq_lens")}
    o, lse = lib.attn_decode_paged_multi(qm.cuda(), d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                                         scale)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    return o, lse


@pytest.mark.parametrize("lens,Hq,Hkv,q_len", [
    ([100, 17, 1, 2000], 32, 1, 4),      # 128 rows per tile (MQA)
    ([50, 3, 700, 4096], 32, 8, 8),      # group 4 x 8 tokens
    ([33, 5000], 8, 2, 2),
    ([2, 40, 0], 16, 4, 4),              # a cache shorter than q_len: rows without keys
    ([513, 64], 12, 4, 7),               # group 3 x 7 = 21 rows
])
def test_decode_multi_token(lib, lens, Hq, Hkv, q_len):
    shape = DecodeShape("multi", B=len(lens), Hq=Hq, Hkv=Hkv, D=128, len_lo=1, len_hi=1)
    kv = decode_inputs(shape, 77 + sum(lens), seq_lens=lens, extra_pages=2)
    qm = decode_queries(shape, q_len, 78 + q_len)
    o, lse = _run_decode_multi(lib, kv, qm, shape.scale)
    o_ref, l_ref = oracle.paged_decode(qm, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    _check(o, o_ref, lse, l_ref, what=f"{lens} q_len={q_len}")


def test_decode_multi_token_full_workload(lib):
    """The batch-64 MQA cache with 4 new tokens per sequence (all 128 rows of
    the tile used)."""
    shape = MQA_DECODE
    kv = decode_inputs(shape, seed_of(2))
    qm = decode_queries(shape, 4, seed_of(2) + 100)
    o, lse = _run_decode_multi(lib, kv, qm, shape.scale)
    o_ref, l_ref = oracle.paged_decode(qm, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    _check(o, o_ref, lse, l_ref, what="mqa q_len=4")


def test_decode_multi_of_one_token_is_decode(lib):
    shape = DecodeShape("one", B=5, Hq=32, Hkv=4, D=128, len_lo=10, len_hi=900)
    kv = decode_inputs(shape, 79)
    o1, l1 = _run_decode(lib, kv, shape.scale)
    o2, l2 = _run_decode_multi(lib, kv, kv.q[:, :, None], shape.scale)
    assert torch.equal(o1, o2[:, :, 0]) and torch.equal(l1, l2[:, :, 0])


# ------------------------------------------- chunked prefill over pages, KV append
def _paged_case(lens, Hq, Hkv, D, seed, nan_tail=False):
    shape = DecodeShape("paged", B=len(lens), Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=1)
    kv = decode_inputs(shape, seed, seq_lens=lens, extra_pages=3)
    if nan_tail:
        for b, n in enumerate(lens):
            npg = (n + 15) // 16
            if npg and n % 16:
                last = int(kv.block_table[b, npg - 1])
                kv.k_pages[last, n % 16:] = float("nan")
                kv.v_pages[last, n % 16:] = float("nan")
    return shape, kv


@pytest.mark.parametrize("lens,Hq,Hkv,Lq,D,window,nan_tail", [
    ([500, 200, 1000], 8, 2, 200, 128, 0, False),     # GQA, chunk after a cached prefix
    ([130, 77], 4, 4, 130, 64, 0, False),              # MHA, one cache shorter than the chunk
    ([700, 300], 6, 2, 256, 128, 100, True),           # group of 3, sliding window, NaN tail slots
    ([129, 16, 1], 32, 8, 17, 128, 0, True),
])
def test_prefill_paged(lib, lens, Hq, Hkv, Lq, D, window, nan_tail):
    shape, kv = _paged_case(lens, Hq, Hkv, D, 90 + Lq, nan_tail)
    q = decode_queries(shape, Lq, 91 + Lq)
    d = {n: getattr(kv, n).cuda() for n in ("k_pages", "v_pages", "block_table", "seq_lens")}
    o, lse = lib.attn_prefill_paged(q.cuda(), d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                                    shape.scale, window)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    o_ref, l_ref = oracle.paged_decode(q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale,
                                       window=window)
    assert torch.isfinite(o.float()).all()
    _check(o, o_ref, lse, l_ref, what=f"paged prefill {lens} Lq={Lq} W={window}")


def test_prefill_paged_equals_contiguous_prefill(lib):
    """Sequences of equal length whose whole cache is the chunk: the paged
    kernel reads the same K/V blocks as attn_fwd on the contiguous tensors and
    must give identical bits."""
    B, Hq, Hkv, L, D = 2, 8, 2, 384, 128
    shape = DecodeShape("eq", B=B, Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=1)
    kv = decode_inputs(shape, 95, seq_lens=[L] * B)
    q = decode_queries(shape, L, 96)
    k = torch.stack([torch.from_numpy(oracle.gather_pages(kv.k_pages, kv.block_table[b], L, 16)).to(torch.bfloat16)
                     .permute(1, 0, 2) for b in range(B)])
    v = torch.stack([torch.from_numpy(oracle.gather_pages(kv.v_pages, kv.block_table[b], L, 16)).to(torch.bfloat16)
                     .permute(1, 0, 2) for b in range(B)])
    d = {n: getattr(kv, n).cuda() for n in ("k_pages", "v_pages", "block_table", "seq_lens")}
    o1, l1 = lib.attn_prefill_paged(q.cuda(), d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                                    shape.scale)
    o2, l2 = lib.attn_fwd(q.cuda(), k.contiguous().cuda(), v.contiguous().cuda(), shape.scale, True, 0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_kv_append_then_prefill(lib):
    """Append a chunk's K/V into the pages (exactly the oracle's scatter), then
    attend the chunk over the whole cache."""
    lens, Ln = [300, 40, 17], 40
    shape, kv = _paged_case(lens, 8, 2, 128, 97)
    g = torch.Generator().manual_seed(98)
    k_new = torch.randn(3, 2, Ln, 128, generator=g).to(torch.bfloat16)
    v_new = torch.randn(3, 2, Ln, 128, generator=g).to(torch.bfloat16)
    d = {n: getattr(kv, n).cuda() for n in ("k_pages", "v_pages", "block_table", "seq_lens")}
    lib.attn_kv_append(k_new.cuda(), v_new.cuda(), d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"])
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    kp_ref, vp_ref = oracle.kv_append(kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, k_new, v_new)
    assert np.array_equal(d["k_pages"].double().cpu().numpy(), kp_ref)
    assert np.array_equal(d["v_pages"].double().cpu().numpy(), vp_ref)
    q = decode_queries(shape, Ln, 99)
    o, lse = lib.attn_prefill_paged(q.cuda(), d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                                    shape.scale)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.paged_decode(q, kp_ref, vp_ref, kv.block_table, kv.seq_lens, shape.scale)
    _check(o, o_ref, lse, l_ref, what="append + paged prefill")


def test_kv_append_rejects_bad_page_ids(lib):
    shape, kv = _paged_case([40, 20], 4, 2, 128, 100)
    kv.block_table[1, 0] = kv.num_pages + 3
    k_new = torch.zeros(2, 2, 8, 128, dtype=torch.bfloat16)
    d = {n: getattr(kv, n).cuda() for n in ("k_pages", "v_pages", "block_table", "seq_lens")}
    before = d["k_pages"].clone()
    lib.attn_kv_append(k_new.cuda(), k_new.cuda(), d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"])
    assert lib.attn_last_device_error() == lib.ATTN_ERR_BOUNDS
    # sequence 0 was written; of sequence 1 (positions 12..19) only the
    # tokens on its good page (16..19) were, the ones on the bad page skipped
    kp_ref, vp_ref = oracle.kv_append(kv.k_pages, kv.v_pages, kv.block_table[:1], kv.seq_lens[:1], k_new[:1],
                                      k_new[:1])
    kp_ref, _ = oracle.kv_append(kp_ref, vp_ref, kv.block_table[1:], kv.seq_lens[1:], k_new[1:, :, 4:],
                                 k_new[1:, :, 4:])
    assert np.array_equal(d["k_pages"].double().cpu().numpy(), kp_ref)
    assert not torch.equal(before, d["k_pages"])


def test_decode_invariant_to_page_permutation(lib):
    shape = DecodeShape("perm", B=4, Hq=32, Hkv=1, D=128, len_lo=100, len_hi=900)
    kv = decode_inputs(shape, 5)
    o1, l1 = _run_decode(lib, kv, shape.scale)
    perm = torch.randperm(kv.num_pages, generator=torch.Generator().manual_seed(1))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(kv.num_pages)
    kp = torch.empty_like(kv.k_pages)
    vp = torch.empty_like(kv.v_pages)
    kp[inv] = kv.k_pages
    vp[inv] = kv.v_pages
    kv.k_pages, kv.v_pages = kp, vp
    kv.block_table = inv[kv.block_table.long()].int()
    o2, l2 = _run_decode(lib, kv, shape.scale)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_bounds_check_reports_bad_page(lib):
    shape = DecodeShape("bounds", B=2, Hq=32, Hkv=1, D=128, len_lo=1, len_hi=1)
    kv = decode_inputs(shape, 3, seq_lens=[40, 20])
    kv.block_table[1, 0] = kv.num_pages + 7       # out of the pool
    prev = lib.attn_set_debug(lib.ATTN_DEBUG_BOUNDS, 0)
    try:
        d = {n: getattr(kv, n).cuda() for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
        lib.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], shape.scale)
        assert lib.attn_last_device_error() == lib.ATTN_ERR_BOUNDS
        assert lib.attn_last_device_error() == 0      # cleared by the read
    finally:
        lib.attn_set_debug(prev, 0)

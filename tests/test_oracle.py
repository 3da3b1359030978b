"""Pins for the float64 oracle (CPU only).

Each test ties an oracle function to something other than itself: scalar
brute force, torch's float64 SDPA library routine, a closed form, an
invariant the pages state, or the exact result of a reduction to a simpler
case.  Together they are chosen so that a dropped scale, a wrong sign, a
transposed operand, a wrong GQA head map, an off-by-one window edge, a wrong
causal alignment or a wrong LSE base fails at least one test.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import PrefillShape, DecodeShape, prefill_inputs, decode_inputs, prefill_inputs_fp8


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


# ---------------------------------------------------------------- brute force
def _brute(q, k, v, scale, causal, window):
    """Scalar triple loop straight from softmax's definition, with the mask
    written as explicit index inequalities (bottom-right causal alignment,
    window of W keys including the query's own position)."""
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    Dv = v.shape[3]
    rep = Hq // Hkv
    o = np.zeros((B, Hq, Lq, Dv))
    lse = np.full((B, Hq, Lq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            g = h // rep
            for i in range(Lq):
                pos = i + (Lk - Lq)          # the query's position among the keys
                logits = []
                for j in range(Lk):
                    if causal and j > pos:
                        continue
                    if window > 0 and j <= pos - window:
                        continue
                    dot = 0.0
                    for d in range(D):
                        dot += float(q[b, h, i, d]) * float(k[b, g, j, d])
                    logits.append((j, scale * dot))
                if not logits:
                    continue
                mx = max(s for _, s in logits)
                den = sum(math.exp(s - mx) for _, s in logits)
                lse[b, h, i] = mx + math.log(den)
                for d in range(Dv):
                    o[b, h, i, d] = sum(math.exp(s - mx) / den * float(v[b, g, j, d]) for j, s in logits)
    return o, lse


BRUTE_CASES = [
    # B, Hq, Hkv, Lq, Lk, D, causal, window
    (1, 1, 1, 5, 5, 3, False, 0),
    (2, 2, 1, 4, 7, 4, False, 0),     # MQA, Lq != Lk
    (1, 4, 2, 6, 6, 2, True, 0),      # GQA causal
    (1, 2, 2, 3, 8, 4, True, 0),      # causal, Lq < Lk (bottom-right)
    (1, 3, 1, 7, 7, 3, True, 3),      # MQA window 3
    (2, 2, 1, 5, 9, 2, True, 2),      # window with Lq < Lk
    (1, 2, 2, 6, 6, 4, True, 1),      # window 1
]


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,D,causal,window", BRUTE_CASES)
def test_definition_matches_brute_force(B, Hq, Hkv, Lq, Lk, D, causal, window):
    q = _rand((B, Hq, Lq, D), 1)
    k = _rand((B, Hkv, Lk, D), 2)
    v = _rand((B, Hkv, Lk, D + 1), 3)     # Dv != D catches a transposed P.V
    scale = 0.37
    o, lse = oracle.attention(q, k, v, scale, causal, window)
    ob, lb = _brute(q.numpy(), k.numpy(), v.numpy(), scale, causal, window)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-13)


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,D,causal,window", BRUTE_CASES)
@pytest.mark.parametrize("blocks", [(1, 1), (2, 3), (7, 7), (128, 128)])
def test_online_recurrence_matches_brute_force(B, Hq, Hkv, Lq, Lk, D, causal, window, blocks):
    q = _rand((B, Hq, Lq, D), 4)
    k = _rand((B, Hkv, Lk, D), 5)
    v = _rand((B, Hkv, Lk, D), 6)
    o, lse = oracle.online_softmax_attention(q, k, v, 0.5, causal, window, *blocks)
    ob, lb = _brute(q.numpy(), k.numpy(), v.numpy(), 0.5, causal, window)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


# ---------------------------------------------------- library routine (torch)
@pytest.mark.parametrize("Hq,Hkv,L,causal", [(4, 4, 33, False), (4, 4, 40, True), (8, 2, 29, True), (6, 1, 17, False)])
def test_definition_matches_torch_sdpa(Hq, Hkv, L, causal):
    """torch's SDPA in float64 computes the same definition (its causal mask
    is top-left aligned, identical to ours when Lq == Lk).  The math backend
    is requested explicitly: it forms softmax(scale * Q K^T) V as written, so
    the comparison does not depend on which fused CPU kernel torch picks."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    q = _rand((2, Hq, L, 16), 7)
    k = _rand((2, Hkv, L, 16), 8)
    v = _rand((2, Hkv, L, 16), 9)
    scale = 1 / math.sqrt(16)
    with sdpa_kernel(SDPBackend.MATH):
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, is_causal=causal, scale=scale, enable_gqa=(Hq != Hkv))
    o, lse = oracle.attention(q, k, v, scale, causal)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
    # LSE against torch.logsumexp over the masked score matrix
    kk = k.repeat_interleave(Hq // Hkv, dim=1)
    s = scale * q @ kk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------- closed forms
def test_identical_keys_give_mean_of_values_and_log_count():
    """All keys equal: every visible key has the same logit s, so softmax is
    uniform -- O_i is the mean of the visible V rows and LSE_i = s + ln n_i."""
    L, D = 37, 8
    q = _rand((1, 1, L, D), 10)
    key = _rand((D,), 11)
    k = key.expand(1, 1, L, D).clone()
    v = _rand((1, 1, L, D), 12)
    o, lse = oracle.attention(q, k, v, 0.3, causal=True, window=5)
    vn = v.numpy()[0, 0]
    for i in range(L):
        lo, hi = max(0, i - 4), i + 1
        s = 0.3 * float(q[0, 0, i] @ key)
        np.testing.assert_allclose(o[0, 0, i], vn[lo:hi].mean(axis=0), rtol=0, atol=1e-13)
        assert abs(lse[0, 0, i] - (s + math.log(hi - lo))) < 1e-12


def test_one_dominant_logit_returns_its_value_row():
    L, D = 20, 16
    q = _rand((1, 2, 1, D), 13)
    k = _rand((1, 2, L, D), 14)
    v = _rand((1, 2, L, D), 15)
    j = 11
    for h in range(2):
        k[0, h, j] = 100.0 * q[0, h, 0] / q[0, h, 0].norm()
    o, _ = oracle.attention(q, k, v, 1.0)
    for h in range(2):
        np.testing.assert_allclose(o[0, h, 0], v[0, h, j].numpy(), rtol=0, atol=1e-30)


def test_window_one_returns_own_value_row():
    """W = 1: each query sees only its own key, so O_i = V_i and
    LSE_i = scale * q_i . k_i exactly."""
    q = _rand((1, 2, 9, 4), 16)
    k = _rand((1, 2, 9, 4), 17)
    v = _rand((1, 2, 9, 4), 18)
    o, lse = oracle.attention(q, k, v, 0.7, causal=True, window=1)
    np.testing.assert_array_equal(o, v.numpy())
    np.testing.assert_allclose(lse, 0.7 * (q * k).sum(-1).numpy(), rtol=0, atol=1e-15)


def test_causal_row_zero_is_first_value_row():
    q = _rand((1, 3, 12, 8), 19)
    k = _rand((1, 3, 12, 8), 20)
    v = _rand((1, 3, 12, 8), 21)
    o, lse = oracle.attention(q, k, v, 0.25, causal=True)
    np.testing.assert_array_equal(o[:, :, 0], v.numpy()[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.25 * (q[:, :, 0] * k[:, :, 0]).sum(-1).numpy(), rtol=0, atol=1e-15)


def test_decode_query_sees_every_key():
    """Bottom-right causal alignment: one query row against Lk keys sees all
    of them, i.e. causal == non-causal for Lq = 1."""
    q = _rand((2, 4, 1, 8), 22)
    k = _rand((2, 2, 30, 8), 23)
    v = _rand((2, 2, 30, 8), 24)
    a = oracle.attention(q, k, v, 0.3, causal=True)
    b = oracle.attention(q, k, v, 0.3, causal=False)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_shift_invariance_of_a_row():
    """Adding a constant c to every logit of a row leaves O unchanged and
    shifts LSE by c (safe softmax).  The shift is made through an extra
    feature column: q gets c/scale, every key gets 1."""
    L, D, scale, c = 15, 6, 0.4, 3.25
    q = _rand((1, 1, L, D), 25)
    k = _rand((1, 1, L, D), 26)
    v = _rand((1, 1, L, D), 27)
    q2 = torch.cat([q, torch.full((1, 1, L, 1), c / scale, dtype=torch.float64)], -1)
    k2 = torch.cat([k, torch.ones((1, 1, L, 1), dtype=torch.float64)], -1)
    o1, l1 = oracle.attention(q, k, v, scale, causal=True)
    o2, l2 = oracle.attention(q2, k2, v, scale, causal=True)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + c, rtol=0, atol=1e-12)


def test_fully_masked_rows_are_zero_with_minus_inf_lse():
    q = _rand((1, 1, 4, 4), 28)
    k = torch.zeros((1, 1, 0, 4), dtype=torch.float64)
    v = torch.zeros((1, 1, 0, 4), dtype=torch.float64)
    o, lse = oracle.attention(q, k, v, 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    # Lq > Lk causal: the first Lq - Lk rows have no visible key
    q = _rand((1, 1, 6, 4), 29)
    k = _rand((1, 1, 3, 4), 30)
    v = _rand((1, 1, 3, 4), 31)
    o, lse = oracle.attention(q, k, v, 1.0, causal=True)
    assert np.all(o[0, 0, :3] == 0) and np.all(np.isneginf(lse[0, 0, :3]))
    assert np.all(np.isfinite(lse[0, 0, 3:]))


# ------------------------------------------------------------- invariants
def test_gqa_equals_mha_after_repeat_kv():
    """The GQA section of p3: repeat_kv duplicates each K/V head for its
    group; GQA on Hkv heads must equal MHA on the duplicated heads, bit for bit."""
    q = _rand((2, 8, 21, 8), 32)
    k = _rand((2, 2, 21, 8), 33)
    v = _rand((2, 2, 21, 8), 34)
    a = oracle.attention(q, k, v, 0.35, causal=True, window=6)
    b = oracle.attention(q, oracle.repeat_kv(k, 4), oracle.repeat_kv(v, 4), 0.35, causal=True, window=6)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    # repeat_kv puts a group's copies next to each other
    rk = oracle.repeat_kv(k, 4)
    np.testing.assert_array_equal(rk[:, 5], k.numpy()[:, 1])


def test_window_at_least_length_equals_causal():
    q = _rand((1, 2, 30, 4), 35)
    k = _rand((1, 2, 30, 4), 36)
    v = _rand((1, 2, 30, 4), 37)
    c = oracle.attention(q, k, v, 0.5, causal=True)
    for w in (30, 31, 1000):
        wres = oracle.attention(q, k, v, 0.5, causal=True, window=w)
        np.testing.assert_array_equal(wres[0], c[0])
        np.testing.assert_array_equal(wres[1], c[1])
    # and a smaller window really differs
    w29 = oracle.attention(q, k, v, 0.5, causal=True, window=29)
    assert not np.array_equal(w29[0], c[0])


def test_visible_key_range_counts():
    assert oracle.visible_key_range(0, 4, 4, False, 0) == (0, 4)
    assert oracle.visible_key_range(2, 4, 4, True, 0) == (0, 3)
    assert oracle.visible_key_range(0, 2, 5, True, 0) == (0, 4)
    assert oracle.visible_key_range(9, 10, 10, True, 4) == (6, 10)
    assert oracle.visible_key_range(1, 10, 10, True, 4) == (0, 2)


def test_rows_heads_batches_subset_matches_full():
    q = _rand((2, 4, 50, 8), 38)
    k = _rand((2, 2, 50, 8), 39)
    v = _rand((2, 2, 50, 8), 40)
    o, lse = oracle.attention(q, k, v, 0.3, causal=True, window=7)
    rows = [0, 3, 17, 49]
    o2, l2 = oracle.attention(q, k, v, 0.3, causal=True, window=7, rows=rows, heads=[1, 3], batches=[1])
    np.testing.assert_array_equal(o2[0], o[1][[1, 3]][:, rows])
    np.testing.assert_array_equal(l2[0], lse[1][[1, 3]][:, rows])


def test_row_chunking_does_not_change_results(monkeypatch):
    import oracle.sdpa as oa
    q = _rand((1, 2, 40, 8), 41)
    k = _rand((1, 1, 40, 8), 42)
    v = _rand((1, 1, 40, 8), 43)
    full = oracle.attention(q, k, v, 0.3, causal=True)
    monkeypatch.setattr(oa, "_MAX_SCORE_ELEMS", 40 * 3)   # 3 rows per chunk
    chunked = oracle.attention(q, k, v, 0.3, causal=True)
    # BLAS may block a 3-row product differently from a 40-row one: rounding only
    np.testing.assert_allclose(full[0], chunked[0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(full[1], chunked[1], rtol=0, atol=1e-14)


# --------------------------------------------------------- paged decode
def _small_decode(seq_lens, Hq=4, Hkv=2, D=8, extra=3, seed=50):
    shape = DecodeShape("t", B=len(seq_lens), Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=40)
    return shape, decode_inputs(shape, seed, seq_lens=list(seq_lens), extra_pages=extra)


def test_paged_decode_equals_contiguous_definition():
    shape, kv = _small_decode([5, 16, 17, 33])
    o, lse = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    for b, n in enumerate(kv.seq_lens.tolist()):
        npg = (n + 15) // 16
        ids = kv.block_table[b, :npg].long()
        kb = kv.k_pages[ids].reshape(npg * 16, shape.Hkv, shape.D)[:n].permute(1, 0, 2)
        vb = kv.v_pages[ids].reshape(npg * 16, shape.Hkv, shape.D)[:n].permute(1, 0, 2)
        ob, lb = _brute(kv.q[b][None, :, None].double().numpy(), kb[None].double().numpy(),
                        vb[None].double().numpy(), 0.3, False, 0)
        np.testing.assert_allclose(o[b], ob[0, :, 0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[b], lb[0, :, 0], rtol=0, atol=1e-13)


def test_paged_decode_values_of_another_width():
    """Keys of width 8 and values of width 5 (latent shapes): each sequence's
    result is the scalar brute force over its gathered cache, one query token
    and the last three (bottom-right causal)."""
    shape = DecodeShape("w", B=3, Hq=4, Hkv=2, D=8, len_lo=1, len_hi=40, Dv=5)
    kv = decode_inputs(shape, 52, seq_lens=[3, 17, 31], extra_pages=2)
    assert kv.v_pages.shape[-1] == 5
    q3 = torch.randn(3, 4, 3, 8, generator=torch.Generator().manual_seed(53)).to(torch.bfloat16)
    for q, multi in ((kv.q, False), (q3, True)):
        o, lse = oracle.paged_decode(q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
        for b, n in enumerate(kv.seq_lens.tolist()):
            npg = (n + 15) // 16
            ids = kv.block_table[b, :npg].long()
            kb = kv.k_pages[ids].reshape(npg * 16, 2, 8)[:n].permute(1, 0, 2)
            vb = kv.v_pages[ids].reshape(npg * 16, 2, 5)[:n].permute(1, 0, 2)
            qb = (q[b][None] if multi else q[b][None, :, None]).double().numpy()
            ob, lb = _brute(qb, kb[None].double().numpy(), vb[None].double().numpy(), 0.3, multi, 0)
            got_o, got_l = (o[b], lse[b]) if multi else (o[b][:, None], lse[b][:, None])
            np.testing.assert_allclose(got_o, ob[0], rtol=0, atol=1e-13)
            np.testing.assert_allclose(got_l, lb[0], rtol=0, atol=1e-13)


def test_paged_decode_invariant_to_page_permutation():
    """Re-scatter the pages to new pool slots and permute the block table to
    match: the result must not change (PagedAttention section of p3)."""
    shape, kv = _small_decode([7, 32, 50, 1], seed=51)
    o, lse = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    perm = torch.randperm(kv.num_pages, generator=torch.Generator().manual_seed(3))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(kv.num_pages)
    k2 = torch.empty_like(kv.k_pages)
    v2 = torch.empty_like(kv.v_pages)
    k2[inv] = kv.k_pages          # page p moves to slot inv[p]
    v2[inv] = kv.v_pages
    t2 = inv[kv.block_table.long()].int()
    o2, l2 = oracle.paged_decode(kv.q, k2, v2, t2, kv.seq_lens, 0.3)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, l2)


def test_paged_decode_empty_sequence():
    shape, kv = _small_decode([0, 3])
    o, lse = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def test_multi_token_decode_rows_equal_truncated_single_token_decode():
    """Row i of a q_len-token decode is the single-token decode of that token
    over the cache truncated just after it (len - q_len + i + 1 tokens): the
    bottom-right causal alignment checked against an independent route."""
    shape, kv = _small_decode([20, 33, 5, 16], Hq=4, Hkv=2, D=8, seed=52)
    q_len = 3
    g = torch.Generator().manual_seed(9)
    qm = torch.randn(shape.B, shape.Hq, q_len, shape.D, generator=g).to(torch.bfloat16)
    o, lse = oracle.paged_decode(qm, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    assert o.shape == (shape.B, shape.Hq, q_len, shape.D) and lse.shape == (shape.B, shape.Hq, q_len)
    for i in range(q_len):
        trunc = (kv.seq_lens - q_len + i + 1).clamp(min=0)
        o1, l1 = oracle.paged_decode(qm[:, :, i], kv.k_pages, kv.v_pages, kv.block_table, trunc, 0.3)
        np.testing.assert_allclose(o[:, :, i], o1, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], l1, rtol=0, atol=1e-13)


def test_multi_token_decode_of_one_token_is_single_token_decode():
    shape, kv = _small_decode([9, 40, 17], seed=53)
    o1, l1 = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    o4, l4 = oracle.paged_decode(kv.q[:, :, None], kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    np.testing.assert_array_equal(o4[:, :, 0], o1)
    np.testing.assert_array_equal(l4[:, :, 0], l1)


def test_multi_token_decode_rows_without_keys():
    """A cache shorter than q_len leaves the first rows with no key at all:
    O = 0, LSE = -inf; the last row still sees the whole cache."""
    shape, kv = _small_decode([2, 6], seed=54)
    q_len = 4
    qm = torch.randn(shape.B, shape.Hq, q_len, shape.D, generator=torch.Generator().manual_seed(4))
    o, lse = oracle.paged_decode(qm, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    assert np.all(o[0, :, :2] == 0) and np.all(np.isneginf(lse[0, :, :2]))
    assert np.all(np.isfinite(lse[0, :, 2:])) and np.all(np.isfinite(lse[1]))
    o1, l1 = oracle.paged_decode(qm[:, :, -1], kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3)
    np.testing.assert_allclose(o[:, :, -1], o1, rtol=0, atol=1e-13)


def test_kv_append_then_decode_equals_contiguous_attention():
    """Append a chunk of new tokens to paged caches, then attend the chunk's
    queries over the cache: equals plain causal attention over the
    contiguous sequence (cached prefix + chunk), bottom-right aligned."""
    g = torch.Generator().manual_seed(11)
    B, Hq, Hkv, D, Ln = 3, 4, 2, 8, 5
    prefix = [7, 16, 0]
    lens = [n + Ln for n in prefix]
    shape = DecodeShape("t", B=B, Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=1)
    kv = decode_inputs(shape, 60, seq_lens=lens, extra_pages=2)
    k_new = torch.randn(B, Hkv, Ln, D, generator=g)
    v_new = torch.randn(B, Hkv, Ln, D, generator=g)
    q = torch.randn(B, Hq, Ln, D, generator=g)
    kp, vp = oracle.kv_append(kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, k_new, v_new)
    o, lse = oracle.paged_decode(q, kp, vp, kv.block_table, kv.seq_lens, 0.3)
    for b in range(B):
        pre_k = oracle.gather_pages(kv.k_pages, kv.block_table[b], prefix[b], 16).transpose(1, 0, 2)
        pre_v = oracle.gather_pages(kv.v_pages, kv.block_table[b], prefix[b], 16).transpose(1, 0, 2)
        kb = np.concatenate([pre_k, k_new[b].double().numpy()], axis=1)[None]
        vb = np.concatenate([pre_v, v_new[b].double().numpy()], axis=1)[None]
        ob, lb = _brute(q[b][None].double().numpy(), kb, vb, 0.3, True, 0)
        np.testing.assert_allclose(o[b], ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], lb[0], rtol=0, atol=1e-12)


def test_kv_append_touches_only_the_new_slots():
    shape, kv = _small_decode([20, 3], Hq=4, Hkv=2, D=8, seed=61)
    Ln = 4
    k_new = torch.randn(2, 2, Ln, 8, generator=torch.Generator().manual_seed(5))
    kp, vp = oracle.kv_append(kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, k_new, k_new)
    changed = np.argwhere(np.any(kp != kv.k_pages.double().numpy(), axis=(2, 3)))
    expect = set()
    for b, n in enumerate(kv.seq_lens.tolist()):
        for t in range(Ln):
            pos = n - Ln + t
            if pos >= 0:
                expect.add((int(kv.block_table[b, pos // 16]), pos % 16))
    assert {tuple(x) for x in changed} <= expect and len(expect) > 0


def test_paged_window_equals_contiguous_window():
    """A sliding window over the paged cache equals the contiguous windowed
    attention of the gathered sequence (bottom-right aligned)."""
    shape, kv = _small_decode([30, 47], Hq=4, Hkv=2, D=8, seed=62)
    q = torch.randn(2, 4, 6, 8, generator=torch.Generator().manual_seed(8))
    o, lse = oracle.paged_decode(q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, 0.3, window=5)
    for b, n in enumerate(kv.seq_lens.tolist()):
        kb = oracle.gather_pages(kv.k_pages, kv.block_table[b], n, 16).transpose(1, 0, 2)[None]
        vb = oracle.gather_pages(kv.v_pages, kv.block_table[b], n, 16).transpose(1, 0, 2)[None]
        ob, lb = _brute(q[b][None].double().numpy(), kb, vb, 0.3, True, 5)
        np.testing.assert_allclose(o[b], ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], lb[0], rtol=0, atol=1e-12)


# ------------------------------------------------------------------ backward
def _autograd_grads(q, k, v, do, scale, causal, window):
    """Gradients by float64 autograd of a separately written forward (masked
    softmax of the scores, GQA by repeating K/V heads)."""
    qt, kt, vt = (torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in (q, k, v))
    B, Hq, Lq, D = qt.shape
    Hkv, Lk = kt.shape[1], kt.shape[2]
    kr = kt.repeat_interleave(Hq // Hkv, dim=1)
    vr = vt.repeat_interleave(Hq // Hkv, dim=1)
    s = scale * qt @ kr.transpose(-1, -2)
    i = torch.arange(Lq)[:, None] + (Lk - Lq)
    j = torch.arange(Lk)[None, :]
    allowed = torch.ones(Lq, Lk, dtype=torch.bool)
    if causal:
        allowed &= j <= i
        if window > 0:
            allowed &= j > i - window
    s = s.masked_fill(~allowed, float("-inf"))
    out = torch.softmax(s, dim=-1) @ vr
    out.backward(torch.tensor(np.asarray(do, dtype=np.float64)))
    return out.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,D,causal,window", [
    (1, 2, 2, 5, 5, 4, False, 0),
    (2, 4, 2, 9, 9, 8, True, 0),
    (1, 6, 2, 7, 11, 4, True, 0),      # Lq < Lk, bottom-right causal
    (1, 4, 1, 12, 12, 8, True, 3),     # MQA, sliding window
])
def test_attention_backward_equals_autograd(B, Hq, Hkv, Lq, Lk, D, causal, window):
    g = torch.Generator().manual_seed(21)
    q = torch.randn(B, Hq, Lq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, Lk, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, Lk, D, generator=g, dtype=torch.float64)
    do = torch.randn(B, Hq, Lq, D, generator=g, dtype=torch.float64)
    o, lse = oracle.attention(q, k, v, 0.4, causal, window)
    dq, dk, dv = oracle.attention_backward(q, k, v, o, do, lse, 0.4, causal, window)
    o_ref, dq_ref, dk_ref, dv_ref = _autograd_grads(q, k, v, do, 0.4, causal, window)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dq, dq_ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, dk_ref, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, dv_ref, rtol=0, atol=1e-11)


def test_attention_backward_finite_differences():
    """Central differences of L = sum(O * dO) against the analytic gradients
    for a few entries of each input."""
    g = torch.Generator().manual_seed(22)
    q = torch.randn(1, 2, 6, 4, generator=g, dtype=torch.float64).numpy()
    k = torch.randn(1, 1, 6, 4, generator=g, dtype=torch.float64).numpy()
    v = torch.randn(1, 1, 6, 4, generator=g, dtype=torch.float64).numpy()
    do = torch.randn(1, 2, 6, 4, generator=g, dtype=torch.float64).numpy()
    o, lse = oracle.attention(q, k, v, 0.5, True, 0)
    dq, dk, dv = oracle.attention_backward(q, k, v, o, do, lse, 0.5, True, 0)

    def loss(q_, k_, v_):
        return float((oracle.attention(q_, k_, v_, 0.5, True, 0)[0] * do).sum())

    eps = 1e-6
    for arr, grad, idx in ((q, dq, (0, 1, 3, 2)), (k, dk, (0, 0, 2, 1)), (v, dv, (0, 0, 4, 3)), (k, dk, (0, 0, 0, 0))):
        plus, minus = arr.copy(), arr.copy()
        plus[idx] += eps
        minus[idx] -= eps
        args_p = [plus if a is arr else a for a in (q, k, v)]
        args_m = [minus if a is arr else a for a in (q, k, v)]
        fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert abs(fd - grad[idx]) < 1e-7, (idx, fd, grad[idx])


def test_attention_backward_gqa_sums_over_the_group():
    """The K/V gradients of a GQA head equal the MHA gradients of the
    repeat_kv-duplicated heads summed over each group."""
    g = torch.Generator().manual_seed(23)
    q = torch.randn(1, 4, 8, 4, generator=g, dtype=torch.float64).numpy()
    k = torch.randn(1, 2, 8, 4, generator=g, dtype=torch.float64).numpy()
    v = torch.randn(1, 2, 8, 4, generator=g, dtype=torch.float64).numpy()
    do = torch.randn(1, 4, 8, 4, generator=g, dtype=torch.float64).numpy()
    o, lse = oracle.attention(q, k, v, 0.5, True, 0)
    dq, dk, dv = oracle.attention_backward(q, k, v, o, do, lse, 0.5, True, 0)
    kr, vr = oracle.repeat_kv(k, 2), oracle.repeat_kv(v, 2)
    o2, lse2 = oracle.attention(q, kr, vr, 0.5, True, 0)
    dq2, dk2, dv2 = oracle.attention_backward(q, kr, vr, o2, do, lse2, 0.5, True, 0)
    np.testing.assert_allclose(dq, dq2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(1, 2, 2, 8, 4).sum(axis=2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(1, 2, 2, 8, 4).sum(axis=2), rtol=0, atol=1e-13)


def test_merge_partials_equals_unsplit():
    """Split the keys into parts, attend each part, merge by LSE: equals
    attention over all keys (float64, to rounding)."""
    q = _rand((1, 3, 1, 8), 60)
    k = _rand((1, 3, 100, 8), 61)
    v = _rand((1, 3, 100, 8), 62)
    full_o, full_l = oracle.attention(q, k, v, 0.4)
    cuts = [0, 13, 13, 64, 100]     # one empty part
    los, oos = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o_s, l_s = oracle.attention(q, k[:, :, a:b], v[:, :, a:b], 0.4)
        los.append(l_s)
        oos.append(o_s)
    o, l = oracle.merge_partials(np.stack(los), np.stack(oos))
    np.testing.assert_allclose(o, full_o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l, full_l, rtol=0, atol=1e-13)
    # all parts empty -> zero output, -inf lse
    o, l = oracle.merge_partials(np.full((2, 3), -np.inf), np.zeros((2, 3, 4)))
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_kv_cache_formula_matches_allocated_pool():
    """p3's formula batch*max_seq_len*n_kv_heads*head_dim*sizeof(half)*2
    equals the bytes of K+V pages when every sequence fills its pages, and
    GQA shrinks it by the group size relative to MHA."""
    lens = [64, 64, 64]
    shape, kv = _small_decode(lens, Hq=8, Hkv=2, D=16, extra=0)
    allocated = (kv.k_pages.numel() + kv.v_pages.numel()) * kv.k_pages.element_size()
    assert oracle.kv_cache_bytes(3, 64, 2, 16, 2) == allocated
    assert oracle.kv_cache_bytes(3, 64, 8, 16) == 4 * oracle.kv_cache_bytes(3, 64, 2, 16)
    # MQA (p2 §2.1): batch x seq_len x 1 x d_k per cache
    assert oracle.kv_cache_bytes(2, 10, 1, 128) == 2 * 10 * 1 * 128 * 2 * 2


# ------------------------------------------------------------------ fp8
def test_e4m3_dequantisation_known_codes():
    """OCP FP8 e4m3 (float8_e4m3fn): 0x38 = 1.0, 0x7E = 448 (max finite),
    0x01 = 2^-9 (smallest subnormal), 0xC0 = -2.0."""
    codes = torch.tensor([0x38, 0x7E, 0x01, 0xC0], dtype=torch.uint8).view(torch.float8_e4m3fn)
    vals = oracle.dequantize_e4m3(codes, 0.5)
    np.testing.assert_array_equal(vals, [0.5, 224.0, 2.0 ** -10, -1.0])


def test_fp8_attention_is_definition_on_dequantised_values():
    shape = PrefillShape("t", B=1, Hq=2, Hkv=2, Lq=9, Lk=9, D=4, causal=True, fp8=True)
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, 3)
    o, lse = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, 0.5, causal=True)
    ob, lb = _brute((q8.double() * sq).numpy(), (k8.double() * sk).numpy(), (v8.double() * sv).numpy(),
                    0.5, True, 0)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-13)
    # quantisation scale: amax maps to 448
    assert abs(float((q8.float().abs().max()))) == 448.0


def test_e5m2_dequantisation_known_codes():
    """OCP FP8 e5m2 (float8_e5m2, 5 exponent bits with bias 15, 2 mantissa
    bits): 0x3C = 1.0, 0x7B = 1.75 * 2^15 = 57344 (max finite), 0x01 =
    2^-16 (smallest subnormal), 0xC0 = -2.0."""
    codes = torch.tensor([0x3C, 0x7B, 0x01, 0xC0], dtype=torch.uint8).view(torch.float8_e5m2)
    vals = oracle.dequantize_e5m2(codes, 0.5)
    np.testing.assert_array_equal(vals, [0.5, 28672.0, 2.0 ** -17, -1.0])


def test_e5m2_attention_is_definition_on_dequantised_values():
    shape = PrefillShape("t", B=1, Hq=2, Hkv=1, Lq=7, Lk=11, D=4, causal=True, fp8=True)
    q8, k8, v8, sq, sk, sv = prefill_inputs_fp8(shape, 4, fmt="e5m2")
    assert q8.dtype == torch.float8_e5m2
    o, lse = oracle.attention_fp8(q8, k8, v8, sq, sk, sv, 0.5, causal=True, window=3)
    ob, lb = _brute((q8.double() * sq).numpy(), (k8.double() * sk).numpy(), (v8.double() * sv).numpy(),
                    0.5, True, 3)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-13)
    # quantisation scale: amax maps to the largest finite e5m2 value
    assert float(q8.float().abs().max()) == 57344.0


def test_tiny_workload_golden_rows():
    """Regression fixture written by tests/golden/make_golden.py (which
    calls only the oracle): selected rows of the tiny MHA workload."""
    import json
    import os
    from workloads import TINY_MHA, seed_of
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_mha_rows.json")
    gold = json.load(open(path))
    q, k, v = prefill_inputs(TINY_MHA, seed_of(0))
    o, lse = oracle.attention(q, k, v, TINY_MHA.scale, False, rows=gold["rows"])
    np.testing.assert_allclose(o[0, :, :, :4], np.array(gold["o_first4"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], np.array(gold["lse"]), rtol=0, atol=1e-12)

"""Float64 reference implementations (test infrastructure only; see the
package docstring).  Inputs may be torch tensors of any float dtype (bf16,
float8_e4m3fn, ...) or numpy arrays; they are converted exactly to float64.

Page short names used in citations:
  * p1 -- "注意力机制深度优化" (kler.cn)
  * p2 -- MQA / GQA / Flash Attention article (tqpw.cn), by section number
  * p3 -- "LLM 中的 Attention 实现及优化" (zeeklog.com)
  * p5 -- "003-注意力机制详解：从基础Attention到DeepSeek的优化策略" (lakecityint.com)
"""
from __future__ import annotations

import numpy as np

try:  # torch is only needed to read torch tensors (bf16 / fp8 storage)
    import torch
except ImportError:  # pragma: no cover
    torch = None

# Largest number of score entries materialised at once (8 B each): 2 GB.
_MAX_SCORE_ELEMS = 1 << 28


def _f64(x) -> np.ndarray:
    if torch is not None and isinstance(x, torch.Tensor):
        return x.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def visible_key_range(i: int, Lq: int, Lk: int, causal: bool, window: int):
    """Half-open range [lo, hi) of keys that query row ``i`` attends to.

    * non-causal: all ``Lk`` keys.
    * causal: the upper-right triangle is masked (p1 §一.2 "Causal Mask
      计算优化").  With Lq != Lk the triangle is aligned to the bottom-right
      corner, so query ``i`` sees keys ``0 .. i + (Lk - Lq)``; this is the
      reading that reduces to "keys 0..i" when Lq == Lk and to "every cached
      key" for a single decode query.
    * window W > 0 (causal only): each token sees at most W tokens, itself
      included -- keys ``max(0, i' - W + 1) .. i'`` with ``i' = i + Lk - Lq``
      (sliding-window section of p3; banded mask of p5 §三.2).
    """
    if not causal:
        return 0, Lk
    hi = min(max(i + (Lk - Lq) + 1, 0), Lk)
    lo = max(0, hi - window) if window > 0 else 0
    return lo, hi


def _row_ranges(Lq, Lk, causal, window, rows):
    lo = np.empty(len(rows), dtype=np.int64)
    hi = np.empty(len(rows), dtype=np.int64)
    for n, i in enumerate(rows):
        lo[n], hi[n] = visible_key_range(int(i), Lq, Lk, causal, window)
    return lo, hi


def _attend_rows(q_rows, k, v, scale, lo, hi):
    """Plain definition for a set of query rows of one head.

    q_rows [R, D]; k, v [Lk, Dk] / [Lk, Dv]; lo/hi the visible ranges.
    Returns O [R, Dv] and LSE [R] (natural log of the scaled logits).
    Safe softmax: the row max is subtracted before exponentiating (p5 §一
    ``safe_softmax``)."""
    R = q_rows.shape[0]
    Dv = v.shape[1]
    o = np.zeros((R, Dv), dtype=np.float64)
    lse = np.full(R, -np.inf, dtype=np.float64)
    if R == 0:
        return o, lse
    c0 = int(lo.min())
    c1 = int(hi.max())
    if c1 <= c0:
        return o, lse
    s = scale * (q_rows @ k[c0:c1].T)                     # [R, c1-c0]
    cols = np.arange(c0, c1)[None, :]
    masked = (cols < lo[:, None]) | (cols >= hi[:, None])
    s[masked] = -np.inf
    m = s.max(axis=1)
    has = np.isfinite(m)
    if not has.any():
        return o, lse
    sh = s[has] - m[has][:, None]
    e = np.exp(sh)
    denom = e.sum(axis=1)
    lse[has] = m[has] + np.log(denom)
    o[has] = (e / denom[:, None]) @ v[c0:c1]
    return o, lse


def attention(q, k, v, scale: float, causal: bool = False, window: int = 0,
              rows=None, heads=None, batches=None):
    """O = softmax(scale * Q K^T + mask) V and the per-row LSE, in float64.

    Layout ``[B, H, L, D]`` (batch, heads, seqlen, head_dim), the layout of the
    HF-Llama ``view(...).transpose(1, 2)`` lines in the GQA section of p3.
    ``q`` has Hq heads and ``k``/``v`` Hkv heads with ``Hq % Hkv == 0``; query
    head ``h`` uses key/value head ``h // (Hq // Hkv)`` -- the grouping of
    p2 §3.1 (h heads in g groups, ``assert h % g == 0``) and MQA (one K/V head
    for all query heads, p2 §2.1).  The full score matrix is materialised
    (p5 §一 ``attention_naive``), in row chunks only to bound memory.

    ``rows``/``heads``/``batches`` optionally restrict which outputs are
    computed (each output row depends only on its own query row), for
    sampled parity at full size.  Returns (O [B', H', R, Dv], LSE [B', H', R]).
    """
    q = _f64(q) if not isinstance(q, np.ndarray) or q.dtype != np.float64 else q
    k = _f64(k) if not isinstance(k, np.ndarray) or k.dtype != np.float64 else k
    v = _f64(v) if not isinstance(v, np.ndarray) or v.dtype != np.float64 else v
    B, Hq, Lq, D = q.shape
    Bk, Hkv, Lk, Dk = k.shape
    assert Bk == B and Dk == D and v.shape[:3] == (B, Hkv, Lk)
    assert Hkv >= 1 and Hq % Hkv == 0, "query heads must split evenly into K/V groups"
    if window > 0:
        assert causal, "a sliding window is defined on top of the causal mask"
    group = Hq // Hkv
    rows = np.arange(Lq) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = range(Hq) if heads is None else list(heads)
    batches = range(B) if batches is None else list(batches)
    Dv = v.shape[3]
    out = np.zeros((len(batches), len(heads), len(rows), Dv), dtype=np.float64)
    lse = np.full((len(batches), len(heads), len(rows)), -np.inf, dtype=np.float64)
    lo_all, hi_all = _row_ranges(Lq, Lk, causal, window, rows)
    chunk = max(1, _MAX_SCORE_ELEMS // max(Lk, 1))
    for bi, b in enumerate(batches):
        for hi_, h in enumerate(heads):
            kvh = h // group
            for r0 in range(0, len(rows), chunk):
                sel = slice(r0, r0 + chunk)
                o_c, l_c = _attend_rows(q[b, h, rows[sel]], k[b, kvh], v[b, kvh], scale,
                                        lo_all[sel], hi_all[sel])
                out[bi, hi_, sel] = o_c
                lse[bi, hi_, sel] = l_c
    return out, lse


def dequantize_e4m3(x8, s: float) -> np.ndarray:
    """Value of a per-tensor scaled e4m3 tensor: float64(x8) * s (the
    ``torch_dtype=torch.float8_e4m3fn`` format named in p1 §一.1)."""
    return _f64(x8) * float(s)


def dequantize_e5m2(x8, s: float) -> np.ndarray:
    """Value of a per-tensor scaled e5m2 tensor: float64(x8) * s (the
    ``torch_dtype=torch.float8_e5m2`` format named in p1 §四.2).  Both 8-bit
    formats convert exactly to float64; the two functions differ only in the
    format they are pinned against."""
    return _f64(x8) * float(s)


def attention_backward(q, k, v, o, do, lse, scale: float, causal: bool = False, window: int = 0):
    """Gradients of O = softmax(scale * Q K^T + mask) V with respect to Q, K
    and V, in float64, from the forward's O and per-row LSE.

    Follows the recomputation of the tqpw.cn article §4.1 (the backward pass
    recomputes the attention weights instead of storing them; p5 §一 notes the
    stored score matrix as the cost being avoided): P = exp(scale * Q K^T -
    LSE) row by row (masked entries 0), then with Dvec = rowsum(dO * O)

        dV = P^T dO,   dP = dO V^T,   dS = P * (dP - Dvec),
        dQ = scale * dS K,   dK = scale * dS^T Q.

    GQA/MQA: the K/V gradients of a K/V head sum over the query heads of its
    group.  Layout [B, H, L, D] as ``attention``.  Returns (dQ, dK, dV)."""
    q, k, v, o, do = (_f64(x) for x in (q, k, v, o, do))
    lse = _f64(lse)
    B, Hq, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    group = Hq // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    lo_all, hi_all = _row_ranges(Lq, Lk, causal, window, np.arange(Lq))
    chunk = max(1, _MAX_SCORE_ELEMS // max(Lk, 1))
    cols = np.arange(Lk)[None, :]
    for b in range(B):
        for h in range(Hq):
            kvh = h // group
            for r0 in range(0, Lq, chunk):
                r1 = min(Lq, r0 + chunk)
                lo, hi = lo_all[r0:r1], hi_all[r0:r1]
                s = scale * (q[b, h, r0:r1] @ k[b, kvh].T)
                masked = (cols < lo[:, None]) | (cols >= hi[:, None])
                li = lse[b, h, r0:r1]
                p_ = np.zeros_like(s)
                live = np.isfinite(li)
                p_[live] = np.exp(s[live] - li[live][:, None])
                p_[masked] = 0.0
                dvec = (do[b, h, r0:r1] * o[b, h, r0:r1]).sum(axis=1)
                dv[b, kvh] += p_.T @ do[b, h, r0:r1]
                dp = do[b, h, r0:r1] @ v[b, kvh].T
                ds = p_ * (dp - dvec[:, None])
                dq[b, h, r0:r1] = scale * (ds @ k[b, kvh])
                dk[b, kvh] += scale * (ds.T @ q[b, h, r0:r1])
    return dq, dk, dv


def attention_fp8(q8, k8, v8, q_scale, k_scale, v_scale, scale: float,
                  causal: bool = False, window: int = 0, **kw):
    """Attention on 8-bit inputs (e4m3 or e5m2, per-tensor scales): the plain
    definition applied to the exact dequantised values, so the oracle
    measures kernel error and not quantisation error."""
    deq = dequantize_e5m2 if (torch is not None and isinstance(q8, torch.Tensor)
                              and q8.dtype == torch.float8_e5m2) else dequantize_e4m3
    return attention(deq(q8, q_scale), deq(k8, k_scale), deq(v8, v_scale), scale, causal, window, **kw)


def online_softmax_attention(q, k, v, scale: float, causal: bool = False, window: int = 0,
                             block_q: int = 128, block_k: int = 128):
    """The tiled FlashAttention forward of p5 §二, step by step, in float64.

    For each query block: ``acc = 0``, ``max_vec = -inf``, ``sum_vec = 0``;
    for each key/value block: scores = scale * Qi Kj^T (masked entries -inf),
    ``new_max = max(max_vec, rowmax(scores))``, rescale factor
    ``exp(max_vec - new_max)`` applied to ``acc`` and ``sum_vec``,
    ``exp_scores = exp(scores - new_max)``, ``acc += exp_scores Vj``,
    ``sum_vec += rowsum(exp_scores)``, ``max_vec = new_max``; finally
    ``output = acc / sum_vec``.  The max is taken per row (the reading of the
    garbled ``scores_ij.max()``).  Rows that have seen no visible key yet keep
    ``max_vec = -inf`` and contribute nothing (guard for masks, which the
    page's sketch leaves out).  Also returns ``LSE = max_vec + log(sum_vec)``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    group = Hq // Hkv
    Dv = v.shape[3]
    out = np.zeros((B, Hq, Lq, Dv))
    lse = np.full((B, Hq, Lq), -np.inf)
    ranges = [visible_key_range(i, Lq, Lk, causal, window) for i in range(Lq)]
    lo_all = np.array([r[0] for r in ranges], dtype=np.int64)
    hi_all = np.array([r[1] for r in ranges], dtype=np.int64)
    for b in range(B):
        for h in range(Hq):
            kvh = h // group
            for i0 in range(0, Lq, block_q):
                qi = q[b, h, i0:i0 + block_q]
                lo = lo_all[i0:i0 + block_q, None]
                hi = hi_all[i0:i0 + block_q, None]
                acc = np.zeros((qi.shape[0], Dv))
                max_vec = np.full(qi.shape[0], -np.inf)
                sum_vec = np.zeros(qi.shape[0])
                for j0 in range(0, Lk, block_k):
                    kj = k[b, kvh, j0:j0 + block_k]
                    vj = v[b, kvh, j0:j0 + block_k]
                    scores = scale * (qi @ kj.T)
                    cols = np.arange(j0, j0 + kj.shape[0])[None, :]
                    scores[(cols < lo) | (cols >= hi)] = -np.inf
                    new_max = np.maximum(max_vec, scores.max(axis=1))
                    live = np.isfinite(new_max)
                    factor = np.ones_like(new_max)
                    factor[live] = np.exp(max_vec[live] - new_max[live])
                    acc *= factor[:, None]
                    sum_vec *= factor
                    exp_scores = np.zeros_like(scores)
                    exp_scores[live] = np.exp(scores[live] - new_max[live][:, None])
                    acc += exp_scores @ vj
                    sum_vec += exp_scores.sum(axis=1)
                    max_vec = new_max
                ok = sum_vec > 0
                out[b, h, i0:i0 + block_q][ok] = acc[ok] / sum_vec[ok][:, None]
                lse_blk = np.full(qi.shape[0], -np.inf)
                lse_blk[ok] = max_vec[ok] + np.log(sum_vec[ok])
                lse[b, h, i0:i0 + block_q] = lse_blk
    return out, lse


def repeat_kv(x, n_rep: int) -> np.ndarray:
    """Duplicate each K/V head ``n_rep`` times along the head axis:
    (batch, num_kv_heads, seqlen, head_dim) -> (batch, num_kv_heads*n_rep,
    seqlen, head_dim), heads of one group adjacent (``repeat_kv`` in the GQA
    section of p3)."""
    x = _f64(x)
    return np.repeat(x, n_rep, axis=1)


def gather_pages(pages, block_table_row, seq_len: int, page_size: int) -> np.ndarray:
    """Contiguous K (or V) of one sequence, [seq_len, Hkv, D], read from a
    pool of fixed-size pages through its block-table row (PagedAttention:
    non-contiguous small-block storage, PagedAttention section of p3)."""
    pages = _f64(pages)
    n_pages = (seq_len + page_size - 1) // page_size
    table = np.asarray(_f64(block_table_row), dtype=np.int64)[:n_pages]
    if n_pages == 0:
        return np.zeros((0,) + pages.shape[2:], dtype=np.float64)
    flat = pages[table].reshape((n_pages * page_size,) + pages.shape[2:])
    return flat[:seq_len]


def kv_append(k_pages, v_pages, block_table, seq_lens, k_new, v_new, page_size: int = 16):
    """Write the K/V of each sequence's newest tokens into its pages.

    k_new, v_new [B, Hkv, L_new, D]; seq_lens [B] counts the cached tokens
    with the new ones included, so token t of sequence b goes to position
    ``seq_lens[b] - L_new + t``: page ``block_table[b, pos // page_size]``,
    slot ``pos % page_size`` (the KV-cache layout of the PagedAttention
    section of p3).  Positions below 0 are skipped.  Returns new pools
    (float64); nothing else of the pools changes."""
    kp = _f64(k_pages).copy()
    vp = _f64(v_pages).copy()
    kn, vn = _f64(k_new), _f64(v_new)
    table = np.asarray(_f64(block_table), dtype=np.int64)
    B, Hkv, Ln, D = kn.shape
    for b in range(B):
        n = int(np.asarray(_f64(seq_lens))[b])
        for t in range(Ln):
            pos = n - Ln + t
            if pos < 0:
                continue
            page = table[b, pos // page_size]
            kp[page, pos % page_size] = kn[b, :, t]
            vp[page, pos % page_size] = vn[b, :, t]
    return kp, vp


def paged_decode(q, k_pages, v_pages, block_table, seq_lens, scale: float, page_size: int = 16, window: int = 0):
    """Decode over a paged KV cache.

    q [B, Hq, D] (one new token per sequence) or [B, Hq, q_len, D] (the last
    q_len tokens of each sequence, e.g. draft tokens to verify); pools
    [num_pages, page_size, Hkv, D]; block_table [B, max_pages]; seq_lens [B]
    (cached tokens, the q_len new ones included).  Each sequence's cache is
    gathered into the contiguous ``[B, Hkv, seq_len, D]`` view (KV-cache
    section of p3) and the plain definition is applied: with one query row it
    sees every cached key; with q_len rows, row i is the token at position
    seq_len - q_len + i and sees the keys up to it (the causal mask aligned at
    the bottom-right corner); ``window`` > 0 further limits every row to its
    last ``window`` keys (sliding window of p3).  Returns O [B, Hq, Dv] and
    LSE [B, Hq] (or [B, Hq, q_len, Dv] and [B, Hq, q_len]); a row without keys
    gives O = 0 and LSE = -inf.  The same call defines chunked prefill over
    a paged cache (q_len in the hundreds or thousands)."""
    q = _f64(q)
    multi = q.ndim == 4
    if not multi:
        q = q[:, :, None, :]
    B, Hq, Lq, D = q.shape
    lens = [int(x) for x in np.asarray(_f64(seq_lens))]
    Dv = _f64(v_pages[:1]).shape[-1] if len(v_pages) else D
    out = np.zeros((B, Hq, Lq, Dv))
    lse = np.full((B, Hq, Lq), -np.inf)
    kp, vp = _f64(k_pages), _f64(v_pages)
    table = np.asarray(_f64(block_table), dtype=np.int64)
    for b in range(B):
        kb = gather_pages(kp, table[b], lens[b], page_size)      # [len, Hkv, D]
        vb = gather_pages(vp, table[b], lens[b], page_size)
        kb = kb.transpose(1, 0, 2)[None]                          # [1, Hkv, len, D]
        vb = vb.transpose(1, 0, 2)[None]
        o_b, l_b = attention(q[b][None], kb, vb, scale, causal=multi or window > 0, window=window)
        out[b] = o_b[0]
        lse[b] = l_b[0]
    if not multi:
        return out[:, :, 0], lse[:, :, 0]
    return out, lse


def merge_partials(lse_parts, o_parts):
    """Merge attention computed separately over disjoint key subsets.

    ``lse_parts`` [S, ...] and ``o_parts`` [S, ..., Dv] are the LSE and the
    normalised output of each part.  The result is the attention over the
    union: ``LSE = log sum_s exp(lse_s)`` and ``O = sum_s exp(lse_s - LSE) o_s``.
    This is the same rescaling the online recurrence of p5 §二 applies between
    blocks, taken in one step; parts with no keys (``lse = -inf``) weigh 0."""
    lse_parts = _f64(lse_parts)
    o_parts = _f64(o_parts)
    m = lse_parts.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.exp(lse_parts - m_safe[None])                  # exp(-inf) = 0
    tot = w.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, tot, 1.0)), -np.inf)
    wn = np.where(finite[None], w / np.where(finite, tot, 1.0)[None], 0.0)
    o = (wn[..., None] * o_parts).sum(axis=0)
    return o, lse


def kv_cache_bytes(batch: int, max_seq_len: int, n_kv_heads: int, head_dim: int,
                   elem_bytes: int = 2) -> int:
    """KV-cache size formula of p3 (KV-cache section):
    ``batch * max_seq_len * n_kv_heads * head_dim * sizeof(half) * 2``
    (K and V).  With n_kv_heads = n_heads it is the MHA figure; GQA divides it
    by the group size."""
    return batch * max_seq_len * n_kv_heads * head_dim * elem_bytes * 2


"""Float64 CPU oracle for the attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call, link
or execute anything in this package: only ``tests/``, the smoke check in
``__graft_entry__.py`` and the CPU-baseline leg of ``bench.py`` use it.  It
shares no code with the CUDA library (``attention_flash_attn_02_b200``) and
neither imports the other; the only common module is ``workloads`` (seeded
random inputs, no attention arithmetic).

What it computes is the plain definition of softmax attention, written out in
float64 on the exact input values:

    S = scale * Q K^T (+ mask),  LSE_i = log sum_j exp(S_ij),
    O_i = sum_j exp(S_ij - LSE_i) V_j

-- the ``attention_naive`` + ``safe_softmax`` listing of section 一 of the
page "003-注意力机制详解：从基础Attention到DeepSeek的优化策略" (lakecityint.com),
with masks, GQA/MQA head sharing, paged KV gathering and split merging added
as the other pages define them.  Each function cites the passage it follows.

Parity pins (``tests/test_oracle.py``) tie every function to something other
than itself: brute-force scalar loops, ``torch``'s float64 SDPA library
routine, closed forms (identical keys, one dominant logit, window W = 1),
GQA == MHA after ``repeat_kv``, window >= L == causal, block-table
permutation invariance, split-merge == unsplit, and the KV-cache size
formula against allocated bytes.  No function here is "parity unpinned".
"""
from .sdpa import (  # noqa: F401
    attention,
    attention_backward,
    attention_fp8,
    dequantize_e4m3,
    dequantize_e5m2,
    gather_pages,
    kv_cache_bytes,
    merge_partials,
    online_softmax_attention,
    kv_append,
    paged_decode,
    repeat_kv,
    visible_key_range,
)

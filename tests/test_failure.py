"""Failure detection without a GPU fault.

Every wait inside the kernels is bounded.  With the ATTN_DEBUG_STALL testing
hook the TMA producers issue no loads, so the waits on their barriers run out
(after a short limit set here); the kernels then unwind, release TMEM and
return, and attn_last_device_error() reports ATTN_ERR_TIMEOUT.  The tests also
check that the CUDA context stays usable: the next normal call is correct.
No test traps, faults or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import DecodeShape, PrefillShape, decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000  # 20 ms per wait while the hook is on


def _prefill(lib):
    shape = PrefillShape("f", 1, 4, 2, 300, 300, 128, True)
    q, k, v = prefill_inputs(shape, 3)
    o, lse = lib.attn_fwd(q.cuda(), k.cuda(), v.cuda(), shape.scale, True, 0)
    return shape, (q, k, v), o, lse


def _decode(lib):
    shape = DecodeShape("f", B=3, Hq=32, Hkv=1, D=128, len_lo=1, len_hi=1)
    kv = decode_inputs(shape, 4, seq_lens=[40, 700, 5])
    d = {n: getattr(kv, n).cuda() for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
    o, lse = lib.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], shape.scale)
    return shape, kv, o, lse


@pytest.mark.parametrize("run", [_prefill, _decode], ids=["prefill", "decode"])
def test_bounded_wait_reports_timeout_and_context_survives(lib, run):
    assert lib.attn_last_device_error() == 0
    prev = lib.attn_set_debug(lib.ATTN_DEBUG_STALL, LIMIT_NS)
    try:
        run(lib)
        assert lib.attn_last_device_error() == lib.ATTN_ERR_TIMEOUT
        assert lib.attn_last_device_error() == 0  # the status word was cleared by the read
    finally:
        lib.attn_set_debug(prev & ~lib.ATTN_DEBUG_STALL, 0)
    # the context is intact: a normal call runs and matches the oracle
    shape, inputs, o, lse = run(lib)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    if run is _prefill:
        o_ref, l_ref = oracle.attention(*inputs, shape.scale, True)
    else:
        kv = inputs
        o_ref, l_ref = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    assert np.abs(o.double().cpu().numpy() - o_ref).max() <= 1e-2
    assert np.abs(lse.double().cpu().numpy() - l_ref).max() <= 1e-3

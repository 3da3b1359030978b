"""The allocation-free decode entry point (attn_decode_paged_noalloc).

It serves callers that cannot allocate device memory when they run decode:
its scratch is a fixed array inside the library instead of a caller-provided
workspace.  These GPU tests call it through the C ABI, twice in a row (the
array keeps the first call's contents), and compare its output with the
float64 oracle and with the regular entry point's on the same inputs, within
the parity tolerance used for decode everywhere else.  The file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from workloads import MQA_DECODE, DecodeShape, decode_inputs, seed_of

pytestmark = pytest.mark.gpu

O_TOL = 1e-2
LSE_TOL = 1e-3


def _noalloc_call(cdll, d, shape, o, lse):
    num_pages, page_size, Hkv, _ = d["k_pages"].shape
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return cdll.attn_decode_paged_noalloc(
        p(d["q"]), p(d["k_pages"]), p(d["v_pages"]), p(d["block_table"]), p(d["seq_lens"]), p(o), p(lse),
        shape.B, shape.Hq, Hkv, shape.D, page_size, num_pages, d["block_table"].shape[1],
        ctypes.c_float(shape.scale), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("which", ["workload", "edge"])
def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls(lib, which):
    cdll = lib.load()
    if which == "workload":
        shape = MQA_DECODE
        kv = decode_inputs(shape, seed_of(2))
    else:
        shape = DecodeShape("edge", B=5, Hq=32, Hkv=4, D=128, len_lo=1, len_hi=1)
        kv = decode_inputs(shape, 17, seq_lens=[1, 0, 700, 16, 4097], extra_pages=3)
    d = {n: getattr(kv, n).cuda() for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
    ref_o, ref_l = lib.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                                         shape.scale)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    fin_ref = np.isfinite(l_ref)
    for _ in range(2):
        o = torch.full_like(ref_o, float("nan"))
        lse = torch.full_like(ref_l, float("nan"))
        st = _noalloc_call(cdll, d, shape, o, lse)
        assert st == 0, lib.attn_status_str(st)
        torch.cuda.synchronize()
        assert lib.attn_last_device_error() == 0
        do = (o.double() - ref_o.double()).abs().max().item()
        fin = torch.isfinite(ref_l)
        assert torch.equal(torch.isfinite(lse), fin)
        dl = (lse[fin].double() - ref_l[fin].double()).abs().max().item() if fin.any() else 0.0
        assert do <= O_TOL and dl <= LSE_TOL, (do, dl)
        # against the oracle
        on, ln = o.double().cpu().numpy(), lse.double().cpu().numpy()
        assert np.array_equal(np.isfinite(ln), fin_ref)
        eo = np.abs(on - o_ref).max()
        el = np.abs(ln[fin_ref] - l_ref[fin_ref]).max() if fin_ref.any() else 0.0
        assert eo <= O_TOL and el <= LSE_TOL, (eo, el)


def test_noalloc_call_allocates_no_device_memory(lib):
    """After the set-up call (the first on the device, here with B = 0, which
    loads the array), a decode call leaves the device's free memory and the
    caching allocator's counters unchanged."""
    cdll = lib.load()
    shape = DecodeShape("alloc", B=8, Hq=32, Hkv=1, D=128, len_lo=100, len_hi=3000)
    kv = decode_inputs(shape, 18)
    d = {n: getattr(kv, n).cuda() for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
    o = torch.empty_like(d["q"])
    lse = torch.empty(d["q"].shape[:2], dtype=torch.float32, device="cuda")
    setup = DecodeShape("setup", B=0, Hq=32, Hkv=1, D=128, len_lo=1, len_hi=1)
    assert _noalloc_call(cdll, d, setup, o, lse) == 0
    assert _noalloc_call(cdll, d, shape, o, lse) == 0      # first real call: kernels loaded
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    stats0 = torch.cuda.memory_stats()
    assert _noalloc_call(cdll, d, shape, o, lse) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    stats1 = torch.cuda.memory_stats()
    assert lib.attn_last_device_error() == 0
    assert free1 == free0
    for key in ("allocation.all.allocated", "segment.all.allocated", "reserved_bytes.all.current"):
        assert stats1.get(key, 0) == stats0.get(key, 0), key


def test_noalloc_checks_arguments_like_the_workspace_entry_point(lib):
    """An unsupported shape is refused as attn_decode_paged refuses it, even
    when its scratch would also be too large for the array."""
    cdll = lib.load()
    fake = ctypes.c_void_p(0x10000)
    B, Hq, D, max_pages = 256, 64, 96, 4096         # D = 96: not built
    st = cdll.attn_decode_paged_noalloc(fake, fake, fake, fake, fake, fake, fake, B, Hq, 1, D, 16, 10,
                                        max_pages, ctypes.c_float(0.1), ctypes.c_void_p(0))
    assert st == lib.ATTN_ERR_UNSUPPORTED


def test_noalloc_rejects_sizes_beyond_its_array(lib):
    cdll = lib.load()
    limit = 32 << 20
    B, Hq, D, max_pages = 256, 64, 128, 4096
    assert lib.attn_decode_workspace_bytes(B, Hq, max_pages, D) > limit
    fake = ctypes.c_void_p(0x10000)
    st = cdll.attn_decode_paged_noalloc(fake, fake, fake, fake, fake, fake, fake, B, Hq, 1, D, 16, 10,
                                        max_pages, ctypes.c_float(0.1), ctypes.c_void_p(0))
    assert st == lib.ATTN_ERR_INVALID
    msg = lib.attn_last_error_message()
    assert "scratch" in msg and "invalid argument" not in msg

"""GPU parity of attn_fwd_mla: attention whose queries and keys have width
D_qk and whose values have width D_v (each 64..256), the shapes of attention
in a latent space (latent projection of the Flash MLA page, §2.1), against
the float64 oracle on the same seeded inputs.

Tolerances are those of the bf16 workloads: max |O - O_ref| <= 1e-2, mean
<= 1e-3, |LSE - LSE_ref| <= 1e-3 -- except where rounding the exact O to
bf16 alone moves it further: bf16 keeps 8 significant bits, so for |O| in
[4, 8) half an ulp is 1.56e-2, and rows that average two values can reach
such |O|.  There each element may differ from the exact value by the rounding
of that value to bf16 plus 4e-3, i.e. the kernel stays within 4e-3 of the
correctly rounded output.  The oracle's definition is independent of the
widths; its brute-force pins already use D_v != D.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import LATENT_192_128, LATENT_256, PrefillShape, prefill_inputs, seed_of

pytestmark = pytest.mark.gpu

TOL = (1e-2, 1e-3)
LSE_TOL = 1e-3


def _check(o, lse, o_ref, l_ref, what):
    o = o.double().cpu().numpy()
    lse = lse.double().cpu().numpy()
    d = np.abs(o - o_ref)
    rounding = np.abs(torch.from_numpy(o_ref).to(torch.bfloat16).double().numpy() - o_ref)
    bound = np.maximum(TOL[0], rounding + 4e-3)
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(lse), fin), f"{what}: LSE finiteness differs"
    dl = np.abs(lse[fin] - l_ref[fin]).max() if fin.any() else 0.0
    worst = np.unravel_index(np.argmax(d - bound), d.shape)
    assert np.all(d <= bound) and d.mean() <= TOL[1] and dl <= LSE_TOL, \
        f"{what}: max {d.max():.3e} (at {worst}: {d[worst]:.3e} > {bound[worst]:.3e}) mean {d.mean():.3e} lse {dl:.3e}"
    if (~fin).any():
        assert np.all(o[~fin] == 0)


def _run(lib, shape, seed, k=None, v=None):
    q, k0, v0 = prefill_inputs(shape, seed)
    k = k0 if k is None else k
    v = v0 if v is None else v
    o, lse = lib.attn_fwd_mla(q.cuda(), k.cuda(), v.cuda(), shape.scale, shape.causal, shape.window)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    assert o.shape[-1] == shape.dv
    return (q, k0, v0), o, lse


WIDTHS = [(64, 64), (128, 128), (192, 128), (256, 256), (256, 128), (128, 256), (64, 192), (192, 192)]
SHAPES = [
    (1, 2, 2, 300, 300, True, 0),      # ragged tail, causal
    (1, 4, 1, 129, 129, False, 0),     # MQA, non-causal
    (2, 8, 2, 200, 500, True, 0),      # GQA, Lq < Lk (bottom-right)
    (1, 2, 2, 150, 70, True, 0),       # Lq > Lk: first rows see no key
    (1, 4, 2, 400, 400, True, 2),      # rows of two keys
    (1, 3, 1, 333, 333, True, 100),    # group of 3, window
]


@pytest.mark.parametrize("dqk,dv", WIDTHS)
@pytest.mark.parametrize("B,Hq,Hkv,Lq,Lk,causal,window", SHAPES)
def test_latent_sweep(lib, dqk, dv, B, Hq, Hkv, Lq, Lk, causal, window):
    shape = PrefillShape("latent", B, Hq, Hkv, Lq, Lk, dqk, causal, window=window, Dv=dv)
    (q, k, v), o, lse = _run(lib, shape, 41 + dqk + dv + Lq + window)
    o_ref, l_ref = oracle.attention(q, k, v, shape.scale, causal, window)
    _check(o, lse, o_ref, l_ref, str(shape))


@pytest.mark.parametrize("dqk,dv", [(64, 64), (256, 256), (192, 128)])
def test_latent_tiny_rows(lib, dqk, dv):
    """One to a few query rows and keys: single-block units."""
    for L in (1, 2, 63, 64, 65):
        shape = PrefillShape("tiny", 1, 2, 1, L, L, dqk, True, Dv=dv)
        (q, k, v), o, lse = _run(lib, shape, 7 + L)
        o_ref, l_ref = oracle.attention(q, k, v, shape.scale, True, 0)
        _check(o, lse, o_ref, l_ref, str(shape))


@pytest.mark.parametrize("shape,idx", [(LATENT_192_128, 1), (LATENT_256, 3)])
def test_latent_full_size(lib, shape, idx):
    """The latent workloads (B4 Hq32 Hkv8 L4096 causal, D_qk/D_v 192/128 and
    256/256): every row of batch 0's first K/V group (heads 0-3) and of the
    last batch's last group (heads 28-31), in row chunks."""
    (q, k, v), o, lse = _run(lib, shape, seed_of(idx))
    for b, heads in ((0, [0, 1, 2, 3]), (shape.B - 1, [28, 29, 30, 31])):
        for r0 in range(0, shape.Lq, 2048):
            rows = list(range(r0, r0 + 2048))
            o_ref, l_ref = oracle.attention(q, k, v, shape.scale, True, 0, rows=rows, heads=heads, batches=[b])
            _check(o[b][heads][:, rows], lse[b][heads][:, rows], o_ref[0], l_ref[0], f"{shape.name} b{b} r{r0}")


def test_latent_never_visible_blocks_are_not_read(lib):
    """Keys no row can see hold NaN (0 * NaN would reach O if multiplied):
    Lq = 300 over Lk = 1000 with a window of 189, so keys 0..511 (eight
    64-key blocks) are invisible to every row."""
    shape = PrefillShape("nan", 1, 4, 2, 300, 1000, 256, True, window=189, Dv=128)
    q, k, v = prefill_inputs(shape, 43)
    lo0, _ = oracle.visible_key_range(0, 300, 1000, True, 189)
    assert lo0 == 512
    kn, vn = k.clone(), v.clone()
    kn[:, :, :lo0] = float("nan")
    vn[:, :, :lo0] = float("nan")
    _, o, lse = _run(lib, shape, 43, k=kn, v=vn)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    o_ref, l_ref = oracle.attention(q, k, v, shape.scale, True, 189)
    _check(o, lse, o_ref, l_ref, "nan prefix")


def test_latent_rejects_unsupported_widths(lib):
    q = torch.zeros(1, 2, 8, 96, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.AttnError) as e:
        lib.attn_fwd_mla(q, q, v)
    assert e.value.status == lib.ATTN_ERR_UNSUPPORTED


# ------------------------------------------------------------------ decode
from workloads import DecodeShape, decode_inputs, decode_queries  # noqa: E402


def _decode_case(lens, Hq, Hkv, D, Dv, seed, nan_tail=False):
    shape = DecodeShape("ld", B=len(lens), Hq=Hq, Hkv=Hkv, D=D, len_lo=1, len_hi=1, Dv=Dv)
    kv = decode_inputs(shape, seed, seq_lens=lens, extra_pages=3)
    if nan_tail:
        for b, n in enumerate(lens):
            npg = (n + 15) // 16
            if npg and n % 16:
                last = int(kv.block_table[b, npg - 1])
                kv.k_pages[last, n % 16:] = float("nan")
                kv.v_pages[last, n % 16:] = float("nan")
    return shape, kv


@pytest.mark.parametrize("D", [64, 192, 256])
@pytest.mark.parametrize("lens,Hq,Hkv", [
    ([1, 15, 16, 17, 512, 513, 3000, 0], 32, 1),
    ([3, 100, 1000, 2049], 32, 4),
    ([50, 33, 16], 12, 4),               # group of 3
    ([300, 77], 128, 1),                 # four softmax warps
])
def test_decode_widths(lib, D, lens, Hq, Hkv):
    """attn_decode_paged at head widths other than 128."""
    shape, kv = _decode_case(lens, Hq, Hkv, D, D, 60 + D + sum(lens), nan_tail=True)
    d = {n: getattr(kv, n).cuda() for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
    o, lse = lib.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"], shape.scale)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    o_ref, l_ref = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    _check(o, lse, o_ref, l_ref, f"decode D={D} {lens}")


@pytest.mark.parametrize("dqk,dv", [(192, 128), (256, 128), (128, 256), (64, 192), (256, 256), (128, 64)])
@pytest.mark.parametrize("lens,Hq,Hkv,q_len", [
    ([100, 17, 1, 2000, 0], 32, 1, 1),
    ([50, 3, 700, 4096], 32, 8, 4),
    ([513, 64], 12, 4, 7),
])
def test_decode_latent_widths(lib, dqk, dv, lens, Hq, Hkv, q_len):
    """attn_decode_paged_mla: keys of width D_qk, values of width D_v, one or
    several new tokens per sequence, NaN in the unused slots of last pages."""
    shape, kv = _decode_case(lens, Hq, Hkv, dqk, dv, 70 + dqk + dv + q_len, nan_tail=True)
    q = decode_queries(shape, q_len, 71 + q_len)
    d = {n: getattr(kv, n).cuda() for n in ("k_pages", "v_pages", "block_table", "seq_lens")}
    o, lse = lib.attn_decode_paged_mla(q.cuda(), d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                                       shape.scale)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    assert o.shape == (len(lens), Hq, q_len, dv)
    o_ref, l_ref = oracle.paged_decode(q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens, shape.scale)
    _check(o, lse, o_ref, l_ref, f"decode {dqk}/{dv} {lens} q_len={q_len}")


LATENT_DECODE = DecodeShape("latent_mqa_paged_decode_B64_H32_Hkv1_D256_len512_8192", B=64, Hq=32, Hkv=1, D=256,
                            len_lo=512, len_hi=8192)


def test_decode_latent_full_workload(lib):
    """MQA decode in a 256-wide latent space: the batch-64 paged decode
    workload's lengths and layout with D = 256, every row against the
    oracle."""
    kv = decode_inputs(LATENT_DECODE, seed_of(2))
    d = {n: getattr(kv, n).cuda() for n in ("q", "k_pages", "v_pages", "block_table", "seq_lens")}
    o, lse = lib.attn_decode_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["seq_lens"],
                                   LATENT_DECODE.scale)
    torch.cuda.synchronize()
    assert lib.attn_last_device_error() == 0
    o_ref, l_ref = oracle.paged_decode(kv.q, kv.k_pages, kv.v_pages, kv.block_table, kv.seq_lens,
                                       LATENT_DECODE.scale)
    _check(o, lse, o_ref, l_ref, LATENT_DECODE.name)

"""C-ABI checks that need no GPU: the shared library builds and loads, it
exports every entry point include/attn.h declares, and host-side argument
validation answers with the documented status codes before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def cdll():
    from attention_flash_attn_02_b200 import build as b
    path = b.build()
    import attention_flash_attn_02_b200 as attn
    return attn.load(path)


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", src)
    return names


def test_header_declares_the_entry_points():
    names = _declared_symbols()
    for n in ("attn_fwd", "attn_fwd_fp8", "attn_decode_paged", "attn_decode_paged_multi", "attn_decode_workspace_bytes",
              "attn_last_device_error", "attn_status_str", "attn_set_debug", "attn_version"):
        assert n in names


def test_library_exports_every_declared_symbol(cdll):
    for n in _declared_symbols():
        assert hasattr(cdll, n), f"{n} declared in include/ but not exported"


def test_no_internal_symbols_exported(cdll):
    out = os.popen(f"nm -D --defined-only {cdll._name}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert exported, "nm listed no exports"
    extra = {s for s in exported if s.startswith("attn") and s not in set(_declared_symbols())}
    assert not extra, extra


def test_status_strings_and_version(cdll):
    import attention_flash_attn_02_b200 as attn
    assert attn.attn_status_str(0) == "ATTN_OK"
    assert attn.attn_status_str(-1) == "ATTN_ERR_INVALID"
    assert attn.attn_status_str(-4) == "ATTN_ERR_TIMEOUT"
    assert attn.attn_status_str(-5) == "ATTN_ERR_BOUNDS"
    assert attn.attn_status_str(7) == "ATTN_UNKNOWN_STATUS"
    assert attn.attn_version() == 1


def test_workspace_size_formula(cdll):
    import attention_flash_attn_02_b200 as attn
    # a sequence of P pages is cut into at most ceil(P / 32) + 1 segments; each
    # leaves D + 1 floats per query head; plus one int per (sequence, head)
    # rows x segments x (D + 1) floats: each partial and its log-sum-exp
    assert attn.attn_decode_workspace_bytes(64, 32, 512, 128) == 64 * 32 * 17 * 129 * 4
    assert attn.attn_decode_workspace_bytes(2, 4, 33, 128) == 2 * 4 * 3 * 129 * 4
    assert attn.attn_decode_workspace_bytes(0, 4, 33, 128) == 0


_P = ctypes.c_void_p
FAKE = _P(0x10000)  # aligned, never dereferenced: validation fails before any launch


def _fwd(cdll, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Lq=8, Lk=8, D=128,
             scale=0.1, causal=1, window=0)
    a.update(kw)
    return cdll.attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Lq"],
                         a["Lk"], a["D"], a["scale"], a["causal"], a["window"], _P(0))


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), -1),            # heads do not split into groups
    (dict(Hkv=0), -1),
    (dict(Lq=-1), -1),
    (dict(causal=0, window=16), -1),    # a window needs the causal mask
    (dict(causal=2), -1),
    (dict(scale=0.0), -1),
    (dict(scale=float("nan")), -1),
    (dict(q=_P(0x10008)), -1),          # misaligned
    (dict(q=_P(0)), -1),                # null
    (dict(D=96), -2),                   # valid, not built
    (dict(D=256), -2),
    (dict(Lq=0), 0),                    # nothing to do: no launch
    (dict(B=0), 0),
])
def test_fwd_host_validation(cdll, kw, code):
    assert _fwd(cdll, **kw) == code


def test_fwd_fp8_host_validation(cdll):
    f = cdll.attn_fwd_fp8
    args = [FAKE] * 5 + [1, 2, 2, 8, 8, 128, 0.1, 1, 0]
    assert f(*args, 1.0, 1.0, 0.0, _P(0)) == -1          # descale must be > 0
    args64 = [FAKE] * 5 + [1, 2, 2, 8, 8, 64, 0.1, 1, 0]
    assert f(*args64, 1.0, 1.0, 1.0, _P(0)) == -2        # fp8 only for D = 128
    args0 = [FAKE] * 5 + [1, 2, 2, 0, 8, 128, 0.1, 1, 0]
    assert f(*args0, 1.0, 1.0, 1.0, _P(0)) == 0


def _dec(cdll, **kw):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=FAKE, B=2, Hq=32, Hkv=1, D=128,
             page=16, num_pages=10, max_pages=5, scale=0.1, ws=FAKE, ws_bytes=1 << 20)
    a.update(kw)
    return cdll.attn_decode_paged(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["o"], a["lse"], a["B"],
                                  a["Hq"], a["Hkv"], a["D"], a["page"], a["num_pages"], a["max_pages"],
                                  a["scale"], a["ws"], a["ws_bytes"], _P(0))


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=33, Hkv=2), -1),           # heads do not split into groups
    (dict(ws_bytes=16), -1),            # workspace too small
    (dict(ws=_P(0)), -1),
    (dict(sl=_P(0)), -1),
    (dict(bt=_P(0x10002)), -1),         # misaligned int32 table
    (dict(page=32), -2),                # only 16-token pages are built
    (dict(D=96), -2),                   # widths 64, 128, 192, 256 are built
    (dict(Hq=256, Hkv=1), -2),          # group > 128
    (dict(B=0), 0),
])
def test_decode_host_validation(cdll, kw, code):
    assert _dec(cdll, **kw) == code


def _decm(cdll, **kw):
    a = dict(q=FAKE, kp=FAKE, vp=FAKE, bt=FAKE, sl=FAKE, o=FAKE, lse=FAKE, B=2, Hq=32, Hkv=1, q_len=4, D=128,
             page=16, num_pages=10, max_pages=5, scale=0.1, ws=FAKE, ws_bytes=1 << 22)
    a.update(kw)
    return cdll.attn_decode_paged_multi(a["q"], a["kp"], a["vp"], a["bt"], a["sl"], a["o"], a["lse"], a["B"],
                                        a["Hq"], a["Hkv"], a["q_len"], a["D"], a["page"], a["num_pages"],
                                        a["max_pages"], a["scale"], a["ws"], a["ws_bytes"], _P(0))


@pytest.mark.parametrize("kw,code", [
    (dict(q_len=0), -1),
    (dict(q_len=5), -2),                # 32 heads x 5 tokens > 128 rows of one tile
    (dict(Hq=64, Hkv=2, q_len=4, ws_bytes=16), -1),  # supported (32 x 4 rows): only the workspace stops it
    (dict(ws_bytes=2 * 32 * 1 * 129 * 4 * 3), -1),  # room for one token per head only
    (dict(B=0), 0),
])
def test_decode_multi_host_validation(cdll, kw, code):
    assert _decm(cdll, **kw) == code


def test_set_debug_returns_previous_flags(cdll):
    import attention_flash_attn_02_b200 as attn
    attn.attn_set_debug(1, 0)
    assert attn.attn_set_debug(0, 0) == 1
    assert attn.attn_set_debug(0, 0) == 0


def test_missing_library_fails_loudly(tmp_path):
    import attention_flash_attn_02_b200 as attn
    saved = attn._lib
    attn._lib = None
    try:
        with pytest.raises(FileNotFoundError):
            attn.load(str(tmp_path / "nope.so"))
    finally:
        attn._lib = saved


def _ptxas_log(kernel, regs=128, spill_st=0, spill_ld=0):
    return (f"ptxas info    : Compiling entry function '_ZN4attn{kernel}Ev' for 'sm_100a'\n"
            f"ptxas info    : Function properties for _ZN4attn{kernel}Ev\n"
            f"    0 bytes stack frame, {spill_st} bytes spill stores, {spill_ld} bytes spill loads\n"
            f"ptxas info    : Used {regs} registers, used 2 barriers\n")


def test_build_check_accepts_clean_prefill_log():
    from attention_flash_attn_02_b200.build import check_register_counts
    check_register_counts(_ptxas_log("14prefill_kernel") + _ptxas_log("19decode_split_kernel", regs=148))


def test_build_check_rejects_wrong_launch_count_and_spills():
    from attention_flash_attn_02_b200.build import check_register_counts
    with pytest.raises(RuntimeError, match="registers"):
        check_register_counts(_ptxas_log("14prefill_kernel", regs=168))
    with pytest.raises(RuntimeError, match="spills"):
        check_register_counts(_ptxas_log("14prefill_kernel", spill_st=44, spill_ld=40))
    with pytest.raises(RuntimeError, match="spills"):
        check_register_counts(_ptxas_log("14prefill_kernel") + _ptxas_log("10bwd_kernel", spill_st=8))
    with pytest.raises(RuntimeError, match="no prefill"):
        check_register_counts(_ptxas_log("19decode_split_kernel"))

"""Python binding of libattn_sm100.so (B200 fused attention).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/attn.h``.  PyTorch supplies device
memory and the current stream.  If the shared library is missing, every call
raises -- there is no fallback.

Functions mirror the C entry points:

* ``attn_fwd(q, k, v, scale=None, causal=False, window=0, o=None, lse=None)``
* ``attn_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, ...)``
* ``attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, ...)``
* ``attn_decode_workspace_bytes(B, Hq, max_pages_per_seq, D)``
* ``attn_last_device_error()``, ``attn_status_str(code)``,
  ``attn_set_debug(flags, wait_timeout_ns)``, ``attn_version()``
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libattn_sm100.so")

ATTN_OK = 0
ATTN_ERR_INVALID = -1
ATTN_ERR_UNSUPPORTED = -2
ATTN_ERR_CUDA = -3
ATTN_ERR_TIMEOUT = -4
ATTN_ERR_BOUNDS = -5
ATTN_DEBUG_BOUNDS = 1
ATTN_DEBUG_STALL = 2

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        detail = ""
        if status == ATTN_ERR_CUDA:
            detail = " -- " + attn_last_error_message()
        super().__init__(f"{what} failed: {attn_status_str(status)} ({status}){detail}")


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads the shared library (once).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise FileNotFoundError(
            f"{path} not found: build it with `python -m attention_flash_attn_02_b200.build`")
    lib = ctypes.CDLL(path)
    c_int, c_float, c_void_p, c_size_t = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
    lib.attn_fwd.argtypes = [c_void_p] * 5 + [c_int] * 6 + [c_float, c_int, c_int, c_void_p]
    lib.attn_fwd.restype = c_int
    lib.attn_fwd_fp8.argtypes = [c_void_p] * 5 + [c_int] * 6 + [c_float, c_int, c_int] + [c_float] * 3 + [c_void_p]
    lib.attn_fwd_fp8.restype = c_int
    lib.attn_fwd_e5m2.argtypes = lib.attn_fwd_fp8.argtypes
    lib.attn_fwd_e5m2.restype = c_int
    lib.attn_fwd_mla.argtypes = [c_void_p] * 5 + [c_int] * 7 + [c_float, c_int, c_int, c_void_p]
    lib.attn_fwd_mla.restype = c_int
    lib.attn_decode_workspace_bytes.argtypes = [c_int] * 4
    lib.attn_decode_workspace_bytes.restype = c_size_t
    lib.attn_decode_paged.argtypes = [c_void_p] * 7 + [c_int] * 7 + [c_float, c_void_p, c_size_t, c_void_p]
    lib.attn_decode_paged.restype = c_int
    lib.attn_decode_paged_multi.argtypes = [c_void_p] * 7 + [c_int] * 8 + [c_float, c_void_p, c_size_t, c_void_p]
    lib.attn_decode_paged_multi.restype = c_int
    lib.attn_decode_paged_mla.argtypes = [c_void_p] * 7 + [c_int] * 9 + [c_float, c_void_p, c_size_t, c_void_p]
    lib.attn_decode_paged_mla.restype = c_int
    lib.attn_prefill_paged.argtypes = [c_void_p] * 7 + [c_int] * 8 + [c_float, c_int, c_void_p]
    lib.attn_prefill_paged.restype = c_int
    lib.attn_kv_append.argtypes = [c_void_p] * 6 + [c_int] * 7 + [c_void_p]
    lib.attn_kv_append.restype = c_int
    lib.attn_bwd_workspace_bytes.argtypes = [c_int] * 4
    lib.attn_bwd_workspace_bytes.restype = c_size_t
    lib.attn_bwd.argtypes = [c_void_p] * 9 + [c_int] * 6 + [c_float, c_int, c_int, c_void_p, c_size_t, c_void_p]
    lib.attn_bwd.restype = c_int
    lib.attn_decode_paged_noalloc.argtypes = [c_void_p] * 7 + [c_int] * 7 + [c_float, c_void_p]
    lib.attn_decode_paged_noalloc.restype = c_int
    lib.attn_last_device_error.argtypes = [c_void_p]
    lib.attn_last_device_error.restype = c_int
    lib.attn_status_str.argtypes = [c_int]
    lib.attn_status_str.restype = ctypes.c_char_p
    lib.attn_set_debug.argtypes = [c_int, ctypes.c_ulonglong]
    lib.attn_set_debug.restype = c_int
    lib.attn_last_error_message.argtypes = []
    lib.attn_last_error_message.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    lib.attn_version.restype = c_int
    _lib = lib
    return lib


def attn_status_str(status: int) -> str:
    return load().attn_status_str(int(status)).decode()


def _check(status: int, what: str):
    if status != ATTN_OK:
        raise AttnError(status, what)


def _stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() > 0 else ctypes.c_void_p(0)


def attn_fwd(q, k, v, scale: Optional[float] = None, causal: bool = False, window: int = 0,
             o=None, lse=None, stream=None):
    """bf16 attention forward.  q [B,Hq,Lq,D], k/v [B,Hkv,Lk,D], contiguous,
    on the GPU.  Returns (o bf16 [B,Hq,Lq,D], lse fp32 [B,Hq,Lq])."""
    import torch
    lib = load()
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty((B, Hq, Lq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    for t in (q, k, v, o, lse):
        if not t.is_contiguous():
            raise ValueError("attn_fwd: tensors must be contiguous")
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("attn_fwd: q, k, v must be bfloat16")
    st = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq, Lk, D,
                      float(scale), int(bool(causal)), int(window), _stream_handle(stream))
    _check(st, "attn_fwd")
    return o, lse


def attn_fwd_mla(q, k, v, scale: Optional[float] = None, causal: bool = False, window: int = 0,
                 o=None, lse=None, stream=None):
    """bf16 attention with query/key width D_qk and value width D_v (each 64,
    128, 192 or 256): q [B, Hq, Lq, D_qk], k [B, Hkv, Lk, D_qk], v [B, Hkv, Lk,
    D_v]; returns (o [B, Hq, Lq, D_v] bf16, lse [B, Hq, Lq] fp32).  The default
    scale is 1/sqrt(D_qk)."""
    import torch
    lib = load()
    B, Hq, Lq, Dqk = q.shape
    Hkv, Lk, Dv = k.shape[1], k.shape[2], v.shape[3]
    if k.shape[3] != Dqk or v.shape[:3] != k.shape[:3]:
        raise ValueError("attn_fwd_mla: k must be [B, Hkv, Lk, D_qk] and v [B, Hkv, Lk, D_v]")
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    if o is None:
        o = torch.empty((B, Hq, Lq, Dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise TypeError("attn_fwd_mla: q, k, v must be contiguous bfloat16")
    st = lib.attn_fwd_mla(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq, Lk, Dqk, Dv,
                          float(scale), int(bool(causal)), int(window), _stream_handle(stream))
    _check(st, "attn_fwd_mla")
    return o, lse


def attn_fwd_fp8(q, k, v, q_descale: float, k_descale: float, v_descale: float,
                 scale: Optional[float] = None, causal: bool = False, window: int = 0,
                 o=None, lse=None, stream=None):
    """e4m3 attention forward (bf16 output); tensors torch.float8_e4m3fn."""
    return _fwd_8bit("attn_fwd_fp8", "float8_e4m3fn", q, k, v, q_descale, k_descale, v_descale, scale, causal,
                     window, o, lse, stream)


def attn_fwd_e5m2(q, k, v, q_descale: float, k_descale: float, v_descale: float,
                  scale: Optional[float] = None, causal: bool = False, window: int = 0,
                  o=None, lse=None, stream=None):
    """e5m2 attention forward (bf16 output); tensors torch.float8_e5m2."""
    return _fwd_8bit("attn_fwd_e5m2", "float8_e5m2", q, k, v, q_descale, k_descale, v_descale, scale, causal,
                     window, o, lse, stream)


def _fwd_8bit(name, dtype_name, q, k, v, q_descale, k_descale, v_descale, scale, causal, window, o, lse,
              stream):
    import torch
    lib = load()
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty((B, Hq, Lq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    for t in (q, k, v):
        if t.dtype != getattr(torch, dtype_name) or not t.is_contiguous():
            raise TypeError(f"{name}: q, k, v must be contiguous {dtype_name}")
    st = getattr(lib, name)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Lq, Lk, D,
                            float(scale), int(bool(causal)), int(window), float(q_descale),
                            float(k_descale), float(v_descale), _stream_handle(stream))
    _check(st, name)
    return o, lse


def attn_decode_workspace_bytes(B: int, Hq: int, max_pages_per_seq: int, D: int) -> int:
    return int(load().attn_decode_workspace_bytes(B, Hq, max_pages_per_seq, D))


def attn_bwd_workspace_bytes(B: int, Hq: int, Lq: int, D: int) -> int:
    return int(load().attn_bwd_workspace_bytes(B, Hq, Lq, D))


def attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, scale: Optional[float] = None,
                      o=None, lse=None, workspace=None, stream=None):
    """Single-token paged decode.  q [B,Hq,D] bf16; pools [P,16,Hkv,D] bf16;
    block_table [B,max_pages] int32; seq_lens [B] int32; all on the GPU.
    Returns (o bf16 [B,Hq,D], lse fp32 [B,Hq])."""
    import torch
    lib = load()
    B, Hq, D = q.shape
    num_pages, page_size, Hkv, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    need = lib.attn_decode_workspace_bytes(B, Hq, max(max_pages, 1), D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("attn_decode_paged: block_table and seq_lens must be int32")
    st = lib.attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens),
                               _ptr(o), _ptr(lse), B, Hq, Hkv, D, page_size, num_pages, max_pages,
                               float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream_handle(stream))
    _check(st, "attn_decode_paged")
    return o, lse


def attn_decode_paged_multi(q, k_pages, v_pages, block_table, seq_lens, scale: Optional[float] = None,
                            o=None, lse=None, workspace=None, stream=None):
    """Paged decode of the last q_len cached tokens of each sequence (query
    token i sees the cache up to its own position).  q [B,Hq,q_len,D] bf16;
    pools, block_table and seq_lens as attn_decode_paged.  Returns
    (o bf16 [B,Hq,q_len,D], lse fp32 [B,Hq,q_len])."""
    import torch
    lib = load()
    B, Hq, q_len, D = q.shape
    num_pages, page_size, Hkv, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty((B, Hq, q_len, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, q_len), dtype=torch.float32, device=q.device)
    need = lib.attn_decode_workspace_bytes(B, Hq * q_len, max(max_pages, 1), D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("attn_decode_paged_multi: block_table and seq_lens must be int32")
    st = lib.attn_decode_paged_multi(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens),
                                     _ptr(o), _ptr(lse), B, Hq, Hkv, q_len, D, page_size, num_pages, max_pages,
                                     float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream_handle(stream))
    _check(st, "attn_decode_paged_multi")
    return o, lse


def attn_decode_paged_mla(q, k_pages, v_pages, block_table, seq_lens, scale: Optional[float] = None,
                          o=None, lse=None, workspace=None, stream=None):
    """Paged decode with query/key width D_qk and value width D_v (each 64,
    128, 192 or 256).  q [B,Hq,q_len,D_qk] bf16 (the last q_len cached tokens);
    k_pages [P,16,Hkv,D_qk], v_pages [P,16,Hkv,D_v] bf16; block_table
    [B,max_pages] int32; seq_lens [B] int32.  The default scale is
    1/sqrt(D_qk).  Returns (o bf16 [B,Hq,q_len,D_v], lse fp32 [B,Hq,q_len])."""
    import torch
    lib = load()
    B, Hq, q_len, Dqk = q.shape
    num_pages, page_size, Hkv, _ = k_pages.shape
    Dv = v_pages.shape[3]
    max_pages = block_table.shape[1]
    if k_pages.shape[3] != Dqk or v_pages.shape[:3] != k_pages.shape[:3]:
        raise ValueError("attn_decode_paged_mla: k_pages must be [P,16,Hkv,D_qk] and v_pages [P,16,Hkv,D_v]")
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    if o is None:
        o = torch.empty((B, Hq, q_len, Dv), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, q_len), dtype=torch.float32, device=q.device)
    need = lib.attn_decode_workspace_bytes(B, Hq * q_len, max(max_pages, 1), Dv)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("attn_decode_paged_mla: block_table and seq_lens must be int32")
    st = lib.attn_decode_paged_mla(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens),
                                   _ptr(o), _ptr(lse), B, Hq, Hkv, q_len, Dqk, Dv, page_size, num_pages, max_pages,
                                   float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream_handle(stream))
    _check(st, "attn_decode_paged_mla")
    return o, lse


def attn_prefill_paged(q, k_pages, v_pages, block_table, seq_lens, scale: Optional[float] = None, window: int = 0,
                       o=None, lse=None, stream=None):
    """Chunked prefill over a paged cache: the last Lq cached tokens of each
    sequence attend causally to the cache.  q [B,Hq,Lq,D] bf16; pools
    [P,16,Hkv,D] bf16; block_table [B,max_pages] int32; seq_lens [B] int32.
    Returns (o bf16 [B,Hq,Lq,D], lse fp32 [B,Hq,Lq])."""
    import torch
    lib = load()
    B, Hq, Lq, D = q.shape
    num_pages, page_size, Hkv, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty((B, Hq, Lq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("attn_prefill_paged: block_table and seq_lens must be int32")
    st = lib.attn_prefill_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens), _ptr(o),
                                _ptr(lse), B, Hq, Hkv, Lq, D, page_size, num_pages, max_pages, float(scale),
                                int(window), _stream_handle(stream))
    _check(st, "attn_prefill_paged")
    return o, lse


def attn_kv_append(k_new, v_new, k_pages, v_pages, block_table, seq_lens, stream=None):
    """Write k_new/v_new [B,Hkv,L_new,D] bf16 into the pools at positions
    seq_lens[b] - L_new + t (in place)."""
    import torch
    lib = load()
    B, Hkv, L_new, D = k_new.shape
    num_pages, page_size, _, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("attn_kv_append: block_table and seq_lens must be int32")
    st = lib.attn_kv_append(_ptr(k_new), _ptr(v_new), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                            _ptr(seq_lens), B, Hkv, L_new, D, page_size, num_pages, max_pages,
                            _stream_handle(stream))
    _check(st, "attn_kv_append")
    return k_pages, v_pages


def attn_bwd(q, k, v, o, dout, lse, scale: Optional[float] = None, causal: bool = False, window: int = 0,
             dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of attn_fwd: q [B,Hq,Lq,D], k/v [B,Hkv,Lk,D], o and dout
    [B,Hq,Lq,D] bf16, lse [B,Hq,Lq] fp32 (attn_fwd's).  Returns (dq, dk, dv)
    bf16."""
    import torch
    lib = load()
    B, Hq, Lq, D = q.shape
    _, Hkv, Lk, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = attn_bwd_workspace_bytes(B, Hq, Lq, D)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                      B, Hq, Hkv, Lq, Lk, D, float(scale), int(bool(causal)), int(window), _ptr(workspace),
                      workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check(st, "attn_bwd")
    return dq, dk, dv


def attn_decode_paged_noalloc(q, k_pages, v_pages, block_table, seq_lens, scale: Optional[float] = None,
                              o=None, lse=None, stream=None):
    """attn_decode_paged without a workspace argument, for callers that cannot
    allocate device memory when they run decode: the scratch is a fixed array
    inside the library (ATTN_DECODE_NOALLOC_SCRATCH_BYTES).  Calls that overlap
    on the GPU share that array and must not run concurrently.  Returns
    (o bf16 [B,Hq,D], lse fp32 [B,Hq]); outputs may be passed in to avoid any
    allocation in this wrapper too."""
    import torch
    lib = load()
    B, Hq, D = q.shape
    num_pages, page_size, Hkv, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("attn_decode_paged_noalloc: block_table and seq_lens must be int32")
    st = lib.attn_decode_paged_noalloc(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(seq_lens),
                                       _ptr(o), _ptr(lse), B, Hq, Hkv, D, page_size, num_pages, max_pages,
                                       float(scale), _stream_handle(stream))
    _check(st, "attn_decode_paged_noalloc")
    return o, lse


def attn_last_device_error(stream=None) -> int:
    return int(load().attn_last_device_error(_stream_handle(stream)))


def attn_set_debug(flags: int, wait_timeout_ns: int = 0) -> int:
    return int(load().attn_set_debug(int(flags), int(wait_timeout_ns)))


def attn_last_error_message() -> str:
    return load().attn_last_error_message().decode()


def attn_version() -> int:
    return int(load().attn_version())

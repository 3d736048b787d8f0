"""Paged KV-cache attention for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libpkv.so``, whose C ABI is declared in
``include/pkv.h``.  Each function here has the name of the C entry point it
calls and only marshals arguments: it checks dtypes and devices, passes raw
device pointers, the current CUDA stream and the pool geometry, and turns a
non-zero status into ``PkvError``.  All computation runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback, and importing this module
fails if the library has not been built
(``python paged_kv_attention_37_b200/build.py``).

Tensors (all CUDA, contiguous):
  k_pool, v_pool  bf16 [num_pages, Hkv, page_size, d]
  page_table      int32 [B, max_pages]
  kv_lens         int32 [B]      keys per request, including this step's token
  q (decode)      bf16 [B, Hq, d]
  q (prefill)     bf16 [total_q, Hq, d] with cu_q_lens int32 [B+1]
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "PkvError", "LIB_PATH", "pool_desc", "pkv_kv_append", "pkv_decode_workspace_bytes",
    "pkv_paged_attn_decode", "pkv_split_k_combine", "pkv_paged_attn_chunked_prefill",
    "pkv_status_string", "pkv_device_error_flags", "decode_workspace",
    "pkv_paged_attn_decode_static", "pkv_qk_norm_rope_append", "pkv_kv_append_cow",
    "pkv_verify_workspace_bytes", "verify_workspace", "pkv_paged_attn_verify", "pkv_paged_attn_decode_flags",
    "DECODE_METADATA_READY", "pkv_mixed_workspace_bytes", "mixed_workspace", "pkv_paged_attn_mixed",
    "pkv_paged_attn_decode_append",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpkv.so")

FLAG_WAIT_TIMEOUT = 0x1
FLAG_BAD_LENGTH = 0x2
FLAG_BAD_SLOT = 0x4
FLAG_BAD_QUERY_ROWS = 0x8
FLAG_BAD_PAGE = 0x10
FLAG_INTERNAL = 0x20
FLAG_NO_FREE_PAGE = 0x40

DECODE_METADATA_READY = 0x1  # pkv_paged_attn_decode_flags option bit


class PkvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {pkv_status_string(status)} (status {status})")
        self.status = status


class _PoolDesc(ctypes.Structure):
    _fields_ = [("num_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python paged_kv_attention_37_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    lib.pkv_kv_append.argtypes = [P, P, P, I32, P, P, _PoolDesc, P]
    lib.pkv_kv_append.restype = ctypes.c_int
    lib.pkv_decode_workspace_bytes.argtypes = [I32, I32, I32, I32, I32]
    lib.pkv_decode_workspace_bytes.restype = SZ
    lib.pkv_paged_attn_decode.argtypes = [P, I32, I32, P, P, _PoolDesc, P, I32, P, F32, I32, P, SZ,
                                          P, P, P]
    lib.pkv_paged_attn_decode.restype = ctypes.c_int
    lib.pkv_split_k_combine.argtypes = [P, P, P, I32, I32, I32, I32, P, P, P]
    lib.pkv_split_k_combine.restype = ctypes.c_int
    lib.pkv_paged_attn_chunked_prefill.argtypes = [P, P, I32, I32, I32, I32, P, P, P, _PoolDesc, P,
                                                   I32, F32, P, P]
    lib.pkv_paged_attn_chunked_prefill.restype = ctypes.c_int
    lib.pkv_status_string.argtypes = [ctypes.c_int]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_device_error_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
    lib.pkv_device_error_flags.restype = ctypes.c_int
    lib.pkv_qk_norm_rope_append.argtypes = [P, P, P, I32, I32, P, P, P, P, F32, F32, P, P, P, _PoolDesc, P]
    lib.pkv_qk_norm_rope_append.restype = ctypes.c_int
    lib.pkv_kv_append_cow.argtypes = [P, P, P, P, I32, P, I32, I32, P, P, I32, P, P, P, _PoolDesc, P]
    lib.pkv_kv_append_cow.restype = ctypes.c_int
    lib.pkv_paged_attn_decode_flags.argtypes = [P, I32, I32, P, P, _PoolDesc, P, I32, P, F32, I32, P, SZ,
                                                P, P, ctypes.c_uint32, P]
    lib.pkv_paged_attn_decode_flags.restype = ctypes.c_int
    lib.pkv_paged_attn_decode_append.argtypes = [P, P, P, I32, I32, P, P, _PoolDesc, P, I32, P, F32, I32, P, SZ,
                                                 P, P, ctypes.c_uint32, P]
    lib.pkv_paged_attn_decode_append.restype = ctypes.c_int
    lib.pkv_mixed_workspace_bytes.argtypes = [I32, I32, I32, I32]
    lib.pkv_mixed_workspace_bytes.restype = SZ
    lib.pkv_paged_attn_mixed.argtypes = [P, P, I32, I32, I32, P, P, I32, P, I32, P, I32, P, I32, P, P, _PoolDesc,
                                         F32, P, SZ, P, P, P, P]
    lib.pkv_paged_attn_mixed.restype = ctypes.c_int
    lib.pkv_verify_workspace_bytes.argtypes = [I32, I32, I32, I32, I32]
    lib.pkv_verify_workspace_bytes.restype = SZ
    lib.pkv_paged_attn_verify.argtypes = [P, P, I32, I32, I32, I32, P, P, P, _PoolDesc, P, I32, F32, I32, P,
                                          SZ, P, P]
    lib.pkv_paged_attn_verify.restype = ctypes.c_int
    return lib


_lib = _load()


# ------------------------------------------------------------- marshalling
def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype, ndim: int | None = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")


def _check(fn: str, status: int):
    if status != 0:
        raise PkvError(fn, status)


def pool_desc(k_pool: torch.Tensor) -> _PoolDesc:
    n, hkv, p, d = k_pool.shape
    return _PoolDesc(n, p, hkv, d)


# -------------------------------------------------------------- entry points
def pkv_status_string(status: int) -> str:
    return _lib.pkv_status_string(int(status)).decode()


def pkv_device_error_flags(clear: bool = True) -> int:
    """Synchronise the device and return (and by default clear) the error word."""
    v = ctypes.c_uint32(0)
    _check("pkv_device_error_flags", _lib.pkv_device_error_flags(ctypes.byref(v), int(clear)))
    return int(v.value)


def pkv_kv_append(k_new, v_new, slot_mapping, k_pool, v_pool, stream=None):
    """Bit-copy rows k_new/v_new [T, Hkv, d] into pool slots (slot = page*P + offset)."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, n, torch.bfloat16, 3)
    _need(slot_mapping, "slot_mapping", torch.int32, 1)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    T = k_new.shape[0]
    if slot_mapping.shape[0] != T or v_new.shape != k_new.shape:
        raise ValueError("k_new, v_new and slot_mapping disagree on the token count")
    if k_new.shape[1:] != (k_pool.shape[1], k_pool.shape[3]) or v_pool.shape != k_pool.shape:
        raise ValueError("row shape does not match the pool")
    _check("pkv_kv_append", _lib.pkv_kv_append(
        _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), T, _ptr(k_pool), _ptr(v_pool),
        pool_desc(k_pool), _stream(stream)))


def pkv_decode_workspace_bytes(batch, num_q_heads, head_dim, max_kv_len, partition_tokens=0) -> int:
    return int(_lib.pkv_decode_workspace_bytes(batch, num_q_heads, head_dim, max_kv_len,
                                               partition_tokens))


def decode_workspace(batch, num_q_heads, head_dim, max_kv_len, partition_tokens=0, device=None):
    """A zero-filled workspace of the size pkv_paged_attn_decode needs."""
    n = pkv_decode_workspace_bytes(batch, num_q_heads, head_dim, max_kv_len, partition_tokens)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def pkv_paged_attn_decode(q, k_pool, v_pool, page_table, kv_lens, scale, partition_tokens=0,
                          workspace=None, out=None, out_lse=None, stream=None):
    """Decode attention (q_len = 1) of q [B, Hq, d] over each request's pages.

    Returns ``out`` (bf16 [B, Hq, d]); fills ``out_lse`` (fp32 [B, Hq]) if given.
    ``workspace`` (uint8, zero-filled before first use) defaults to a new one.
    """
    return pkv_paged_attn_decode_flags(q, k_pool, v_pool, page_table, kv_lens, scale, partition_tokens,
                                       workspace, out, out_lse, 0, stream)


def pkv_paged_attn_decode_flags(q, k_pool, v_pool, page_table, kv_lens, scale, partition_tokens=0,
                                workspace=None, out=None, out_lse=None, flags=0, stream=None):
    """pkv_paged_attn_decode with option bits (DECODE_METADATA_READY: the
    kernel just ahead on the stream writes neither kv_lens nor page_table)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    _need(kv_lens, "kv_lens", torch.int32, 1)
    B, hq, d = q.shape
    max_pages = page_table.shape[1]
    if page_table.shape[0] != B or kv_lens.shape[0] != B:
        raise ValueError("page_table / kv_lens rows must equal the batch")
    if workspace is None:
        workspace = decode_workspace(B, hq, d, max_pages * k_pool.shape[2], partition_tokens,
                                     q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3)
    if out_lse is not None:
        _need(out_lse, "out_lse", torch.float32, 2)
    _check("pkv_paged_attn_decode_flags", _lib.pkv_paged_attn_decode_flags(
        _ptr(q), B, hq, _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(page_table),
        max_pages, _ptr(kv_lens), float(scale), int(partition_tokens), _ptr(workspace),
        workspace.numel(), _ptr(out), _ptr(out_lse), int(flags), _stream(stream)))
    return out


def pkv_paged_attn_decode_append(q, k_new, v_new, k_pool, v_pool, page_table, kv_lens, scale, partition_tokens=0,
                                 workspace=None, out=None, out_lse=None, flags=0, stream=None):
    """One decode step in one launch: request r's new row (k_new[r], v_new[r],
    [B, Hkv, d]) is written to its pool slot at position kv_lens[r] - 1 and
    attended to as that key; otherwise as pkv_paged_attn_decode_flags."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    _need(kv_lens, "kv_lens", torch.int32, 1)
    B, hq, d = q.shape
    max_pages = page_table.shape[1]
    if page_table.shape[0] != B or kv_lens.shape[0] != B:
        raise ValueError("page_table / kv_lens rows must equal the batch")
    if tuple(k_new.shape) != (B, k_pool.shape[1], d) or k_new.shape != v_new.shape:
        raise ValueError("k_new / v_new must be [batch, Hkv, d]")
    if workspace is None:
        workspace = decode_workspace(B, hq, d, max_pages * k_pool.shape[2], partition_tokens, q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3)
    if out_lse is not None:
        _need(out_lse, "out_lse", torch.float32, 2)
    _check("pkv_paged_attn_decode_append", _lib.pkv_paged_attn_decode_append(
        _ptr(q), _ptr(k_new), _ptr(v_new), B, hq, _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool),
        _ptr(page_table), max_pages, _ptr(kv_lens), float(scale), int(partition_tokens), _ptr(workspace),
        workspace.numel(), _ptr(out), _ptr(out_lse), int(flags), _stream(stream)))
    return out


def pkv_split_k_combine(part_o, part_lse, num_splits, out=None, out_lse=None, stream=None):
    """Merge fp32 partials part_o [B, Hq, S, d] / part_lse [B, Hq, S] -> bf16 [B, Hq, d]."""
    _need(part_o, "part_o", torch.float32, 4)
    _need(part_lse, "part_lse", torch.float32, 3)
    _need(num_splits, "num_splits", torch.int32, 1)
    B, hq, S, d = part_o.shape
    if out is None:
        out = torch.empty((B, hq, d), dtype=torch.bfloat16, device=part_o.device)
    _need(out, "out", torch.bfloat16, 3)
    if out_lse is not None:
        _need(out_lse, "out_lse", torch.float32, 2)
    _check("pkv_split_k_combine", _lib.pkv_split_k_combine(
        _ptr(part_o), _ptr(part_lse), _ptr(num_splits), B, hq, d, S, _ptr(out), _ptr(out_lse),
        _stream(stream)))
    return out


def pkv_paged_attn_chunked_prefill(q, cu_q_lens, ctx_offsets, k_pool, v_pool, page_table, scale,
                                   max_q_len, out=None, stream=None):
    """Causal attention of prompt chunks q [total_q, Hq, d] at context offsets."""
    _need(q, "q", torch.bfloat16, 3)
    _need(cu_q_lens, "cu_q_lens", torch.int32, 1)
    _need(ctx_offsets, "ctx_offsets", torch.int32, 1)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    total_q, hq, d = q.shape
    B = ctx_offsets.shape[0]
    if cu_q_lens.shape[0] != B + 1 or page_table.shape[0] != B:
        raise ValueError("cu_q_lens must have B+1 entries and page_table B rows")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3)
    _check("pkv_paged_attn_chunked_prefill", _lib.pkv_paged_attn_chunked_prefill(
        _ptr(q), _ptr(cu_q_lens), B, hq, total_q, int(max_q_len), _ptr(ctx_offsets),
        _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(page_table), page_table.shape[1],
        float(scale), _ptr(out), _stream(stream)))
    return out


def pkv_mixed_workspace_bytes(batch_dec, num_q_heads, head_dim, max_kv_len) -> int:
    return int(_lib.pkv_mixed_workspace_bytes(batch_dec, num_q_heads, head_dim, max_kv_len))


def mixed_workspace(batch_dec, num_q_heads, head_dim, max_kv_len, device=None):
    """A zero-filled workspace of the size pkv_paged_attn_mixed needs."""
    n = pkv_mixed_workspace_bytes(batch_dec, num_q_heads, head_dim, max_kv_len)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def pkv_paged_attn_mixed(q_pre, cu_q_lens, ctx_offsets, page_table_pre, max_q_len, q_dec, page_table_dec,
                         kv_lens, k_pool, v_pool, scale, workspace=None, out_pre=None, out_dec=None,
                         out_lse_dec=None, stream=None):
    """Prefill chunks (q_pre [total_q, Hq, d], cu_q_lens, ctx_offsets) and decode
    requests (q_dec [B, Hq, d], kv_lens) of one batch in a single persistent
    launch; returns (out_pre, out_dec)."""
    _need(q_pre, "q_pre", torch.bfloat16, 3)
    _need(cu_q_lens, "cu_q_lens", torch.int32, 1)
    _need(ctx_offsets, "ctx_offsets", torch.int32, 1)
    _need(page_table_pre, "page_table_pre", torch.int32, 2)
    _need(q_dec, "q_dec", torch.bfloat16, 3)
    _need(page_table_dec, "page_table_dec", torch.int32, 2)
    _need(kv_lens, "kv_lens", torch.int32, 1)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    total_q, hq, d = q_pre.shape
    bp, bd = ctx_offsets.shape[0], q_dec.shape[0]
    if cu_q_lens.shape[0] != bp + 1 or page_table_pre.shape[0] != bp:
        raise ValueError("cu_q_lens must have B+1 entries and page_table_pre B rows")
    if page_table_dec.shape[0] != bd or kv_lens.shape[0] != bd or q_dec.shape[1:] != q_pre.shape[1:]:
        raise ValueError("decode tensors disagree on the batch or the head shape")
    if workspace is None:
        workspace = mixed_workspace(bd, hq, d, page_table_dec.shape[1] * k_pool.shape[2], q_pre.device)
    _need(workspace, "workspace", torch.uint8, 1)
    out_pre = torch.empty_like(q_pre) if out_pre is None else out_pre
    out_dec = torch.empty_like(q_dec) if out_dec is None else out_dec
    _need(out_pre, "out_pre", torch.bfloat16, 3)
    _need(out_dec, "out_dec", torch.bfloat16, 3)
    if out_lse_dec is not None:
        _need(out_lse_dec, "out_lse_dec", torch.float32, 2)
    _check("pkv_paged_attn_mixed", _lib.pkv_paged_attn_mixed(
        _ptr(q_pre), _ptr(cu_q_lens), bp, total_q, int(max_q_len), _ptr(ctx_offsets), _ptr(page_table_pre),
        page_table_pre.shape[1], _ptr(q_dec), bd, _ptr(page_table_dec), page_table_dec.shape[1],
        _ptr(kv_lens), hq, _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), float(scale), _ptr(workspace),
        workspace.numel(), _ptr(out_pre), _ptr(out_dec), _ptr(out_lse_dec), _stream(stream)))
    return out_pre, out_dec


def pkv_verify_workspace_bytes(total_q, num_q_heads, head_dim, max_kv_len, partition_tokens=0) -> int:
    return int(_lib.pkv_verify_workspace_bytes(total_q, num_q_heads, head_dim, max_kv_len, partition_tokens))


def verify_workspace(total_q, num_q_heads, head_dim, max_kv_len, partition_tokens=0, device=None):
    """A workspace of the size pkv_paged_attn_verify needs (no zeroing needed)."""
    n = pkv_verify_workspace_bytes(total_q, num_q_heads, head_dim, max_kv_len, partition_tokens)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def pkv_paged_attn_verify(q, cu_q_lens, ctx_offsets, k_pool, v_pool, page_table, scale, max_q_len,
                          partition_tokens=0, workspace=None, out=None, stream=None):
    """Causal attention of short chunks q [total_q, Hq, d] at context offsets,
    split along the keys (speculative verify); same rows as chunked prefill."""
    _need(q, "q", torch.bfloat16, 3)
    _need(cu_q_lens, "cu_q_lens", torch.int32, 1)
    _need(ctx_offsets, "ctx_offsets", torch.int32, 1)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    total_q, hq, d = q.shape
    B = ctx_offsets.shape[0]
    if cu_q_lens.shape[0] != B + 1 or page_table.shape[0] != B:
        raise ValueError("cu_q_lens must have B+1 entries and page_table B rows")
    if workspace is None:
        workspace = verify_workspace(total_q, hq, d, page_table.shape[1] * k_pool.shape[2],
                                     partition_tokens, q.device)
    _need(workspace, "workspace", torch.uint8, 1)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3)
    _check("pkv_paged_attn_verify", _lib.pkv_paged_attn_verify(
        _ptr(q), _ptr(cu_q_lens), B, hq, total_q, int(max_q_len), _ptr(ctx_offsets), _ptr(k_pool),
        _ptr(v_pool), pool_desc(k_pool), _ptr(page_table), page_table.shape[1], float(scale),
        int(partition_tokens), _ptr(workspace), workspace.numel(), _ptr(out), _stream(stream)))
    return out


def pkv_qk_norm_rope_append(q, k, v, q_norm_weight, k_norm_weight, positions, slot_mapping, k_pool,
                            v_pool, eps=1e-6, rope_theta=1e6, q_out=None, stream=None):
    """RMSNorm + RoPE of this step's q [T, Hq, d] and k [T, Hkv, d] rows, and
    the write of k (rotated) and v into the pool slots; returns q_out."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 3)
    for t, n in ((q_norm_weight, "q_norm_weight"), (k_norm_weight, "k_norm_weight")):
        _need(t, n, torch.bfloat16, 1)
    _need(positions, "positions", torch.int32, 1)
    _need(slot_mapping, "slot_mapping", torch.int32, 1)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    T, hq, d = q.shape
    if k.shape != v.shape or k.shape[0] != T or positions.shape[0] != T or slot_mapping.shape[0] != T:
        raise ValueError("q, k, v, positions and slot_mapping disagree on the token count")
    if k.shape[1:] != (k_pool.shape[1], k_pool.shape[3]) or v_pool.shape != k_pool.shape:
        raise ValueError("row shape does not match the pool")
    if q_norm_weight.shape[0] != d or k_norm_weight.shape[0] != d or q.shape[2] != d:
        raise ValueError("norm weights must have head_dim elements")
    if q_out is None:
        q_out = torch.empty_like(q)
    _need(q_out, "q_out", torch.bfloat16, 3)
    _check("pkv_qk_norm_rope_append", _lib.pkv_qk_norm_rope_append(
        _ptr(q), _ptr(k), _ptr(v), T, hq, _ptr(q_norm_weight), _ptr(k_norm_weight), _ptr(positions),
        _ptr(slot_mapping), float(eps), float(rope_theta), _ptr(q_out), _ptr(k_pool), _ptr(v_pool),
        pool_desc(k_pool), _stream(stream)))
    return q_out


def pkv_kv_append_cow(k_new, v_new, token_req, token_pos, page_table, page_refcount, free_pages,
                      free_used, k_pool, v_pool, stream=None):
    """Append rows k_new/v_new [T, Hkv, d] at (token_req, token_pos), copying
    shared pages first; updates page_table, page_refcount and free_used."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _need(t, n, torch.bfloat16, 3)
    for t, n in ((token_req, "token_req"), (token_pos, "token_pos"), (page_refcount, "page_refcount"),
                 (free_pages, "free_pages"), (free_used, "free_used")):
        _need(t, n, torch.int32, 1)
    _need(page_table, "page_table", torch.int32, 2)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    T = k_new.shape[0]
    if v_new.shape != k_new.shape or token_req.shape[0] != T or token_pos.shape[0] != T:
        raise ValueError("k_new, v_new, token_req and token_pos disagree on the token count")
    if page_refcount.shape[0] != k_pool.shape[0] or v_pool.shape != k_pool.shape:
        raise ValueError("page_refcount must have one count per pool page")
    _check("pkv_kv_append_cow", _lib.pkv_kv_append_cow(
        _ptr(k_new), _ptr(v_new), _ptr(token_req), _ptr(token_pos), T, _ptr(page_table),
        page_table.shape[0], page_table.shape[1], _ptr(page_refcount), _ptr(free_pages),
        free_pages.shape[0], _ptr(free_used), _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool),
        _stream(stream)))


# ------------------------------------------------ decode with built-in scratch
_static_decode = _lib.pkv_paged_attn_decode_static
_static_decode.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                           ctypes.c_void_p, _PoolDesc, ctypes.c_void_p, ctypes.c_int32,
                           ctypes.c_void_p, ctypes.c_float, ctypes.c_int32, ctypes.c_void_p,
                           ctypes.c_void_p, ctypes.c_void_p]
_static_decode.restype = ctypes.c_int


def pkv_paged_attn_decode_static(q, k_pool, v_pool, page_table, kv_lens, scale,
                                 partition_tokens=0, out=None, out_lse=None, stream=None):
    """Decode attention like pkv_paged_attn_decode, but with the library's own
    fixed 32 MiB scratch instead of a workspace, for callers that cannot
    allocate device memory when they run decode (code inside another
    allocator's callbacks, plugins that receive only their input and output
    buffers, servers that must not grow their footprint after start-up).

    Allocates nothing itself when ``out`` (and ``out_lse``, if wanted) are
    given.  Every call on a device shares the one scratch array, so calls must
    not overlap on the GPU; the first call on a device looks the array up and
    should come before any stream capture.  Sizes whose split-K scratch
    exceeds 32 MiB are rejected (PkvError, status PKV_ERR_WORKSPACE).
    """
    _need(q, "q", torch.bfloat16, 3)
    _need(k_pool, "k_pool", torch.bfloat16, 4)
    _need(v_pool, "v_pool", torch.bfloat16, 4)
    _need(page_table, "page_table", torch.int32, 2)
    _need(kv_lens, "kv_lens", torch.int32, 1)
    B, hq, d = q.shape
    if page_table.shape[0] != B or kv_lens.shape[0] != B:
        raise ValueError("page_table / kv_lens rows must equal the batch")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", torch.bfloat16, 3)
    if out_lse is not None:
        _need(out_lse, "out_lse", torch.float32, 2)
    _check("pkv_paged_attn_decode_static", _static_decode(
        _ptr(q), B, hq, _ptr(k_pool), _ptr(v_pool), pool_desc(k_pool), _ptr(page_table),
        page_table.shape[1], _ptr(kv_lens), float(scale), int(partition_tokens), _ptr(out),
        _ptr(out_lse), _stream(stream)))
    return out

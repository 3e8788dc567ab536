"""Python binding of libkvdecode.so: one decode step over a paged KV cache.

The functions here carry the C names of ``include/kvdecode.h`` and do argument
marshalling only (tensor checks, pointers, the current CUDA stream).  Every
step of the computation runs in the library's sm_100a kernels; there is no
Python or CPU fallback.  If the shared library is missing, importing this
package raises ImportError.

PyTorch supplies device memory and streams.  All tensors must be CUDA,
contiguous, on the current device.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "KVD_OK", "KVD_ERR_INVALID", "KVD_ERR_UNSUPPORTED", "KVD_ERR_CUDA", "KVD_ERR_WORKSPACE",
    "KVD_F16", "KVD_BF16", "KVD_PAGE_TOKENS", "KvdError",
    "kvd_append", "kvd_decode_attention", "kvd_decode_step", "kvd_decode_attention_static",
    "kvd_decode_attention_shared_prefix", "kvd_shared_prefix_workspace_size",
    "kvd_quantize_fp8", "kvd_append_fp8", "kvd_decode_attention_fp8", "kvd_decode_step_fp8",
    "kvd_quantize_int8", "kvd_append_int8", "kvd_decode_attention_int8", "kvd_decode_step_int8",
    "kvd_quantize_int4", "kvd_append_int4", "kvd_decode_attention_int4", "kvd_decode_step_int4",
    "kvd_decode_attention_shared_prefix_fp8", "kvd_decode_attention_shared_prefix_int8",
    "kvd_decode_attention_shared_prefix_int4",
    "kvd_merge_lse", "kvd_read_stream", "kvd_set_decode_wait_limit", "KVD_READ_VECTOR", "KVD_READ_BULK",
    "kvd_workspace_size", "KVD_STATIC_WORKSPACE_BYTES",
    "kvd_auto_partitions", "kvd_kv_bytes_per_token", "kvd_read_device_error",
    "kvd_last_error", "alloc_workspace", "library_path", "lib",
]

KVD_OK, KVD_ERR_INVALID, KVD_ERR_UNSUPPORTED, KVD_ERR_CUDA, KVD_ERR_WORKSPACE = 0, 1, 2, 3, 4
KVD_F16, KVD_BF16 = 0, 1
KVD_PAGE_TOKENS = 16
KVD_STATIC_WORKSPACE_BYTES = 8 << 20
KVD_DEVERR_BLOCK_TABLE, KVD_DEVERR_SEQ_LEN, KVD_DEVERR_SLOT, KVD_DEVERR_TIMEOUT = 1, 2, 4, 8
KVD_READ_VECTOR, KVD_READ_BULK = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libkvdecode.so")


def _load():
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python kv_cache_decode_scatters_b200/build.py`")
    L = ctypes.CDLL(path)
    P, I, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    L.kvd_append.restype = I
    L.kvd_append.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P]
    L.kvd_decode_attention.restype = I
    L.kvd_decode_attention.argtypes = [P, P, P, P, P, F, P, I, I, I, I, I, I, I, P, S, P, I, P]
    L.kvd_decode_step.restype = I
    L.kvd_decode_step.argtypes = [P, P, P, P, P, P, P, F, P, I, I, I, I, I, I, I, P, S, P, I, P]
    L.kvd_decode_attention_shared_prefix.restype = I
    L.kvd_decode_attention_shared_prefix.argtypes = [P, P, P, P, P, P, P, F, P, I, I, I, I, I, I,
                                                     P, P, I, I, I, P, S, P, I, P]
    L.kvd_shared_prefix_workspace_size.restype = S
    L.kvd_shared_prefix_workspace_size.argtypes = [I, I, I, I, I, I, I]
    LL = ctypes.c_longlong
    for fmt in ("fp8", "int8", "int4"):
        getattr(L, "kvd_quantize_" + fmt).restype = I
        getattr(L, "kvd_quantize_" + fmt).argtypes = [P, P, P, LL, I, I, P]
        getattr(L, "kvd_append_" + fmt).restype = I
        getattr(L, "kvd_append_" + fmt).argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P]
        getattr(L, "kvd_decode_attention_" + fmt).restype = I
        getattr(L, "kvd_decode_attention_" + fmt).argtypes = [P, P, P, P, P, P, P, F, P, I, I, I, I,
                                                              I, I, I, P, S, P, I, P]
        getattr(L, "kvd_decode_step_" + fmt).restype = I
        getattr(L, "kvd_decode_step_" + fmt).argtypes = [P, P, P, P, P, P, P, P, P, F, P, I, I, I,
                                                         I, I, I, I, P, S, P, I, P]
        getattr(L, "kvd_decode_attention_shared_prefix_" + fmt).restype = I
        getattr(L, "kvd_decode_attention_shared_prefix_" + fmt).argtypes = [
            P, P, P, P, P, P, P, P, P, F, P, I, I, I, I, I, I, P, P, I, I, I, P, S, P, I, P]
    L.kvd_decode_attention_static.restype = I
    L.kvd_decode_attention_static.argtypes = [P, P, P, P, P, F, P, I, I, I, I, I, I, P, I, P]
    L.kvd_merge_lse.restype = I
    L.kvd_merge_lse.argtypes = [P, P, P, I, I, I, I, P, P, I, P]
    L.kvd_workspace_size.restype = S
    L.kvd_workspace_size.argtypes = [I, I, I, I, I]
    L.kvd_auto_partitions.restype = I
    L.kvd_auto_partitions.argtypes = []
    L.kvd_kv_bytes_per_token.restype = S
    L.kvd_kv_bytes_per_token.argtypes = [I, I, I, I]
    L.kvd_read_device_error.restype = I
    L.kvd_read_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), I]
    L.kvd_last_error.restype = ctypes.c_char_p
    L.kvd_last_error.argtypes = []
    L.kvd_read_stream.restype = I
    L.kvd_read_stream.argtypes = [P, S, I, P, P]
    L.kvd_set_decode_wait_limit.restype = I
    L.kvd_set_decode_wait_limit.argtypes = [LL]
    return L


_lib = _load()


def lib():
    """The loaded ctypes library (raw C entry points)."""
    return _lib


class KvdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} failed with status {status}: {kvd_last_error()}")


def kvd_last_error() -> str:
    return _lib.kvd_last_error().decode("utf-8", "replace")


def _check(status: int, where: str):
    if status != KVD_OK:
        raise KvdError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return KVD_F16
    if t.dtype == torch.bfloat16:
        return KVD_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (fp16 or bf16)")


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def kvd_kv_bytes_per_token(layers: int, heads: int, d_head: int, dtype_size: int) -> int:
    return int(_lib.kvd_kv_bytes_per_token(layers, heads, d_head, dtype_size))


def kvd_auto_partitions() -> int:
    return int(_lib.kvd_auto_partitions())


def kvd_workspace_size(B: int, H_q: int, H_kv: int, d: int, num_partitions: int = 0) -> int:
    n = int(_lib.kvd_workspace_size(B, H_q, H_kv, d, num_partitions))
    if n == 0 and B > 0:
        raise KvdError(KVD_ERR_INVALID, "kvd_workspace_size")
    return n


def alloc_workspace(B, H_q, H_kv, d, num_partitions=0, device=None) -> torch.Tensor:
    """A uint8 device buffer of kvd_workspace_size bytes (torch's allocator
    returns 256-byte aligned blocks)."""
    n = kvd_workspace_size(B, H_q, H_kv, d, num_partitions)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def kvd_append(k_cache, v_cache, block_table, slot, k_new, v_new, stream=None):
    """Scatter k_new/v_new [B,H_kv,d] into row slot%16 of page
    block_table[b, slot//16] of k_cache/v_cache [NB,H_kv,16,d] (in place)."""
    NB, H_kv, P, d = k_cache.shape
    if P != KVD_PAGE_TOKENS:
        raise ValueError("cache pages must hold 16 tokens")
    B = k_new.shape[0]
    if v_cache.shape != k_cache.shape or tuple(k_new.shape) != (B, H_kv, d) or v_new.shape != k_new.shape:
        raise ValueError("shape mismatch between caches and new K/V")
    dt = k_cache.dtype
    _check(_lib.kvd_append(_dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
                           _dev(block_table, "block_table", torch.int32),
                           _dev(slot, "slot", torch.int32), _dev(k_new, "k_new", dt),
                           _dev(v_new, "v_new", dt), B, H_kv, d, NB, block_table.shape[1],
                           _dtype_code(k_cache), _stream(stream)),
           "kvd_append")


def kvd_decode_attention(q, k_cache, v_cache, block_table, seq_lens, scale=None, out=None,
                         num_partitions=0, workspace=None, lse_out=None, stream=None):
    """out[b, hq] = softmax(scale * q[b, hq] K_b^T) V_b over the seq_lens[b]
    cached tokens of sequence b (KV head hq // (H_q // H_kv)).  Returns out."""
    B, H_q, d = q.shape
    NB, H_kv, P, d2 = k_cache.shape
    if P != KVD_PAGE_TOKENS or d2 != d:
        raise ValueError("q / cache shape mismatch")
    dt = k_cache.dtype
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(B, H_q, H_kv, d, num_partitions, q.device)
    lse_ptr = None if lse_out is None else _dev(lse_out, "lse_out", torch.float32)
    _check(_lib.kvd_decode_attention(
        _dev(q, "q", dt), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(block_table, "block_table", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), _dev(out, "out", dt), B, H_q, H_kv, d, NB, block_table.shape[1],
        int(num_partitions), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        lse_ptr, _dtype_code(k_cache), _stream(stream)),
        "kvd_decode_attention")
    return out


def kvd_decode_step(q, k_new, v_new, k_cache, v_cache, block_table, seq_lens, scale=None,
                    out=None, num_partitions=0, workspace=None, lse_out=None, stream=None):
    """Append k_new/v_new [B,H_kv,d] at position seq_lens[b]-1 of every
    non-empty sequence, then attend (kvd_append + kvd_decode_attention in one
    launch).  Returns out."""
    B, H_q, d = q.shape
    NB, H_kv, P, d2 = k_cache.shape
    if P != KVD_PAGE_TOKENS or d2 != d:
        raise ValueError("q / cache shape mismatch")
    if tuple(k_new.shape) != (B, H_kv, d) or v_new.shape != k_new.shape:
        raise ValueError("k_new / v_new must be [B, H_kv, d]")
    dt = k_cache.dtype
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(B, H_q, H_kv, d, num_partitions, q.device)
    lse_ptr = None if lse_out is None else _dev(lse_out, "lse_out", torch.float32)
    _check(_lib.kvd_decode_step(
        _dev(q, "q", dt), _dev(k_new, "k_new", dt), _dev(v_new, "v_new", dt),
        _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(block_table, "block_table", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), _dev(out, "out", dt), B, H_q, H_kv, d, NB, block_table.shape[1],
        int(num_partitions), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        lse_ptr, _dtype_code(k_cache), _stream(stream)),
        "kvd_decode_step")
    return out


def kvd_shared_prefix_workspace_size(B, H_q, H_kv, d, n_groups, max_group_size, num_partitions=0):
    n = int(_lib.kvd_shared_prefix_workspace_size(B, H_q, H_kv, d, n_groups, max_group_size,
                                                  num_partitions))
    if n == 0 and B > 0:
        raise KvdError(KVD_ERR_INVALID, "kvd_shared_prefix_workspace_size")
    return n


def kvd_decode_attention_shared_prefix(q, k_cache, v_cache, block_table, seq_lens, group_start,
                                       group_pages, max_group_size, scale=None, out=None,
                                       k_new=None, v_new=None, num_partitions=0, workspace=None,
                                       lse_out=None, stream=None):
    """Decode attention over a batch whose groups of consecutive sequences
    share their first group_pages[g] pages (read once per group).  With
    k_new/v_new it also appends the step's token as kvd_decode_step does."""
    B, H_q, d = q.shape
    NB, H_kv, P, d2 = k_cache.shape
    if P != KVD_PAGE_TOKENS or d2 != d:
        raise ValueError("q / cache shape mismatch")
    n_groups = group_pages.shape[0]
    if group_start.shape[0] != n_groups + 1:
        raise ValueError("group_start must have n_groups + 1 entries")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new or neither")
    dt = k_cache.dtype
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = kvd_shared_prefix_workspace_size(B, H_q, H_kv, d, n_groups, max_group_size, num_partitions)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    kn = None if k_new is None else _dev(k_new, "k_new", dt)
    vn = None if v_new is None else _dev(v_new, "v_new", dt)
    lse_ptr = None if lse_out is None else _dev(lse_out, "lse_out", torch.float32)
    _check(_lib.kvd_decode_attention_shared_prefix(
        _dev(q, "q", dt), kn, vn, _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(block_table, "block_table", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), _dev(out, "out", dt), B, H_q, H_kv, d, NB, block_table.shape[1],
        _dev(group_start, "group_start", torch.int32), _dev(group_pages, "group_pages", torch.int32),
        n_groups, int(max_group_size), int(num_partitions), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), lse_ptr, _dtype_code(k_cache), _stream(stream)),
        "kvd_decode_attention_shared_prefix")
    return out


# Quantised KV caches: E4M3 codes (torch.uint8 storage), INT8 codes (torch.int8)
# or INT4 codes two per byte (torch.uint8), one fp32 scale per (token, KV head,
# 32 channels).
_CODE8 = {"fp8": torch.uint8, "int8": torch.int8, "int4": torch.uint8}
# code bytes of a row of d values
_ROW = {"fp8": lambda d: d, "int8": lambda d: d, "int4": lambda d: d // 2}


def _quantize8(fmt, src, codes, scales, stream):
    d = src.shape[-1]
    n = src.numel() // d
    if codes is None:
        codes = torch.empty(src.shape[:-1] + (_ROW[fmt](d),), dtype=_CODE8[fmt], device=src.device)
    if scales is None:
        scales = torch.empty(src.shape[:-1] + (d // 32,), dtype=torch.float32, device=src.device)
    _check(getattr(_lib, "kvd_quantize_" + fmt)(
        _dev(src, "src"), _dev(codes, "codes", _CODE8[fmt]), _dev(scales, "scales", torch.float32), n, d,
        _dtype_code(src), _stream(stream)), "kvd_quantize_" + fmt)
    return codes, scales


def _append8(fmt, k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, stream):
    NB, H_kv, P, _ = k_codes.shape
    d = k_new.shape[-1]
    B = k_new.shape[0]
    c = _CODE8[fmt]
    _check(getattr(_lib, "kvd_append_" + fmt)(
        _dev(k_codes, "k_codes", c), _dev(v_codes, "v_codes", c),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        _dev(block_table, "block_table", torch.int32), _dev(slot, "slot", torch.int32),
        _dev(k_new, "k_new", k_new.dtype), _dev(v_new, "v_new", k_new.dtype),
        B, H_kv, d, NB, block_table.shape[1], _dtype_code(k_new), _stream(stream)), "kvd_append_" + fmt)


def _decode8(fmt, q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out,
             num_partitions, workspace, lse_out, stream, k_new=None, v_new=None):
    B, H_q, d = q.shape
    NB, H_kv, P, rb = k_codes.shape
    if P != KVD_PAGE_TOKENS or rb != _ROW[fmt](d):
        raise ValueError("q / cache shape mismatch")
    step = k_new is not None
    if step and (tuple(k_new.shape) != (B, H_kv, d) or v_new is None or v_new.shape != k_new.shape):
        raise ValueError("k_new / v_new must be [B, H_kv, d]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(B, H_q, H_kv, d, num_partitions, q.device)
    lse_ptr = None if lse_out is None else _dev(lse_out, "lse_out", torch.float32)
    c = _CODE8[fmt]
    name = ("kvd_decode_step_" if step else "kvd_decode_attention_") + fmt
    new = (_dev(k_new, "k_new", q.dtype), _dev(v_new, "v_new", q.dtype)) if step else ()
    _check(getattr(_lib, name)(
        _dev(q, "q", q.dtype), *new, _dev(k_codes, "k_codes", c), _dev(v_codes, "v_codes", c),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        _dev(block_table, "block_table", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), _dev(out, "out", q.dtype), B, H_q, H_kv, d, NB, block_table.shape[1],
        int(num_partitions), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        lse_ptr, _dtype_code(q), _stream(stream)), name)
    return out


def _shared_prefix8(fmt, q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, group_start,
                    group_pages, max_group_size, scale, out, k_new, v_new, num_partitions, workspace,
                    lse_out, stream):
    B, H_q, d = q.shape
    NB, H_kv, P, rb = k_codes.shape
    if P != KVD_PAGE_TOKENS or rb != _ROW[fmt](d):
        raise ValueError("q / cache shape mismatch")
    n_groups = group_pages.shape[0]
    if group_start.shape[0] != n_groups + 1:
        raise ValueError("group_start must have n_groups + 1 entries")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new or neither")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = kvd_shared_prefix_workspace_size(B, H_q, H_kv, d, n_groups, max_group_size, num_partitions)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    kn = None if k_new is None else _dev(k_new, "k_new", q.dtype)
    vn = None if v_new is None else _dev(v_new, "v_new", q.dtype)
    lse_ptr = None if lse_out is None else _dev(lse_out, "lse_out", torch.float32)
    c = _CODE8[fmt]
    name = "kvd_decode_attention_shared_prefix_" + fmt
    _check(getattr(_lib, name)(
        _dev(q, "q", q.dtype), kn, vn, _dev(k_codes, "k_codes", c), _dev(v_codes, "v_codes", c),
        _dev(k_scale, "k_scale", torch.float32), _dev(v_scale, "v_scale", torch.float32),
        _dev(block_table, "block_table", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), _dev(out, "out", q.dtype), B, H_q, H_kv, d, NB, block_table.shape[1],
        _dev(group_start, "group_start", torch.int32), _dev(group_pages, "group_pages", torch.int32),
        n_groups, int(max_group_size), int(num_partitions), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), lse_ptr, _dtype_code(q), _stream(stream)), name)
    return out


def kvd_decode_attention_shared_prefix_fp8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                                           group_start, group_pages, max_group_size, scale=None,
                                           out=None, k_new=None, v_new=None, num_partitions=0,
                                           workspace=None, lse_out=None, stream=None):
    """kvd_decode_attention_shared_prefix over the E4M3 cache (d = 64 or 128); with
    k_new/v_new the step's token is quantised and appended as in
    kvd_decode_step_fp8.  Returns out."""
    return _shared_prefix8("fp8", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                           group_start, group_pages, max_group_size, scale, out, k_new, v_new,
                           num_partitions, workspace, lse_out, stream)


def kvd_decode_attention_shared_prefix_int8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                                            group_start, group_pages, max_group_size, scale=None,
                                            out=None, k_new=None, v_new=None, num_partitions=0,
                                            workspace=None, lse_out=None, stream=None):
    """kvd_decode_attention_shared_prefix over the INT8 cache (d = 64 or 128).  Returns out."""
    return _shared_prefix8("int8", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                           group_start, group_pages, max_group_size, scale, out, k_new, v_new,
                           num_partitions, workspace, lse_out, stream)


def kvd_decode_attention_shared_prefix_int4(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                                            group_start, group_pages, max_group_size, scale=None,
                                            out=None, k_new=None, v_new=None, num_partitions=0,
                                            workspace=None, lse_out=None, stream=None):
    """kvd_decode_attention_shared_prefix over the INT4 cache (d = 64 or 128).  Returns out."""
    return _shared_prefix8("int4", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                           group_start, group_pages, max_group_size, scale, out, k_new, v_new,
                           num_partitions, workspace, lse_out, stream)


def kvd_quantize_fp8(src, codes=None, scales=None, stream=None):
    """Quantise rows src [..., d] (fp16/bf16) into E4M3 codes (uint8 [..., d])
    and fp32 scales [..., d/32], one per 32 channels.  Returns (codes, scales)."""
    return _quantize8("fp8", src, codes, scales, stream)


def kvd_append_fp8(k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, stream=None):
    """kvd_append for the 8-bit cache (codes [NB,H_kv,16,d], scales [NB,H_kv,16,d/32])."""
    _append8("fp8", k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, stream)


def kvd_decode_attention_fp8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale=None,
                             out=None, num_partitions=0, workspace=None, lse_out=None, stream=None):
    """kvd_decode_attention over the E4M3 cache (d = 64 or 128).  Returns out (q's dtype)."""
    return _decode8("fp8", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out,
                    num_partitions, workspace, lse_out, stream)


def kvd_decode_step_fp8(q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                        scale=None, out=None, num_partitions=0, workspace=None, lse_out=None,
                        stream=None):
    """kvd_decode_step over the E4M3 cache: quantise k_new/v_new [B,H_kv,d] into
    position seq_lens[b]-1 of every non-empty sequence, then attend
    (kvd_append_fp8 + kvd_decode_attention_fp8 in one launch).  Returns out."""
    return _decode8("fp8", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out,
                    num_partitions, workspace, lse_out, stream, k_new, v_new)


def kvd_quantize_int4(src, codes=None, scales=None, stream=None):
    """Quantise rows src [..., d] (fp16/bf16) into INT4 codes, two per byte
    (uint8 [..., d/2], channel 2i in the low nibble of byte i), and fp32
    scales [..., d/32].  Returns (codes, scales)."""
    return _quantize8("int4", src, codes, scales, stream)


def kvd_append_int4(k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, stream=None):
    """kvd_append for the INT4 cache (codes [NB,H_kv,16,d/2], scales [NB,H_kv,16,d/32])."""
    _append8("int4", k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, stream)


def kvd_decode_attention_int4(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale=None,
                              out=None, num_partitions=0, workspace=None, lse_out=None, stream=None):
    """kvd_decode_attention over the INT4 cache (d = 64 or 128).  Returns out."""
    return _decode8("int4", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out,
                    num_partitions, workspace, lse_out, stream)


def kvd_decode_step_int4(q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                         scale=None, out=None, num_partitions=0, workspace=None, lse_out=None,
                         stream=None):
    """kvd_decode_step over the INT4 cache (kvd_append_int4 + kvd_decode_attention_int4
    in one launch).  Returns out."""
    return _decode8("int4", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out,
                    num_partitions, workspace, lse_out, stream, k_new, v_new)


def kvd_quantize_int8(src, codes=None, scales=None, stream=None):
    """Quantise rows src [..., d] (fp16/bf16) into INT8 codes (int8 [..., d])
    and fp32 scales [..., d/32], one per 32 channels.  Returns (codes, scales)."""
    return _quantize8("int8", src, codes, scales, stream)


def kvd_append_int8(k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, stream=None):
    """kvd_append for the INT8 cache (codes [NB,H_kv,16,d], scales [NB,H_kv,16,d/32])."""
    _append8("int8", k_codes, v_codes, k_scale, v_scale, block_table, slot, k_new, v_new, stream)


def kvd_decode_attention_int8(q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale=None,
                              out=None, num_partitions=0, workspace=None, lse_out=None, stream=None):
    """kvd_decode_attention over the INT8 cache (d = 128).  Returns out (q's dtype)."""
    return _decode8("int8", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out,
                    num_partitions, workspace, lse_out, stream)


def kvd_decode_step_int8(q, k_new, v_new, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens,
                         scale=None, out=None, num_partitions=0, workspace=None, lse_out=None,
                         stream=None):
    """kvd_decode_step over the INT8 cache (kvd_append_int8 + kvd_decode_attention_int8
    in one launch).  Returns out."""
    return _decode8("int8", q, k_codes, v_codes, k_scale, v_scale, block_table, seq_lens, scale, out,
                    num_partitions, workspace, lse_out, stream, k_new, v_new)


def kvd_decode_attention_static(q, k_cache, v_cache, block_table, seq_lens, scale=None, out=None,
                                lse_out=None, stream=None):
    """kvd_decode_attention without a workspace argument, for callers that
    cannot allocate device memory: the scratch is the library's fixed
    KVD_STATIC_WORKSPACE_BYTES array (shared by every call on a device, so
    calls overlapping on the GPU race).  `out` must be given by such callers;
    when it is None this wrapper allocates it with torch for convenience."""
    B, H_q, d = q.shape
    NB, H_kv, P, d2 = k_cache.shape
    if P != KVD_PAGE_TOKENS or d2 != d:
        raise ValueError("q / cache shape mismatch")
    dt = k_cache.dtype
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    lse_ptr = None if lse_out is None else _dev(lse_out, "lse_out", torch.float32)
    _check(_lib.kvd_decode_attention_static(
        _dev(q, "q", dt), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(block_table, "block_table", torch.int32), _dev(seq_lens, "seq_lens", torch.int32),
        float(scale), _dev(out, "out", dt), B, H_q, H_kv, d, NB, block_table.shape[1],
        lse_ptr, _dtype_code(k_cache), _stream(stream)),
        "kvd_decode_attention_static")
    return out


def kvd_merge_lse(part_o, part_lse, num_splits_per_seq=None, out=None, lse_out=None,
                  dtype=torch.float16, stream=None):
    """Merge partials part_o [B,H_q,S,d] (fp32), part_lse [B,H_q,S] into out [B,H_q,d]."""
    B, H_q, S, d = part_o.shape
    if out is None:
        out = torch.empty((B, H_q, d), dtype=dtype, device=part_o.device)
    cnt = None if num_splits_per_seq is None else _dev(num_splits_per_seq, "num_splits_per_seq", torch.int32)
    lse_ptr = None if lse_out is None else _dev(lse_out, "lse_out", torch.float32)
    _check(_lib.kvd_merge_lse(_dev(part_o, "part_o", torch.float32),
                              _dev(part_lse, "part_lse", torch.float32), cnt, B, H_q, d, S,
                              _dev(out, "out"), lse_ptr, _dtype_code(out), _stream(stream)),
           "kvd_merge_lse")
    return out


def kvd_read_device_error(clear: bool = True) -> int:
    """Device error bits (KVD_DEVERR_*) since the last clear; synchronises."""
    flags = ctypes.c_uint(0)
    _check(_lib.kvd_read_device_error(ctypes.byref(flags), 1 if clear else 0),
           "kvd_read_device_error")
    return int(flags.value)


def kvd_set_decode_wait_limit(polls: int) -> None:
    """Testing hook: poll limit of the decode kernel's page waits for later
    launches (0 = give up at once and flag KVD_DEVERR_TIMEOUT; negative =
    the default).  Copies in flight are always drained with the full limit."""
    _check(_lib.kvd_set_decode_wait_limit(int(polls)), "kvd_set_decode_wait_limit")


def kvd_read_stream(buf: torch.Tensor, mode: int = KVD_READ_BULK, sink=None, stream=None):
    """Read every byte of the contiguous device tensor `buf` once (mode
    KVD_READ_VECTOR or KVD_READ_BULK), XOR-folding its 32-bit words into
    `sink` (a 1-element int32 device tensor, zeroed here if not given).
    Returns sink."""
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
    nbytes = buf.numel() * buf.element_size()
    _check(_lib.kvd_read_stream(_dev(buf, "buf"), nbytes, int(mode), _dev(sink, "sink", torch.int32),
                                _stream(stream)), "kvd_read_stream")
    return sink

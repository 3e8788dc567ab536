"""CPU oracle for one paged-KV decode step (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  It shares no code with the CUDA
library in ``kv_cache_decode_scatters_b200`` and never imports it.

The arithmetic lives in ``oracle.c`` (binary64, OpenMP over query rows); this
module only marshals numpy arrays into it.  Storage tensors (fp16 / bf16) are
passed as their raw 16-bit words (``uint16``), so the oracle decodes every
value itself.
"""
import ctypes

import numpy as np

from . import build as _build

F16 = 0
BF16 = 1
PAGE_TOKENS = 16

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def load(path):
    """Open an oracle shared library at `path` and declare its signatures."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32 = ctypes.c_int
    L.orc_f16_to_f64.restype = ctypes.c_double
    L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
    L.orc_bf16_to_f64.restype = ctypes.c_double
    L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
    L.orc_kv_bytes_per_token.restype = ctypes.c_longlong
    L.orc_kv_bytes_per_token.argtypes = [i32, i32, i32, i32]
    L.orc_append.restype = i32
    L.orc_append.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32]
    L.orc_attend.restype = i32
    L.orc_attend.argtypes = [P, P, P, P, P, P, P, ctypes.c_double,
                             i32, i32, i32, i32, i32, i32, i32, P, P, i32]
    L.orc_attend_tiled.restype = i32
    L.orc_attend_tiled.argtypes = [P, P, P, P, P, ctypes.c_double,
                                   i32, i32, i32, i32, i32, i32, i32, i32, P]
    L.orc_merge.restype = i32
    L.orc_merge.argtypes = [P, P, P, i32, i32, i32, i32, P, P]
    L.orc_max_threads.restype = i32
    L.orc_max_threads.argtypes = []
    L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [ctypes.c_float]
    L.orc_quantize_fp8.restype = i32
    L.orc_quantize_fp8.argtypes = [P, i32, i32, i32, P, P]
    L.orc_append_fp8.restype = i32
    L.orc_append_fp8.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32]
    L.orc_attend_fp8.restype = i32
    L.orc_attend_fp8.argtypes = [P, P, P, P, P, P, P, ctypes.c_double, i32, i32, i32, i32, i32,
                                 i32, i32, P, P, i32]
    L.orc_int8_decode.restype = ctypes.c_double
    L.orc_int8_decode.argtypes = [ctypes.c_uint8]
    L.orc_int8_encode.restype = ctypes.c_uint8
    L.orc_int8_encode.argtypes = [ctypes.c_float]
    L.orc_quantize_int8.restype = i32
    L.orc_quantize_int8.argtypes = [P, i32, i32, i32, P, P]
    L.orc_append_int8.restype = i32
    L.orc_append_int8.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32]
    L.orc_attend_int8.restype = i32
    L.orc_attend_int8.argtypes = [P, P, P, P, P, P, P, ctypes.c_double, i32, i32, i32, i32, i32,
                                  i32, i32, P, P, i32]
    L.orc_int4_decode.restype = ctypes.c_double
    L.orc_int4_decode.argtypes = [ctypes.c_uint8]
    L.orc_int4_encode.restype = ctypes.c_uint8
    L.orc_int4_encode.argtypes = [ctypes.c_float]
    L.orc_quantize_int4.restype = i32
    L.orc_quantize_int4.argtypes = [P, i32, i32, i32, P, P]
    L.orc_append_int4.restype = i32
    L.orc_append_int4.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32]
    L.orc_attend_int4.restype = i32
    L.orc_attend_int4.argtypes = [P, P, P, P, P, P, P, ctypes.c_double, i32, i32, i32, i32, i32,
                                  i32, i32, P, P, i32]
    return L


class using_library:
    """Context manager: route every call of this module to another build of
    the oracle (the mutation tests load deliberately broken copies)."""

    def __init__(self, path):
        self._path = path
        self._saved = None

    def __enter__(self):
        global _lib
        self._saved = _lib
        _lib = load(self._path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _words(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"storage arrays must be uint16 words, got {a.dtype}")
    return a


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


def f16_to_f64(word):
    return lib().orc_f16_to_f64(int(word))


def bf16_to_f64(word):
    return lib().orc_bf16_to_f64(int(word))


def kv_bytes_per_token(layers, heads, d_head, dtype_size):
    return int(lib().orc_kv_bytes_per_token(layers, heads, d_head, dtype_size))


def append(k_cache, v_cache, block_table, slot, k_new, v_new):
    """In-place scatter of k_new/v_new [B,H_kv,d] into pools [NB,H_kv,16,d]."""
    k_cache = _words(k_cache)
    v_cache = _words(v_cache)
    k_new, v_new = _words(k_new), _words(v_new)
    bt, sl = _i32(block_table), _i32(slot)
    NB, H_kv, P, d = k_cache.shape
    assert P == PAGE_TOKENS
    B = k_new.shape[0]
    _check(lib().orc_append(_ptr(k_cache), _ptr(v_cache), _ptr(bt), _ptr(sl),
                            _ptr(k_new), _ptr(v_new), B, H_kv, d, NB, bt.shape[1]),
           "orc_append")
    return k_cache, v_cache


def attend(q, k_cache, v_cache, block_table, seq_lens, scale, dtype,
           lo=None, hi=None, nthreads=0):
    """One-shot attention (binary64).  Returns (out [B,H_q,d], lse [B,H_q])."""
    q = _words(q)
    k_cache, v_cache = _words(k_cache), _words(v_cache)
    bt, sl = _i32(block_table), _i32(seq_lens)
    B, H_q, d = q.shape
    NB, H_kv, P, d2 = k_cache.shape
    assert P == PAGE_TOKENS and d2 == d
    out = np.zeros((B, H_q, d), dtype=np.float64)
    lse = np.zeros((B, H_q), dtype=np.float64)
    lo, hi = _i32(lo), _i32(hi)
    _check(lib().orc_attend(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt), _ptr(sl),
                            _ptr(lo), _ptr(hi), float(scale), B, H_q, H_kv, d, NB,
                            bt.shape[1], dtype, _ptr(out), _ptr(lse), int(nthreads)),
           "orc_attend")
    return out, lse


def attend_tiled(q, k_cache, v_cache, block_table, seq_lens, scale, dtype, tile):
    q = _words(q)
    k_cache, v_cache = _words(k_cache), _words(v_cache)
    bt, sl = _i32(block_table), _i32(seq_lens)
    B, H_q, d = q.shape
    NB, H_kv, P, _ = k_cache.shape
    out = np.zeros((B, H_q, d), dtype=np.float64)
    _check(lib().orc_attend_tiled(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(bt), _ptr(sl),
                                  float(scale), B, H_q, H_kv, d, NB, bt.shape[1], dtype,
                                  int(tile), _ptr(out)),
           "orc_attend_tiled")
    return out


def merge(part_o, part_lse, counts=None):
    """Merge partials part_o [B,H_q,S,d], part_lse [B,H_q,S] -> (out, lse)."""
    part_o = np.ascontiguousarray(part_o, dtype=np.float64)
    part_lse = np.ascontiguousarray(part_lse, dtype=np.float64)
    B, H_q, S, d = part_o.shape
    out = np.zeros((B, H_q, d), dtype=np.float64)
    lse = np.zeros((B, H_q), dtype=np.float64)
    c = _i32(counts)
    _check(lib().orc_merge(_ptr(part_o), _ptr(part_lse), _ptr(c), B, H_q, d, S,
                           _ptr(out), _ptr(lse)),
           "orc_merge")
    return out, lse


def max_threads():
    return int(lib().orc_max_threads())


# ------------------------------------------------------------ 8-bit KV cache

FP8_GROUP = 32


def e4m3_decode(code):
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(x):
    return int(lib().orc_e4m3_encode(float(x)))


def _quantize8(fn, rows, dtype):
    rows = _words(rows)
    d = rows.shape[-1]
    n = rows.size // d
    codes = np.zeros(rows.shape, dtype=np.uint8)
    scales = np.zeros(rows.shape[:-1] + (d // FP8_GROUP,), dtype=np.float32)
    _check(getattr(lib(), fn)(_ptr(rows), n, d, dtype, _ptr(codes), _ptr(scales)), fn)
    return codes, scales


def _append8(fn, k8, v8, ks, vs, block_table, slot, k_new, v_new, dtype):
    for a in (k8, v8):
        assert a.dtype == np.uint8 and a.flags.c_contiguous
    for a in (ks, vs):
        assert a.dtype == np.float32 and a.flags.c_contiguous
    k_new, v_new = _words(k_new), _words(v_new)
    bt, sl = _i32(block_table), _i32(slot)
    NB, H_kv, P, d = k8.shape
    _check(getattr(lib(), fn)(_ptr(k8), _ptr(v8), _ptr(ks), _ptr(vs), _ptr(bt), _ptr(sl),
                              _ptr(k_new), _ptr(v_new), k_new.shape[0], H_kv, d, NB,
                              bt.shape[1], dtype), fn)


def _attend8(fn, q, k8, v8, ks, vs, block_table, seq_lens, scale, dtype, nthreads):
    q = _words(q)
    bt, sl = _i32(block_table), _i32(seq_lens)
    B, H_q, d = q.shape
    NB, H_kv, P, _ = k8.shape
    out = np.zeros((B, H_q, d), dtype=np.float64)
    lse = np.zeros((B, H_q), dtype=np.float64)
    _check(getattr(lib(), fn)(_ptr(q), _ptr(np.ascontiguousarray(k8)), _ptr(np.ascontiguousarray(v8)),
                              _ptr(np.ascontiguousarray(ks)), _ptr(np.ascontiguousarray(vs)),
                              _ptr(bt), _ptr(sl), float(scale), B, H_q, H_kv, d, NB,
                              bt.shape[1], dtype, _ptr(out), _ptr(lse), int(nthreads)), fn)
    return out, lse


def quantize_fp8(rows, dtype):
    """rows [..., d] storage words -> (codes uint8 [..., d], scales float32 [..., d/32])."""
    return _quantize8("orc_quantize_fp8", rows, dtype)


def append_fp8(k8, v8, ks, vs, block_table, slot, k_new, v_new, dtype):
    """In-place quantised scatter into codes [NB,H_kv,16,d] and scales [NB,H_kv,16,d/32]."""
    _append8("orc_append_fp8", k8, v8, ks, vs, block_table, slot, k_new, v_new, dtype)


def attend_fp8(q, k8, v8, ks, vs, block_table, seq_lens, scale, dtype, nthreads=0):
    """Attention (binary64) over the dequantised 8-bit cache -> (out, lse)."""
    return _attend8("orc_attend_fp8", q, k8, v8, ks, vs, block_table, seq_lens, scale, dtype,
                    nthreads)


def int8_decode(code):
    return lib().orc_int8_decode(int(code))


def int8_encode(x):
    return int(lib().orc_int8_encode(float(x)))


def quantize_int8(rows, dtype):
    """rows [..., d] storage words -> (codes as uint8 bytes of int8 [..., d], scales [..., d/32])."""
    return _quantize8("orc_quantize_int8", rows, dtype)


def append_int8(k8, v8, ks, vs, block_table, slot, k_new, v_new, dtype):
    """In-place INT8 quantised scatter (same layout as append_fp8)."""
    _append8("orc_append_int8", k8, v8, ks, vs, block_table, slot, k_new, v_new, dtype)


def attend_int8(q, k8, v8, ks, vs, block_table, seq_lens, scale, dtype, nthreads=0):
    """Attention (binary64) over the dequantised INT8 cache -> (out, lse)."""
    return _attend8("orc_attend_int8", q, k8, v8, ks, vs, block_table, seq_lens, scale, dtype,
                    nthreads)


# ------------------------------------------------------------ 4-bit KV cache

def int4_decode(nibble):
    return lib().orc_int4_decode(int(nibble))


def int4_encode(x):
    return int(lib().orc_int4_encode(float(x)))


def quantize_int4(rows, dtype):
    """rows [..., d] storage words -> (packed codes uint8 [..., d/2]: channel 2i
    in the low nibble of byte i, 2i+1 in its high nibble; scales [..., d/32])."""
    rows = _words(rows)
    d = rows.shape[-1]
    n = rows.size // d
    codes = np.zeros(rows.shape[:-1] + (d // 2,), dtype=np.uint8)
    scales = np.zeros(rows.shape[:-1] + (d // FP8_GROUP,), dtype=np.float32)
    _check(lib().orc_quantize_int4(_ptr(rows), n, d, dtype, _ptr(codes), _ptr(scales)),
           "orc_quantize_int4")
    return codes, scales


def append_int4(k4, v4, ks, vs, block_table, slot, k_new, v_new, dtype):
    """In-place INT4 quantised scatter into packed codes [NB,H_kv,16,d/2] and
    scales [NB,H_kv,16,d/32]."""
    for a in (k4, v4):
        assert a.dtype == np.uint8 and a.flags.c_contiguous
    for a in (ks, vs):
        assert a.dtype == np.float32 and a.flags.c_contiguous
    k_new, v_new = _words(k_new), _words(v_new)
    bt, sl = _i32(block_table), _i32(slot)
    NB, H_kv, P, half = k4.shape
    _check(lib().orc_append_int4(_ptr(k4), _ptr(v4), _ptr(ks), _ptr(vs), _ptr(bt), _ptr(sl),
                                 _ptr(k_new), _ptr(v_new), k_new.shape[0], H_kv, 2 * half, NB,
                                 bt.shape[1], dtype), "orc_append_int4")


def attend_int4(q, k4, v4, ks, vs, block_table, seq_lens, scale, dtype, nthreads=0):
    """Attention (binary64) over the dequantised INT4 cache -> (out, lse)."""
    q = _words(q)
    bt, sl = _i32(block_table), _i32(seq_lens)
    B, H_q, d = q.shape
    NB, H_kv, P, _ = k4.shape
    out = np.zeros((B, H_q, d), dtype=np.float64)
    lse = np.zeros((B, H_q), dtype=np.float64)
    _check(lib().orc_attend_int4(_ptr(q), _ptr(np.ascontiguousarray(k4)), _ptr(np.ascontiguousarray(v4)),
                                 _ptr(np.ascontiguousarray(ks)), _ptr(np.ascontiguousarray(vs)),
                                 _ptr(bt), _ptr(sl), float(scale), B, H_q, H_kv, d, NB,
                                 bt.shape[1], dtype, _ptr(out), _ptr(lse), int(nthreads)),
           "orc_attend_int4")
    return out, lse

"""The C-ABI library loads, exports every declared entry point and validates
arguments on the host (no GPU needed: every call here returns before any
CUDA work)."""
import ctypes
import os
import re
import subprocess

import pytest

import kv_cache_decode_scatters_b200 as kvd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvdecode.h")


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvd_\w+)\s*\(", text)))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("kvd_append", "kvd_decode_attention", "kvd_merge_lse"):
        assert n in names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", kvd.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(kvd_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for n in names:
        assert hasattr(kvd.lib(), n)


def test_library_has_no_dynamic_cuda_dependency():
    out = subprocess.run(["ldd", kvd.library_path()], capture_output=True, text=True).stdout
    assert "not found" not in out


@pytest.mark.parametrize("args,expect", [
    ((32, 32, 128, 2), 524288),
    ((1, 8, 128, 2), 4096),
    ((1, 1, 128, 2), 512),
    ((80, 8, 128, 2), 327680),
    ((-1, 8, 128, 2), 0),
])
def test_kv_bytes_per_token(args, expect):
    assert kvd.kvd_kv_bytes_per_token(*args) == expect


L = kvd.lib()
NULL = None
DUMMY = ctypes.c_void_p(256)          # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(256 + 2)


def decode(**kw):
    a = dict(q=DUMMY, k=DUMMY, v=DUMMY, bt=DUMMY, sl=DUMMY, scale=0.125, out=DUMMY,
             B=2, H_q=8, H_kv=2, d=128, NB=16, maxb=4, parts=4, ws=DUMMY, wsb=1 << 30,
             lse=NULL, dt=kvd.KVD_F16, stream=NULL)
    a.update(kw)
    return L.kvd_decode_attention(a["q"], a["k"], a["v"], a["bt"], a["sl"], a["scale"], a["out"],
                                  a["B"], a["H_q"], a["H_kv"], a["d"], a["NB"], a["maxb"],
                                  a["parts"], a["ws"], a["wsb"], a["lse"], a["dt"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), kvd.KVD_ERR_UNSUPPORTED),
    (dict(H_q=6, H_kv=4), kvd.KVD_ERR_UNSUPPORTED),
    (dict(H_q=34, H_kv=2), kvd.KVD_ERR_UNSUPPORTED),        # group 17 > 16
    (dict(B=5000), kvd.KVD_ERR_UNSUPPORTED),
    (dict(B=-1), kvd.KVD_ERR_INVALID),
    (dict(H_kv=0), kvd.KVD_ERR_INVALID),
    (dict(NB=0), kvd.KVD_ERR_INVALID),
    (dict(dt=7), kvd.KVD_ERR_INVALID),
    (dict(q=NULL), kvd.KVD_ERR_INVALID),
    (dict(out=NULL), kvd.KVD_ERR_INVALID),
    (dict(q=MISALIGNED), kvd.KVD_ERR_INVALID),
    (dict(parts=-1), kvd.KVD_ERR_INVALID),
    (dict(scale=float("nan")), kvd.KVD_ERR_INVALID),
    (dict(NB=1 << 26, H_kv=2), kvd.KVD_ERR_UNSUPPORTED),  # 2^26 * 2 * 16 >= 2^31
    (dict(ws=NULL), kvd.KVD_ERR_WORKSPACE),
    (dict(wsb=16), kvd.KVD_ERR_WORKSPACE),
    (dict(ws=ctypes.c_void_p(256 + 16)), kvd.KVD_ERR_INVALID),
])
def test_decode_validation(kw, status):
    assert decode(**kw) == status
    assert kvd.kvd_last_error() != ""


def test_step_requires_new_rows():
    a = (DUMMY, NULL, DUMMY, DUMMY, DUMMY, DUMMY, DUMMY, 0.125, DUMMY, 2, 8, 2, 128, 16, 4, 4,
         DUMMY, 1 << 30, NULL, kvd.KVD_F16, NULL)
    assert L.kvd_decode_step(*a) == kvd.KVD_ERR_INVALID
    b = list(a)
    b[1], b[2] = MISALIGNED, DUMMY
    assert L.kvd_decode_step(*b) == kvd.KVD_ERR_INVALID


def test_decode_empty_batch_is_a_no_op():
    assert decode(B=0, q=NULL, out=NULL, ws=NULL) == kvd.KVD_OK


def static(**kw):
    a = dict(q=DUMMY, k=DUMMY, v=DUMMY, bt=DUMMY, sl=DUMMY, scale=0.125, out=DUMMY,
             B=2, H_q=8, H_kv=2, d=128, NB=16, maxb=4, lse=NULL, dt=kvd.KVD_F16, stream=NULL)
    a.update(kw)
    return L.kvd_decode_attention_static(a["q"], a["k"], a["v"], a["bt"], a["sl"], a["scale"],
                                         a["out"], a["B"], a["H_q"], a["H_kv"], a["d"], a["NB"],
                                         a["maxb"], a["lse"], a["dt"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), kvd.KVD_ERR_UNSUPPORTED),
    (dict(H_q=6, H_kv=4), kvd.KVD_ERR_UNSUPPORTED),
    (dict(B=5000), kvd.KVD_ERR_UNSUPPORTED),
    (dict(B=-1), kvd.KVD_ERR_INVALID),
    (dict(H_q=0), kvd.KVD_ERR_INVALID),
    (dict(dt=7), kvd.KVD_ERR_INVALID),
    (dict(scale=float("nan")), kvd.KVD_ERR_INVALID),
    (dict(q=MISALIGNED), kvd.KVD_ERR_INVALID),
    # an empty batch is still validated
    (dict(B=0, dt=7), kvd.KVD_ERR_INVALID),
    (dict(B=0, d=96), kvd.KVD_ERR_UNSUPPORTED),
    (dict(B=0, H_q=6, H_kv=4), kvd.KVD_ERR_UNSUPPORTED),
    (dict(B=0, scale=float("nan")), kvd.KVD_ERR_INVALID),
])
def test_static_validation_matches_workspace_entry_point(kw, status):
    # the fixed-scratch entry point rejects a bad call with the status (and
    # the message) of kvd_decode_attention, before any device work
    assert static(**kw) == status
    msg = kvd.kvd_last_error()
    assert msg != ""
    assert decode(parts=0, **kw) == status
    assert kvd.kvd_last_error() == msg


def test_static_empty_batch_is_a_no_op():
    assert static(B=0, q=NULL, out=NULL) == kvd.KVD_OK


def append(**kw):
    a = dict(k=DUMMY, v=DUMMY, bt=DUMMY, slot=DUMMY, kn=DUMMY, vn=DUMMY, B=2, H_kv=2, d=128,
             NB=16, maxb=4, dt=kvd.KVD_BF16, stream=NULL)
    a.update(kw)
    return L.kvd_append(a["k"], a["v"], a["bt"], a["slot"], a["kn"], a["vn"], a["B"], a["H_kv"],
                        a["d"], a["NB"], a["maxb"], a["dt"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(d=100), kvd.KVD_ERR_UNSUPPORTED),
    (dict(d=136), kvd.KVD_ERR_UNSUPPORTED),
    (dict(B=-3), kvd.KVD_ERR_INVALID),
    (dict(H_kv=0), kvd.KVD_ERR_INVALID),
    (dict(maxb=0), kvd.KVD_ERR_INVALID),
    (dict(k=NULL), kvd.KVD_ERR_INVALID),
    (dict(slot=NULL), kvd.KVD_ERR_INVALID),
    (dict(vn=MISALIGNED), kvd.KVD_ERR_INVALID),
    (dict(dt=-1), kvd.KVD_ERR_INVALID),
])
def test_append_validation(kw, status):
    assert append(**kw) == status


def test_append_empty_batch_is_a_no_op():
    assert append(B=0, k=NULL) == kvd.KVD_OK


@pytest.mark.parametrize("kw,status", [
    (dict(d=32), kvd.KVD_ERR_UNSUPPORTED),
    (dict(S=0), kvd.KVD_ERR_INVALID),
    (dict(po=NULL), kvd.KVD_ERR_INVALID),
    (dict(dt=3), kvd.KVD_ERR_INVALID),
])
def test_merge_validation(kw, status):
    a = dict(po=DUMMY, pl=DUMMY, cnt=NULL, B=2, H_q=4, d=128, S=3, out=DUMMY, lse=NULL,
             dt=kvd.KVD_F16, stream=NULL)
    a.update(kw)
    assert L.kvd_merge_lse(a["po"], a["pl"], a["cnt"], a["B"], a["H_q"], a["d"], a["S"],
                           a["out"], a["lse"], a["dt"], a["stream"]) == status


# ----------------------------------------------------------- 8-bit caches

def decode8(fmt, step=False, **kw):
    a = dict(q=DUMMY, kn=DUMMY, vn=DUMMY, k=DUMMY, v=DUMMY, ks=DUMMY, vs=DUMMY, bt=DUMMY, sl=DUMMY,
             scale=0.125, out=DUMMY, B=2, H_q=8, H_kv=2, d=128, NB=16, maxb=4, parts=4, ws=DUMMY,
             wsb=1 << 30, lse=NULL, dt=kvd.KVD_BF16, stream=NULL)
    a.update(kw)
    tail = (a["k"], a["v"], a["ks"], a["vs"], a["bt"], a["sl"], a["scale"], a["out"], a["B"], a["H_q"],
            a["H_kv"], a["d"], a["NB"], a["maxb"], a["parts"], a["ws"], a["wsb"], a["lse"], a["dt"],
            a["stream"])
    if step:
        return getattr(L, "kvd_decode_step_" + fmt)(a["q"], a["kn"], a["vn"], *tail)
    return getattr(L, "kvd_decode_attention_" + fmt)(a["q"], *tail)


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
@pytest.mark.parametrize("step", [False, True])
@pytest.mark.parametrize("kw,status", [
    (dict(d=96), kvd.KVD_ERR_UNSUPPORTED),                 # the 8-bit tile is d = 64 or 128
    (dict(ks=NULL), kvd.KVD_ERR_INVALID),
    (dict(vs=NULL), kvd.KVD_ERR_INVALID),
    (dict(ks=ctypes.c_void_p(256 + 8)), kvd.KVD_ERR_INVALID),   # scale pools 16-byte aligned
    (dict(k=MISALIGNED), kvd.KVD_ERR_INVALID),
    (dict(H_q=34, H_kv=2), kvd.KVD_ERR_UNSUPPORTED),
    (dict(wsb=16), kvd.KVD_ERR_WORKSPACE),
])
def test_decode8_validation(fmt, step, kw, status):
    assert decode8(fmt, step, **kw) == status
    assert kvd.kvd_last_error() != ""


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
def test_step8_requires_aligned_new_rows(fmt):
    assert decode8(fmt, True, kn=NULL) == kvd.KVD_ERR_INVALID
    assert decode8(fmt, True, vn=MISALIGNED) == kvd.KVD_ERR_INVALID
    assert decode8(fmt, True, B=0, q=NULL, kn=NULL, vn=NULL, out=NULL, ws=NULL) == kvd.KVD_OK


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
@pytest.mark.parametrize("kw,status", [
    (dict(d=48), kvd.KVD_ERR_UNSUPPORTED),
    (dict(d=160), kvd.KVD_ERR_UNSUPPORTED),
    (dict(B=-1), kvd.KVD_ERR_INVALID),
    (dict(ks=NULL), kvd.KVD_ERR_INVALID),
    (dict(kn=MISALIGNED), kvd.KVD_ERR_INVALID),
    (dict(dt=5), kvd.KVD_ERR_INVALID),
])
def test_append8_validation(fmt, kw, status):
    a = dict(k=DUMMY, v=DUMMY, ks=DUMMY, vs=DUMMY, bt=DUMMY, slot=DUMMY, kn=DUMMY, vn=DUMMY, B=2,
             H_kv=2, d=128, NB=16, maxb=4, dt=kvd.KVD_F16, stream=NULL)
    a.update(kw)
    assert getattr(L, "kvd_append_" + fmt)(a["k"], a["v"], a["ks"], a["vs"], a["bt"], a["slot"], a["kn"],
                                            a["vn"], a["B"], a["H_kv"], a["d"], a["NB"], a["maxb"],
                                            a["dt"], a["stream"]) == status


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
@pytest.mark.parametrize("kw,status", [
    (dict(d=40), kvd.KVD_ERR_UNSUPPORTED),
    (dict(n=-1), kvd.KVD_ERR_INVALID),
    (dict(src=NULL), kvd.KVD_ERR_INVALID),
    (dict(n=0, src=NULL), kvd.KVD_OK),
])
def test_quantize8_validation(fmt, kw, status):
    a = dict(src=DUMMY, codes=DUMMY, scales=DUMMY, n=4, d=128, dt=kvd.KVD_BF16, stream=NULL)
    a.update(kw)
    assert getattr(L, "kvd_quantize_" + fmt)(a["src"], a["codes"], a["scales"], a["n"], a["d"], a["dt"],
                                              a["stream"]) == status


# -------------------------------------------------- shared-prefix decode

@pytest.mark.parametrize("kw,status", [
    (dict(ng=-1), kvd.KVD_ERR_INVALID),
    (dict(kn=DUMMY, vn=NULL), kvd.KVD_ERR_INVALID),       # both or neither
    (dict(kn=MISALIGNED, vn=DUMMY), kvd.KVD_ERR_INVALID),
    (dict(gs=NULL), kvd.KVD_ERR_INVALID),
    (dict(gp=NULL), kvd.KVD_ERR_INVALID),
    (dict(mg=0), kvd.KVD_ERR_INVALID),
    (dict(d=96), kvd.KVD_ERR_UNSUPPORTED),
    (dict(q=NULL), kvd.KVD_ERR_INVALID),
])
def test_shared_prefix_validation(kw, status):
    a = dict(q=DUMMY, kn=NULL, vn=NULL, k=DUMMY, v=DUMMY, bt=DUMMY, sl=DUMMY, scale=0.125, out=DUMMY,
             B=4, H_q=8, H_kv=2, d=128, NB=16, maxb=4, gs=DUMMY, gp=DUMMY, ng=2, mg=2, parts=4,
             ws=DUMMY, wsb=1 << 30, lse=NULL, dt=kvd.KVD_F16, stream=NULL)
    a.update(kw)
    st = L.kvd_decode_attention_shared_prefix(
        a["q"], a["kn"], a["vn"], a["k"], a["v"], a["bt"], a["sl"], a["scale"], a["out"], a["B"],
        a["H_q"], a["H_kv"], a["d"], a["NB"], a["maxb"], a["gs"], a["gp"], a["ng"], a["mg"], a["parts"],
        a["ws"], a["wsb"], a["lse"], a["dt"], a["stream"])
    assert st == status
    assert kvd.kvd_last_error() != ""


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
@pytest.mark.parametrize("kw,status", [
    (dict(d=96), kvd.KVD_ERR_UNSUPPORTED),                # quantised prefix passes: d = 64 or 128
    (dict(ng=-1), kvd.KVD_ERR_INVALID),
    (dict(kn=DUMMY, vn=NULL), kvd.KVD_ERR_INVALID),       # both or neither
    (dict(kn=MISALIGNED, vn=DUMMY), kvd.KVD_ERR_INVALID),
    (dict(ks=NULL), kvd.KVD_ERR_INVALID),
    (dict(vs=NULL), kvd.KVD_ERR_INVALID),
    (dict(ks=ctypes.c_void_p(256 + 8)), kvd.KVD_ERR_INVALID),
    (dict(gs=NULL), kvd.KVD_ERR_INVALID),
    (dict(mg=0), kvd.KVD_ERR_INVALID),
])
def test_shared_prefix_quantised_validation(fmt, kw, status):
    a = dict(q=DUMMY, kn=NULL, vn=NULL, k=DUMMY, v=DUMMY, ks=DUMMY, vs=DUMMY, bt=DUMMY, sl=DUMMY,
             scale=0.125, out=DUMMY, B=4, H_q=8, H_kv=2, d=128, NB=16, maxb=4, gs=DUMMY, gp=DUMMY, ng=2,
             mg=2, parts=4, ws=DUMMY, wsb=1 << 30, lse=NULL, dt=kvd.KVD_F16, stream=NULL)
    a.update(kw)
    st = getattr(L, "kvd_decode_attention_shared_prefix_" + fmt)(
        a["q"], a["kn"], a["vn"], a["k"], a["v"], a["ks"], a["vs"], a["bt"], a["sl"], a["scale"],
        a["out"], a["B"], a["H_q"], a["H_kv"], a["d"], a["NB"], a["maxb"], a["gs"], a["gp"], a["ng"],
        a["mg"], a["parts"], a["ws"], a["wsb"], a["lse"], a["dt"], a["stream"])
    assert st == status
    assert kvd.kvd_last_error() != ""


@pytest.mark.parametrize("kw,status", [
    (dict(mode=2), kvd.KVD_ERR_INVALID),
    (dict(nbytes=24), kvd.KVD_ERR_INVALID),
    (dict(src=NULL), kvd.KVD_ERR_INVALID),
    (dict(sink=NULL), kvd.KVD_ERR_INVALID),
    (dict(src=ctypes.c_void_p(256 + 8)), kvd.KVD_ERR_INVALID),
    (dict(nbytes=0, src=NULL), kvd.KVD_OK),
])
def test_read_stream_validation(kw, status):
    a = dict(src=DUMMY, nbytes=4096, mode=kvd.KVD_READ_BULK, sink=DUMMY, stream=NULL)
    a.update(kw)
    assert L.kvd_read_stream(a["src"], a["nbytes"], a["mode"], a["sink"], a["stream"]) == status


def test_wait_limit_hook_accepts_any_value():
    for v in (0, 5, -1, 1 << 40, -7):
        assert L.kvd_set_decode_wait_limit(v) == kvd.KVD_OK


def test_workspace_size_with_explicit_partitions():
    # layout: (B+1) int32 -> 256-byte rounded; slots*G floats -> rounded; slots*G*d floats
    B, H_q, H_kv, d, N = 3, 8, 2, 128, 10
    slots = N + B * H_kv
    G = H_q // H_kv
    expect = 256 + ((slots * G * 4 + 255) // 256) * 256 + slots * G * d * 4
    assert kvd.kvd_workspace_size(B, H_q, H_kv, d, N) == expect


def test_package_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "kvd_copy", os.path.join(ROOT, "kv_cache_decode_scatters_b200", "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    monkeypatch.setattr(os.path, "exists", lambda p: False if p.endswith("libkvdecode.so") else True)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)

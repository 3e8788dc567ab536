"""GPU parity of the 8-bit KV caches (FP8 E4M3 and INT8 codes) against the oracle.

Quantisation and append must be bit-exact (codes and scales); attention over
the 8-bit cache must be within the dtype tolerance of the oracle's attention
over the same dequantised values.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import LSE_TOL, TOL, assert_pools_equal, data_rows, host, odt, oracle_q8, oracle_q8_rows
from synth import build_workload, named_config, step_inputs, to_words

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    return m


FORMATS = ["fp8", "int8"]


@pytest.fixture(params=FORMATS)
def fmt(request):
    return request.param


def gpu_fn(kvd, what, fmt):
    return getattr(kvd, f"kvd_{what}_{fmt}")


def orc_fn(what, fmt):
    return getattr(oracle, f"{what}_{fmt}")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("d", [128, 64])
def test_quantize_bit_exact(kvd, fmt, dtype, d):
    g = torch.Generator().manual_seed(5)
    x = torch.randn(1000, d, generator=g)
    x[3, 17] = 40.0            # outlier channel
    x[5, 32:64] = 0.0          # all-zero group
    x[7] *= 1e-3               # small row
    x[9, 40] = float("nan")    # a NaN element
    x[11, 0:32] = 2.5          # a group with max 127: INT8 scale 1.0, quotients on exact ties
    x[11, 0], x[11, 1], x[11, 2], x[11, 3] = 127.0, 3.5, -2.5, 0.5
    x[13, 5] = -2.0 ** -20     # a value far below its group's step
    x = x.to(dtype)
    codes, scales = gpu_fn(kvd, "quantize", fmt)(x.cuda())
    torch.cuda.synchronize()
    oc, os_ = orc_fn("quantize", fmt)(to_words(x), oracle.BF16 if dtype == torch.bfloat16 else oracle.F16)
    assert np.array_equal(host(codes), oc)
    assert np.array_equal(host(scales).view(np.uint32), os_.view(np.uint32))


def q8_state(kvd, w, fmt):
    """Quantise the workload's 16-bit pools on the GPU."""
    k8, ks = gpu_fn(kvd, "quantize", fmt)(w.k_cache.cuda())
    v8, vs = gpu_fn(kvd, "quantize", fmt)(w.v_cache.cuda())
    torch.cuda.synchronize()
    return k8, v8, ks, vs


def test_append_bit_exact_whole_pool(kvd, fmt):
    w = build_workload("a8", 5, 8, 4, 128, "bf16", [1, 16, 17, 40, 0], seed=1201, spare_pages=3)
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    bt = w.block_table.cuda()
    gpu_fn(kvd, "append", fmt)(k8, v8, ks, vs, bt, si["slot"].cuda(), si["k_new"].cuda(),
                               si["v_new"].cuda())
    torch.cuda.synchronize()
    hk8, hv8, hks, hvs = oracle_q8(w, fmt, si)
    assert_pools_equal((k8, v8, ks, vs), (hk8, hv8, hks, hvs),
                       data_rows(w.k_cache, w.v_cache, w.block_table, si))
    assert kvd.kvd_read_device_error() == 0


CASES = [
    # B, H_q, H_kv, dtype, lens, partitions
    (4, 32, 32, "f16", [1, 15, 16, 300], 0),
    (3, 64, 8, "bf16", [513, 77, 1000], 0),
    (2, 16, 1, "bf16", [40, 130], 0),          # MQA, group 16
    (5, 32, 8, "f16", [3, 0, 45, 0, 200], 7),  # empty sequences, fixed partitions
    (2, 24, 8, "bf16", [700, 31], 1),          # group 3, one partition
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_{c[3]}_N{c[5]}")
def test_decode_matches_oracle(kvd, fmt, case):
    B, H_q, H_kv, dtype, lens, parts = case
    w = build_workload("d8", B, H_q, H_kv, 128, dtype, lens, seed=1300 + CASES.index(case),
                       spare_pages=2)
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    bt = w.block_table.cuda()
    gpu_fn(kvd, "append", fmt)(k8, v8, ks, vs, bt, si["slot"].cuda(), si["k_new"].cuda(),
                               si["v_new"].cuda())
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    out = gpu_fn(kvd, "decode_attention", fmt)(si["q"].cuda(), k8, v8, ks, vs, bt, si["seq_lens"].cuda(),
                                               w.scale, num_partitions=parts, lse_out=lse)
    torch.cuda.synchronize()
    hk8, hv8, hks, hvs = oracle_q8(w, fmt, si)
    assert_pools_equal((k8, v8, ks, vs), (hk8, hv8, hks, hvs),
                       data_rows(w.k_cache, w.v_cache, w.block_table, si))
    ref, ref_lse = orc_fn("attend", fmt)(to_words(si["q"]), hk8, hv8, hks, hvs,
                                         w.block_table.numpy(), si["seq_lens"].numpy(), w.scale, odt(w))
    g = out.float().cpu().double().numpy()
    err = float(np.max(np.abs(g - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"
    fin = np.isfinite(ref_lse)
    gl = lse.cpu().double().numpy()
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) <= LSE_TOL
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(out[b] == 0)
    # against the 16-bit cache, the error is the quantisation's: every value
    # is within half an E4M3 ulp (2^-4 relative) and out is a weighted mean of
    # values, so |out_fp8 - out_16| <= 2^-4 max|v| plus what the changed
    # scores move (checked loosely)
    kc, vc = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    oracle.append(kc, vc, w.block_table.numpy(), si["slot"].numpy(), to_words(si["k_new"]),
                  to_words(si["v_new"]))
    full, _ = oracle.attend(to_words(si["q"]), kc, vc, w.block_table.numpy(), si["seq_lens"].numpy(),
                            w.scale, odt(w))
    vmax = float(np.nanmax(np.abs(si["v_new"].float().numpy())))
    assert np.max(np.abs(g - full)) <= 2 * 2 ** -4 * max(vmax, 4.0)
    assert kvd.kvd_read_device_error() == 0


def test_decode_full_size_gqa70b(kvd, fmt):
    w = named_config("gqa70b", device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    bt = w.block_table.cuda()
    gpu_fn(kvd, "append", fmt)(k8, v8, ks, vs, bt, si["slot"], si["k_new"], si["v_new"])
    out = gpu_fn(kvd, "decode_attention", fmt)(si["q"], k8, v8, ks, vs, bt, si["seq_lens"], w.scale)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    lens = w.seq_lens0.numpy()
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 5, 40})
    (hk8, hv8, hks, hvs), bts, pages = oracle_q8_rows(w, fmt, si, rows)
    idx = torch.tensor(pages, dtype=torch.long, device="cuda")
    sel = torch.tensor(rows, dtype=torch.long)
    rows_ok = data_rows(w.k_cache.index_select(0, idx), w.v_cache.index_select(0, idx), bts,
                        {"slot": si["slot"].cpu()[sel]})
    assert_pools_equal([t.index_select(0, idx) for t in (k8, v8, ks, vs)], (hk8, hv8, hks, hvs), rows_ok)
    sel = torch.tensor(rows, dtype=torch.long)
    ref, _ = orc_fn("attend", fmt)(to_words(si["q"].cpu()[sel]), hk8, hv8, hks, hvs, bts,
                                   si["seq_lens"].cpu()[sel].numpy(), w.scale, oracle.BF16)
    worst = float(np.max(np.abs(out.cpu()[sel].float().double().numpy() - ref)))
    print(f"gqa70b {fmt}: max abs error {worst:.3e} over sequences {rows}")
    assert worst <= TOL[w.dtype]
    assert kvd.kvd_read_device_error() == 0


def _bits(t):
    """A tensor's raw bits (int16 view for 16-bit floats, int32 for fp32), on the host."""
    t = t.detach().cpu()
    return t.view(torch.int16) if t.element_size() == 2 else (t.view(torch.int32) if t.element_size() == 4 else t)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_{c[3]}_N{c[5]}")
def test_fused_step_matches_oracle_and_two_calls(kvd, fmt, case):
    # kvd_decode_step_<fmt>: the pools after the call are the oracle's append
    # (slot = seq_lens - 1) bit for bit, out is within tolerance of the
    # oracle's attention over them, and both are bit-identical to the
    # two-call path (append, then attention with the same partitions)
    B, H_q, H_kv, dtype, lens, parts = case
    w = build_workload("s8", B, H_q, H_kv, 128, dtype, lens, seed=1400 + CASES.index(case),
                       spare_pages=2)
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    two = [t.clone() for t in (k8, v8, ks, vs)]
    bt = w.block_table.cuda()
    q, kn, vn, sl = si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), si["seq_lens"].cuda()
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    out = gpu_fn(kvd, "decode_step", fmt)(q, kn, vn, k8, v8, ks, vs, bt, sl, w.scale,
                                          num_partitions=parts, lse_out=lse)
    gpu_fn(kvd, "append", fmt)(*two, bt, si["slot"].cuda(), kn, vn)
    lse2 = torch.empty_like(lse)
    out2 = gpu_fn(kvd, "decode_attention", fmt)(q, *two, bt, sl, w.scale, num_partitions=parts,
                                                lse_out=lse2)
    torch.cuda.synchronize()
    hk8, hv8, hks, hvs = oracle_q8(w, fmt, si)
    assert_pools_equal((k8, v8, ks, vs), (hk8, hv8, hks, hvs),
                       data_rows(w.k_cache, w.v_cache, w.block_table, si))
    ref, ref_lse = orc_fn("attend", fmt)(to_words(si["q"]), hk8, hv8, hks, hvs, w.block_table.numpy(),
                                         si["seq_lens"].numpy(), w.scale, odt(w))
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"
    fin = np.isfinite(ref_lse)
    gl = lse.cpu().double().numpy()
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) <= LSE_TOL
    for a, b in zip((k8, v8, ks, vs), two):
        assert torch.equal(_bits(a), _bits(b))
    assert torch.equal(_bits(out), _bits(out2)) and torch.equal(_bits(lse), _bits(lse2))
    assert kvd.kvd_read_device_error() == 0


def test_fused_step_full_size_gqa70b(kvd, fmt):
    # the benchmark's 70B-shape GQA step over the 8-bit cache: pools and out
    # bit-identical to the two-call path, sampled sequences against the oracle
    w = named_config("gqa70b", device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    two = [t.clone() for t in (k8, v8, ks, vs)]
    bt = w.block_table.cuda()
    out = gpu_fn(kvd, "decode_step", fmt)(si["q"], si["k_new"], si["v_new"], k8, v8, ks, vs, bt,
                                          si["seq_lens"], w.scale)
    gpu_fn(kvd, "append", fmt)(*two, bt, si["slot"], si["k_new"], si["v_new"])
    out2 = gpu_fn(kvd, "decode_attention", fmt)(si["q"], *two, bt, si["seq_lens"], w.scale)
    torch.cuda.synchronize()
    for a, b in zip((k8, v8, ks, vs), two):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    del two
    lens = w.seq_lens0.numpy()
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 7, 33})
    (hk8, hv8, hks, hvs), bts, pages = oracle_q8_rows(w, fmt, si, rows)
    idx = torch.tensor(pages, dtype=torch.long, device="cuda")
    sel = torch.tensor(rows, dtype=torch.long)
    rows_ok = data_rows(w.k_cache.index_select(0, idx), w.v_cache.index_select(0, idx), bts,
                        {"slot": si["slot"].cpu()[sel]})
    assert_pools_equal([t.index_select(0, idx) for t in (k8, v8, ks, vs)], (hk8, hv8, hks, hvs), rows_ok)
    sel = torch.tensor(rows, dtype=torch.long)
    ref, _ = orc_fn("attend", fmt)(to_words(si["q"].cpu()[sel]), hk8, hv8, hks, hvs, bts,
                                   si["seq_lens"].cpu()[sel].numpy(), w.scale, oracle.BF16)
    worst = float(np.max(np.abs(out.cpu()[sel].float().double().numpy() - ref)))
    assert worst <= TOL[w.dtype], f"max abs error {worst}"
    assert kvd.kvd_read_device_error() == 0


def test_fused_step_rejects_missing_new_rows(kvd, fmt):
    w = build_workload("r8", 2, 8, 8, 128, "f16", [5, 9], seed=1499, spare_pages=1)
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    lib = kvd.lib()
    ws = kvd.alloc_workspace(2, 8, 8, 128, 0, torch.device("cuda"))
    out = torch.empty_like(si["q"]).cuda()
    st = getattr(lib, "kvd_decode_step_" + fmt)(
        si["q"].cuda().data_ptr(), None, None, k8.data_ptr(), v8.data_ptr(), ks.data_ptr(),
        vs.data_ptr(), w.block_table.cuda().data_ptr(), si["seq_lens"].cuda().data_ptr(), w.scale,
        out.data_ptr(), 2, 8, 8, 128, w.num_blocks, w.block_table.shape[1], 0, ws.data_ptr(),
        ws.numel(), None, kvd.KVD_F16, None)
    assert st == kvd.KVD_ERR_INVALID
    assert "k_new" in kvd.kvd_last_error()


def test_fused_step_maximum_batch(kvd, fmt):
    # B = KVD_MAX_BATCH ragged sequences: the per-sequence prefix sums push the
    # tuned two-stage layout past the CTA's shared memory, so the kernel runs
    # with one stage per warp; pools and out must still match the oracle
    B = 4096
    g = np.random.default_rng(4321)
    lens = g.integers(0, 81, size=B)
    lens[::101] = 0
    w = build_workload("max8", B, 8, 2, 128, "bf16", [int(x) for x in lens], seed=1501, spare_pages=4)
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    bt = w.block_table.cuda()
    out = gpu_fn(kvd, "decode_step", fmt)(si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), k8, v8,
                                          ks, vs, bt, si["seq_lens"].cuda(), w.scale)
    torch.cuda.synchronize()
    hk8, hv8, hks, hvs = oracle_q8(w, fmt, si)
    assert_pools_equal((k8, v8, ks, vs), (hk8, hv8, hks, hvs),
                       data_rows(w.k_cache, w.v_cache, w.block_table, si))
    ref, _ = orc_fn("attend", fmt)(to_words(si["q"]), hk8, hv8, hks, hvs, w.block_table.numpy(),
                                   si["seq_lens"].numpy(), w.scale, odt(w))
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"
    assert kvd.kvd_read_device_error() == 0


# ------------------------------------------------- 8-bit caches at d = 64

CASES64 = [
    # B, H_q, H_kv, dtype, lens, partitions
    (4, 16, 16, "f16", [1, 15, 16, 300], 0),     # MHA, page edges
    (3, 32, 8, "bf16", [513, 77, 1000], 0),      # group 4
    (2, 16, 1, "bf16", [40, 130], 0),            # MQA, group 16 (two n-tiles)
    (5, 16, 2, "f16", [3, 0, 45, 0, 200], 7),    # group 8, empty sequences, fixed partitions
    (2, 24, 8, "bf16", [700, 31], 1),            # group 3, one partition
]


@pytest.mark.parametrize("case", CASES64, ids=lambda c: f"d64_B{c[0]}_Hq{c[1]}_Hkv{c[2]}_{c[3]}_N{c[5]}")
def test_fused_step_d64_matches_oracle_and_two_calls(kvd, fmt, case):
    # the 8-bit cache with 64-channel heads (two scale groups per token, 64-byte
    # code rows): pools bit-exact against the oracle's quantising append, out
    # within tolerance of its attention over them, and both bit-identical to
    # the two-call path
    B, H_q, H_kv, dtype, lens, parts = case
    w = build_workload("s8d64", B, H_q, H_kv, 64, dtype, lens, seed=1600 + CASES64.index(case),
                       spare_pages=2)
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    assert ks.shape[-1] == 2
    two = [t.clone() for t in (k8, v8, ks, vs)]
    bt = w.block_table.cuda()
    q, kn, vn, sl = si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), si["seq_lens"].cuda()
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    out = gpu_fn(kvd, "decode_step", fmt)(q, kn, vn, k8, v8, ks, vs, bt, sl, w.scale,
                                          num_partitions=parts, lse_out=lse)
    gpu_fn(kvd, "append", fmt)(*two, bt, si["slot"].cuda(), kn, vn)
    out2 = gpu_fn(kvd, "decode_attention", fmt)(q, *two, bt, sl, w.scale, num_partitions=parts)
    torch.cuda.synchronize()
    hk8, hv8, hks, hvs = oracle_q8(w, fmt, si)
    assert_pools_equal((k8, v8, ks, vs), (hk8, hv8, hks, hvs),
                       data_rows(w.k_cache, w.v_cache, w.block_table, si))
    ref, ref_lse = orc_fn("attend", fmt)(to_words(si["q"]), hk8, hv8, hks, hvs, w.block_table.numpy(),
                                         si["seq_lens"].numpy(), w.scale, odt(w))
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"
    fin = np.isfinite(ref_lse)
    gl = lse.cpu().double().numpy()
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) <= LSE_TOL
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(out[b] == 0)
    for a, b in zip((k8, v8, ks, vs), two):
        assert torch.equal(_bits(a), _bits(b))
    assert torch.equal(_bits(out), _bits(out2))
    assert kvd.kvd_read_device_error() == 0


def test_decode_d64_larger_batch_every_row(kvd, fmt):
    # 16 sequences of 64-channel heads, 32 query / 8 KV heads, lengths over
    # many pages and ragged tails: every row against the oracle
    lens = [2000 - 97 * i for i in range(16)]
    w = build_workload("b8d64", 16, 32, 8, 64, "bf16", lens, seed=1650, spare_pages=3)
    si = step_inputs(w, 0)
    k8, v8, ks, vs = q8_state(kvd, w, fmt)
    bt = w.block_table.cuda()
    out = gpu_fn(kvd, "decode_step", fmt)(si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), k8, v8,
                                          ks, vs, bt, si["seq_lens"].cuda(), w.scale)
    torch.cuda.synchronize()
    hk8, hv8, hks, hvs = oracle_q8(w, fmt, si)
    ref, _ = orc_fn("attend", fmt)(to_words(si["q"]), hk8, hv8, hks, hvs, w.block_table.numpy(),
                                   si["seq_lens"].numpy(), w.scale, odt(w))
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"
    assert kvd.kvd_read_device_error() == 0


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
def test_fused_step_full_size_mha7b_one_query_row(kvd, fmt):
    # the benchmark's 7B-shape MHA step (one query row per KV head, the
    # quantised tile with the scale groups in its N columns) over each
    # quantised cache: pools and out bit-identical to the two-call path,
    # sampled sequences against the oracle
    w = named_config("mha7b", device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    quant = getattr(kvd, "kvd_quantize_" + fmt)
    k8, ks = quant(w.k_cache)
    v8, vs = quant(w.v_cache)
    pools = [k8, v8, ks, vs]
    two = [t.clone() for t in pools]
    bt = w.block_table.cuda()
    out = getattr(kvd, "kvd_decode_step_" + fmt)(si["q"], si["k_new"], si["v_new"], *pools, bt,
                                                  si["seq_lens"], w.scale)
    getattr(kvd, "kvd_append_" + fmt)(*two, bt, si["slot"], si["k_new"], si["v_new"])
    out2 = getattr(kvd, "kvd_decode_attention_" + fmt)(si["q"], *two, bt, si["seq_lens"], w.scale)
    torch.cuda.synchronize()
    for a, b in zip(pools, two):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    del two
    rows = [0, 13, 31]
    (hk, hv, hks, hvs), bts, pages = oracle_q8_rows(w, fmt, si, rows)
    idx = torch.tensor(pages, dtype=torch.long, device="cuda")
    sel = torch.tensor(rows, dtype=torch.long)
    rows_ok = data_rows(w.k_cache.index_select(0, idx), w.v_cache.index_select(0, idx), bts,
                        {"slot": si["slot"].cpu()[sel]})
    assert_pools_equal([t.index_select(0, idx) for t in pools], (hk, hv, hks, hvs), rows_ok)
    ref, _ = getattr(oracle, "attend_" + fmt)(to_words(si["q"].cpu()[sel]), hk, hv, hks, hvs, bts,
                                              si["seq_lens"].cpu()[sel].numpy(), w.scale, odt(w))
    err = float(np.max(np.abs(out.cpu()[sel].float().double().numpy() - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"
    assert kvd.kvd_read_device_error() == 0

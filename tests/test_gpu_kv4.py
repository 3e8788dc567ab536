"""GPU parity of the INT4 KV cache (two codes per byte) against the oracle.

Quantisation and append must be bit-exact (codes and scales), the pools
compared on every slot that holds data; attention over the INT4 cache must be
within the dtype tolerance of the oracle's attention over the same decoded
values, with the oracle's pools from its own quantisation.  The fused step
must give the bits of the two-call path.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (LSE_TOL, assert_out_close, assert_pools_equal, data_rows, host, odt, oracle_q8,
                         oracle_q8_rows)
from synth import build_workload, named_config, step_inputs, to_words

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    return m


def q4_state(kvd, w):
    """Quantise the workload's 16-bit pools on the GPU."""
    k4, ks = kvd.kvd_quantize_int4(w.k_cache.cuda())
    v4, vs = kvd.kvd_quantize_int4(w.v_cache.cuda())
    torch.cuda.synchronize()
    return k4, v4, ks, vs


def _bits(t):
    t = t.detach().cpu()
    return t.view(torch.int16) if t.element_size() == 2 else (t.view(torch.int32) if t.element_size() == 4 else t)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("d", [128, 64])
def test_quantize_bit_exact(kvd, dtype, d):
    g = torch.Generator().manual_seed(45)
    x = torch.randn(1000, d, generator=g)
    x[3, 17] = 40.0            # outlier channel
    x[5, 32:64] = 0.0          # all-zero group
    x[7] *= 1e-3               # small row
    x[9, 40] = float("nan")    # a NaN element
    x[11, 0:32] = 3.5          # a group with max 7 (scale 0.5): quotients on exact ties
    x[11, 0], x[11, 1], x[11, 2], x[11, 3] = 3.5, 1.25, -0.75, 0.25
    x[13, 5] = -2.0 ** -20     # far below its group's step
    x = x.to(dtype)
    codes, scales = kvd.kvd_quantize_int4(x.cuda())
    torch.cuda.synchronize()
    assert codes.shape == (1000, d // 2)
    oc, os_ = oracle.quantize_int4(to_words(x), oracle.BF16 if dtype == torch.bfloat16 else oracle.F16)
    assert np.array_equal(host(codes), oc)
    assert np.array_equal(host(scales).view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("d", [128, 64])
def test_append_bit_exact_whole_pool(kvd, d):
    w = build_workload("a4", 5, 8, 4, d, "bf16", [1, 16, 17, 40, 0], seed=1701, spare_pages=3)
    si = step_inputs(w, 0)
    k4, v4, ks, vs = q4_state(kvd, w)
    bt = w.block_table.cuda()
    kvd.kvd_append_int4(k4, v4, ks, vs, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    torch.cuda.synchronize()
    assert_pools_equal((k4, v4, ks, vs), oracle_q8(w, "int4", si),
                       data_rows(w.k_cache, w.v_cache, w.block_table, si))
    assert kvd.kvd_read_device_error() == 0


CASES = [
    # B, H_q, H_kv, d, dtype, lens, partitions
    (4, 32, 32, 128, "f16", [1, 15, 16, 300], 0),   # MHA, page edges
    (3, 64, 8, 128, "bf16", [513, 77, 1000], 0),    # group 8
    (2, 16, 1, 128, "bf16", [40, 130], 0),          # MQA, group 16 (two n-tiles)
    (5, 32, 8, 128, "f16", [3, 0, 45, 0, 200], 7),  # group 4, empty sequences, fixed partitions
    (2, 24, 8, 128, "bf16", [700, 31], 1),          # group 3, one partition
    (4, 16, 16, 64, "f16", [1, 15, 16, 300], 0),    # d = 64
    (3, 32, 8, 64, "bf16", [513, 77, 1000], 0),
    (2, 16, 1, 64, "f16", [40, 130], 3),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_d{c[3]}_{c[4]}_N{c[6]}")
def test_fused_step_matches_oracle_and_two_calls(kvd, case):
    # kvd_decode_step_int4: the pools after the call are the oracle's append
    # bit for bit, out is within tolerance of the oracle's attention over
    # them, and both are bit-identical to kvd_append_int4 followed by
    # kvd_decode_attention_int4 with the same partitions
    B, H_q, H_kv, d, dtype, lens, parts = case
    w = build_workload("s4", B, H_q, H_kv, d, dtype, lens, seed=1710 + CASES.index(case), spare_pages=2)
    si = step_inputs(w, 0)
    k4, v4, ks, vs = q4_state(kvd, w)
    two = [t.clone() for t in (k4, v4, ks, vs)]
    bt = w.block_table.cuda()
    q, kn, vn, sl = si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), si["seq_lens"].cuda()
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    out = kvd.kvd_decode_step_int4(q, kn, vn, k4, v4, ks, vs, bt, sl, w.scale, num_partitions=parts,
                                   lse_out=lse)
    kvd.kvd_append_int4(*two, bt, si["slot"].cuda(), kn, vn)
    lse2 = torch.empty_like(lse)
    out2 = kvd.kvd_decode_attention_int4(q, *two, bt, sl, w.scale, num_partitions=parts, lse_out=lse2)
    torch.cuda.synchronize()
    hk, hv, hks, hvs = oracle_q8(w, "int4", si)
    assert_pools_equal((k4, v4, ks, vs), (hk, hv, hks, hvs), data_rows(w.k_cache, w.v_cache, w.block_table, si))
    ref, ref_lse = oracle.attend_int4(to_words(si["q"]), hk, hv, hks, hvs, w.block_table.numpy(),
                                      si["seq_lens"].numpy(), w.scale, odt(w))
    g = out.float().cpu().double().numpy()
    assert_out_close(g, ref, w.dtype)
    fin = np.isfinite(ref_lse)
    gl = lse.cpu().double().numpy()
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) <= LSE_TOL
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(out[b] == 0)
    for a, b in zip((k4, v4, ks, vs), two):
        assert torch.equal(_bits(a), _bits(b))
    assert torch.equal(_bits(out), _bits(out2)) and torch.equal(_bits(lse), _bits(lse2))
    # against the 16-bit cache the error is the quantisation's: every value is
    # within half a step (max|x| / 14 of its group), so the output moves by at
    # most a few steps of V plus what the changed scores move (checked loosely)
    kc, vc = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    oracle.append(kc, vc, w.block_table.numpy(), si["slot"].numpy(), to_words(si["k_new"]),
                  to_words(si["v_new"]))
    full, _ = oracle.attend(to_words(si["q"]), kc, vc, w.block_table.numpy(), si["seq_lens"].numpy(),
                            w.scale, odt(w))
    assert np.max(np.abs(g - full)) < 1.0
    assert kvd.kvd_read_device_error() == 0


def test_fused_step_full_size_gqa70b(kvd):
    # the benchmark's 70B-shape GQA step over the INT4 cache: pools and out
    # bit-identical to the two-call path, sampled sequences against the oracle
    w = named_config("gqa70b", device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    k4, v4, ks, vs = q4_state(kvd, w)
    two = [t.clone() for t in (k4, v4, ks, vs)]
    bt = w.block_table.cuda()
    out = kvd.kvd_decode_step_int4(si["q"], si["k_new"], si["v_new"], k4, v4, ks, vs, bt,
                                   si["seq_lens"], w.scale)
    kvd.kvd_append_int4(*two, bt, si["slot"], si["k_new"], si["v_new"])
    out2 = kvd.kvd_decode_attention_int4(si["q"], *two, bt, si["seq_lens"], w.scale)
    torch.cuda.synchronize()
    for a, b in zip((k4, v4, ks, vs), two):
        assert torch.equal(_bits(a), _bits(b))
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    del two
    lens = w.seq_lens0.numpy()
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 7, 33})
    (hk, hv, hks, hvs), bts, pages = oracle_q8_rows(w, "int4", si, rows)
    idx = torch.tensor(pages, dtype=torch.long, device="cuda")
    sel = torch.tensor(rows, dtype=torch.long)
    rows_ok = data_rows(w.k_cache.index_select(0, idx), w.v_cache.index_select(0, idx), bts,
                        {"slot": si["slot"].cpu()[sel]})
    assert_pools_equal([t.index_select(0, idx) for t in (k4, v4, ks, vs)], (hk, hv, hks, hvs), rows_ok)
    ref, _ = oracle.attend_int4(to_words(si["q"].cpu()[sel]), hk, hv, hks, hvs, bts,
                                si["seq_lens"].cpu()[sel].numpy(), w.scale, oracle.BF16)
    assert_out_close(out.cpu()[sel], ref, w.dtype)
    assert kvd.kvd_read_device_error() == 0


def test_maximum_batch(kvd):
    # B = KVD_MAX_BATCH ragged sequences through the fused INT4 step
    B = 4096
    g = np.random.default_rng(4322)
    lens = g.integers(0, 81, size=B)
    lens[::101] = 0
    w = build_workload("max4", B, 8, 2, 128, "bf16", [int(x) for x in lens], seed=1751, spare_pages=4)
    si = step_inputs(w, 0)
    k4, v4, ks, vs = q4_state(kvd, w)
    out = kvd.kvd_decode_step_int4(si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), k4, v4, ks, vs,
                                   w.block_table.cuda(), si["seq_lens"].cuda(), w.scale)
    torch.cuda.synchronize()
    hk, hv, hks, hvs = oracle_q8(w, "int4", si)
    assert_pools_equal((k4, v4, ks, vs), (hk, hv, hks, hvs), data_rows(w.k_cache, w.v_cache, w.block_table, si))
    ref, _ = oracle.attend_int4(to_words(si["q"]), hk, hv, hks, hvs, w.block_table.numpy(),
                                si["seq_lens"].numpy(), w.scale, odt(w))
    # short sequences put some outputs at |out| > 4, where a bf16 value
    # cannot be within 1e-2 of the exact result (the check allows one ulp there)
    assert_out_close(out, ref, w.dtype)
    assert kvd.kvd_read_device_error() == 0

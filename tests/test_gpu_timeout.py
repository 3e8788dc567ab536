"""The decode kernel's bounded-wait failure path, made to run out on purpose.

kvd_set_decode_wait_limit(0) makes each worker warp's first page wait give up
at once: the warp sets KVD_DEVERR_TIMEOUT, drains the copies it has in flight
(with the full poll limit, so every copy lands) and leaves the launch.  No copy
is withheld and nothing waits forever; the test checks that the flag is set,
that the call itself still returns KVD_OK, and that the next call with the
default limit is correct against the oracle on the same context.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import LSE_TOL, TOL, gpu_state, max_err, max_lse_err, oracle_step
from synth import build_workload, step_inputs, to_words

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    yield m
    m.kvd_set_decode_wait_limit(-1)


def decode(kvd, w, si, kc, vc, bt, parts):
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
    out = kvd.kvd_decode_attention(si["q"].cuda(), kc, vc, bt, si["seq_lens"].cuda(), w.scale,
                                   num_partitions=parts, lse_out=lse)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("parts", [0, 3])
def test_wait_timeout_flags_and_next_call_is_correct(kvd, parts):
    w = build_workload("timeout", 3, 32, 8, 128, "bf16", [700, 33, 1500], seed=950, spare_pages=2)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    assert kvd.kvd_read_device_error(clear=True) == 0

    kvd.kvd_set_decode_wait_limit(0)
    try:
        decode(kvd, w, si, kc, vc, bt, parts)     # returns KVD_OK: the failure is on the device
    finally:
        kvd.kvd_set_decode_wait_limit(-1)
    flags = kvd.kvd_read_device_error(clear=True)
    assert flags & kvd.KVD_DEVERR_TIMEOUT, f"flags {flags:#x}"

    # the context is still usable and the default limit gives the right answer
    out, lse = decode(kvd, w, si, kc, vc, bt, parts)
    _, _, ref = oracle_step(w, si)
    assert max_err(out, ref) <= TOL[w.dtype]
    assert max_lse_err(lse, ref) <= LSE_TOL
    assert kvd.kvd_read_device_error() == 0


@pytest.mark.parametrize("fmt", ["fp8", "int8"])
def test_wait_timeout_in_the_8bit_decode(kvd, fmt):
    w = build_workload("timeout8", 2, 16, 4, 128, "f16", [300, 47], seed=951, spare_pages=2)
    si = step_inputs(w, 0)
    quant = getattr(kvd, "kvd_quantize_" + fmt)
    k8, ks = quant(w.k_cache.cuda())
    v8, vs = quant(w.v_cache.cuda())
    bt = w.block_table.cuda()
    step = getattr(kvd, "kvd_decode_step_" + fmt)
    args = (si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    kvd.kvd_set_decode_wait_limit(0)
    try:
        step(*args, k8.clone(), v8.clone(), ks.clone(), vs.clone(), bt, si["seq_lens"].cuda(), w.scale)
        torch.cuda.synchronize()
    finally:
        kvd.kvd_set_decode_wait_limit(-1)
    assert kvd.kvd_read_device_error(clear=True) & kvd.KVD_DEVERR_TIMEOUT
    # the same step with the default limit: against the oracle over the
    # dequantised cache, after the oracle's own quantising append
    k8b, v8b, ksb, vsb = k8.clone(), v8.clone(), ks.clone(), vs.clone()
    out = step(*args, k8b, v8b, ksb, vsb, bt, si["seq_lens"].cuda(), w.scale)
    torch.cuda.synchronize()
    host = lambda t: (lambda a: a.view(np.uint8) if a.dtype == np.int8 else a)(t.cpu().numpy().copy())
    # the oracle's own pools: its quantisation of the 16-bit pool, then its
    # quantising append of the step
    hk, hks = getattr(oracle, "quantize_" + fmt)(to_words(w.k_cache), oracle.F16)
    hv, hvs = getattr(oracle, "quantize_" + fmt)(to_words(w.v_cache), oracle.F16)
    getattr(oracle, "append_" + fmt)(hk, hv, hks, hvs, w.block_table.numpy(), si["slot"].numpy(),
                                     to_words(si["k_new"]), to_words(si["v_new"]), oracle.F16)
    # codes and scales bit for bit on the slots holding data (the encoding of
    # the NaN canary in never-written slots is a convention nothing reads)
    rows = (torch.isfinite(w.k_cache.float()).all(-1) & torch.isfinite(w.v_cache.float()).all(-1)).numpy()
    btn = w.block_table.numpy()
    for b, pos in enumerate(si["slot"].numpy()):
        if pos >= 0:
            rows[btn[b, pos // 16], :, pos % 16] = True
    assert np.array_equal(host(k8b)[rows], hk[rows]) and np.array_equal(host(v8b)[rows], hv[rows])
    assert np.array_equal(host(ksb).view(np.uint32)[rows], hks.view(np.uint32)[rows])
    ref, _ = getattr(oracle, "attend_" + fmt)(to_words(si["q"]), hk, hv, hks, hvs, w.block_table.numpy(),
                                              si["seq_lens"].numpy(), w.scale, oracle.F16)
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype]
    assert kvd.kvd_read_device_error() == 0

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
from gpu_helpers import (LSE_TOL, TOL, assert_pools_equal, data_rows, gpu_state, max_err, max_lse_err,
                         oracle_q8, oracle_step)
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


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
def test_wait_timeout_in_the_quantised_decode(kvd, fmt):
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
    # the same step with the default limit: pools bit for bit on the slots
    # holding data, out against the oracle's attention over its own pools
    pools = [t.clone() for t in (k8, v8, ks, vs)]
    out = step(*args, *pools, bt, si["seq_lens"].cuda(), w.scale)
    torch.cuda.synchronize()
    hk, hv, hks, hvs = oracle_q8(w, fmt, si)
    assert_pools_equal(pools, (hk, hv, hks, hvs), data_rows(w.k_cache, w.v_cache, w.block_table, si))
    ref, _ = getattr(oracle, "attend_" + fmt)(to_words(si["q"]), hk, hv, hks, hvs, w.block_table.numpy(),
                                              si["seq_lens"].numpy(), w.scale, oracle.F16)
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype]
    assert kvd.kvd_read_device_error() == 0

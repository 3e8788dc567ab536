"""GPU parity at the benchmark's full sizes, through the call the benchmark
times (kvd_decode_step, or the shared-prefix call with its fused append) in
the benchmark's launch configuration (automatic partitions).

Every output row of every workload is checked against the fp64 oracle
(max-abs 2e-3 for fp16, 1e-2 for bf16; lse within 1e-3), and the whole pool
against the oracle's append, bit for bit.  Continuous batching runs its 16
consecutive steps and checks every row at steps 0, 7 and 15.  Each test
records its workload's maximum error; the session prints them as a table.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle

from gpu_helpers import LSE_TOL, TOL, gpu_state, max_err, max_lse_err, oracle_step, record_error
from synth import named_config, step_inputs, to_words

pytestmark = pytest.mark.gpu

CHECK_STEPS = (0, 7, 15)


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    return m


def fused_step(kvd, w, si, kc, vc, bt):
    """The benchmark's step: append fused into the decode launch."""
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
    out = kvd.kvd_decode_step(si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), kc, vc, bt,
                              si["seq_lens"].cuda(), w.scale, lse_out=lse)
    torch.cuda.synchronize()
    return out, lse


def host_copy(w):
    return replace(w, k_cache=w.k_cache.cpu(), v_cache=w.v_cache.cpu())


@pytest.mark.parametrize("name", ["tiny", "mha7b", "gqa70b", "long"])
def test_full_size_step_every_row(kvd, name):
    w = named_config(name, device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    out, lse = fused_step(kvd, w, si, kc, vc, bt)
    assert torch.isfinite(out.float()).all(), "non-finite output row"
    wc = host_copy(w)
    sic = {n: t.cpu() for n, t in si.items()}
    okc, ovc, ref = oracle_step(wc, sic)             # every (sequence, query head) row
    assert len(ref) == w.B
    assert np.array_equal(to_words(kc), okc), "append not bit-exact over the pool"
    assert np.array_equal(to_words(vc), ovc), "append not bit-exact over the pool"
    err = max_err(out, ref)
    lse_err = max_lse_err(lse, ref)
    record_error(name, "kvd_decode_step", w.B * w.H_q, err, lse_err, TOL[w.dtype])
    assert err <= TOL[w.dtype], f"{name}: max abs error {err}"
    assert lse_err <= LSE_TOL
    assert kvd.kvd_read_device_error() == 0


def run_cbatch(kvd, shared_prefix):
    w = named_config("cbatch", device="cuda", gen_device="cuda")
    kc, vc, bt = gpu_state(w)
    host_k, host_v = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    wc = host_copy(w)
    per = w.B // w.groups
    gs = torch.arange(0, w.B + 1, per, dtype=torch.int32, device="cuda")
    gp = torch.full((w.groups,), w.prefix_tokens // 16, dtype=torch.int32, device="cuda")
    worst, worst_lse, rows = 0.0, 0.0, 0
    for step in range(w.steps):
        si = step_inputs(w, step)
        if shared_prefix:
            lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
            out = kvd.kvd_decode_attention_shared_prefix(si["q"], kc, vc, bt, si["seq_lens"], gs, gp,
                                                         per, w.scale, k_new=si["k_new"],
                                                         v_new=si["v_new"], lse_out=lse)
            torch.cuda.synchronize()
        else:
            out, lse = fused_step(kvd, w, si, kc, vc, bt)
        assert torch.isfinite(out.float()).all()
        sic = {n: t.cpu() for n, t in si.items()}
        if step in CHECK_STEPS:
            host_k, host_v, ref = oracle_step(wc, sic, host_k, host_v)
            assert len(ref) == w.B
            worst = max(worst, max_err(out, ref))
            worst_lse = max(worst_lse, max_lse_err(lse, ref))
            rows += w.B * w.H_q
        else:
            oracle.append(host_k, host_v, wc.block_table.numpy(), sic["slot"].numpy(),
                          to_words(sic["k_new"]), to_words(sic["v_new"]))
    assert np.array_equal(to_words(kc), host_k) and np.array_equal(to_words(vc), host_v)
    return w, worst, worst_lse, rows


def test_full_size_continuous_batching_16_steps(kvd):
    w, err, lse_err, rows = run_cbatch(kvd, shared_prefix=False)
    record_error("cbatch", "kvd_decode_step, steps 0/7/15", rows, err, lse_err, TOL[w.dtype])
    assert err <= TOL[w.dtype]
    assert lse_err <= LSE_TOL
    assert kvd.kvd_read_device_error() == 0


def test_full_size_continuous_batching_shared_prefix_16_steps(kvd):
    # the cascade path at full size, as the benchmark runs it: 8 groups of 32
    # members sharing a 4096-token prefix, fused append, 16 steps
    w, err, lse_err, rows = run_cbatch(kvd, shared_prefix=True)
    record_error("cbatch --shared-prefix", "kvd_decode_attention_shared_prefix, steps 0/7/15", rows,
                 err, lse_err, TOL[w.dtype])
    assert err <= TOL[w.dtype]
    assert lse_err <= LSE_TOL
    assert kvd.kvd_read_device_error() == 0

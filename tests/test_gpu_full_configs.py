"""GPU parity at the benchmark's full sizes, in the benchmark's launch
configuration (automatic partitions).

The five synthetic decode workloads are run whole on the GPU.  Append is
checked bit-exactly over the whole pool; attention outputs of sampled
sequences (all their query heads) are checked against the fp64 oracle, and
every output row must be finite.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle

from gpu_helpers import LSE_TOL, TOL, gpu_state, gpu_step, max_err, max_lse_err, oracle_step
from synth import named_config, step_inputs, to_words

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    return m


def sample_rows(w, k, seed):
    lens = w.seq_lens0.numpy()
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(w.B, size=min(k, w.B), replace=False).tolist())
    pick.add(int(np.argmax(lens)))
    pick.add(int(np.argmin(lens)))
    return sorted(pick)


@pytest.mark.parametrize("name,k", [("tiny", 1), ("mha7b", 4), ("gqa70b", 4), ("long", 1)])
def test_full_size_single_step(kvd, name, k):
    w = named_config(name, device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    out, lse = gpu_step(kvd, w, si, kc, vc, bt)
    assert torch.isfinite(out.float()).all(), "non-finite output row"
    rows = sample_rows(w, k, 11)
    wc = replace(w, k_cache=w.k_cache.cpu(), v_cache=w.v_cache.cpu())
    sic = {n: t.cpu() for n, t in si.items()}
    okc, ovc, ref = oracle_step(wc, sic, rows=rows)
    assert np.array_equal(to_words(kc), okc), "append not bit-exact over the pool"
    assert np.array_equal(to_words(vc), ovc), "append not bit-exact over the pool"
    err = max_err(out, ref)
    print(f"{name}: max abs error {err:.3e} over sequences {rows}")
    assert err <= TOL[w.dtype]
    assert max_lse_err(lse, ref) <= LSE_TOL
    assert kvd.kvd_read_device_error() == 0


def test_full_size_continuous_batching_16_steps(kvd):
    w = named_config("cbatch", device="cuda", gen_device="cuda")
    kc, vc, bt = gpu_state(w)
    host_k, host_v = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    wc = replace(w, k_cache=w.k_cache.cpu(), v_cache=w.v_cache.cpu())
    rows_by_step = {0: sample_rows(w, 3, 21), 7: sample_rows(w, 3, 22), 15: sample_rows(w, 3, 23)}
    worst = 0.0
    for step in range(w.steps):
        si = step_inputs(w, step)
        out, lse = gpu_step(kvd, w, si, kc, vc, bt)
        assert torch.isfinite(out.float()).all()
        sic = {n: t.cpu() for n, t in si.items()}
        rows = rows_by_step.get(step, [])
        if rows:
            host_k, host_v, ref = oracle_step(wc, sic, host_k, host_v, rows=rows)
            worst = max(worst, max_err(out, ref))
            assert max_lse_err(lse, ref) <= LSE_TOL
        else:
            oracle.append(host_k, host_v, wc.block_table.numpy(), sic["slot"].numpy(),
                          to_words(sic["k_new"]), to_words(sic["v_new"]))
    print(f"cbatch: max abs error {worst:.3e}")
    assert worst <= TOL[w.dtype]
    assert np.array_equal(to_words(kc), host_k) and np.array_equal(to_words(vc), host_v)
    assert kvd.kvd_read_device_error() == 0



def test_full_size_continuous_batching_shared_prefix_16_steps(kvd):
    # the cascade path at full size, as the benchmark runs it: 8 groups of 32
    # members sharing a 4096-token prefix, fused append, 16 steps
    w = named_config("cbatch", device="cuda", gen_device="cuda")
    kc, vc, bt = gpu_state(w)
    host_k, host_v = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    wc = replace(w, k_cache=w.k_cache.cpu(), v_cache=w.v_cache.cpu())
    per = w.B // w.groups
    gs = torch.arange(0, w.B + 1, per, dtype=torch.int32, device="cuda")
    gp = torch.full((w.groups,), w.prefix_tokens // 16, dtype=torch.int32, device="cuda")
    rows_by_step = {0: sample_rows(w, 3, 31), 9: sample_rows(w, 3, 32), 15: sample_rows(w, 3, 33)}
    worst = 0.0
    for step in range(w.steps):
        si = step_inputs(w, step)
        lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
        out = kvd.kvd_decode_attention_shared_prefix(si["q"], kc, vc, bt, si["seq_lens"], gs, gp, per,
                                                     w.scale, k_new=si["k_new"], v_new=si["v_new"],
                                                     lse_out=lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        sic = {n: t.cpu() for n, t in si.items()}
        rows = rows_by_step.get(step, [])
        if rows:
            host_k, host_v, ref = oracle_step(wc, sic, host_k, host_v, rows=rows)
            worst = max(worst, max_err(out, ref))
            assert max_lse_err(lse, ref) <= LSE_TOL
        else:
            oracle.append(host_k, host_v, wc.block_table.numpy(), sic["slot"].numpy(),
                          to_words(sic["k_new"]), to_words(sic["v_new"]))
    print(f"cbatch shared prefix: max abs error {worst:.3e}")
    assert worst <= TOL[w.dtype]
    assert np.array_equal(to_words(kc), host_k) and np.array_equal(to_words(vc), host_v)
    assert kvd.kvd_read_device_error() == 0

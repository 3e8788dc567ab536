"""kvd_decode_attention_static: the entry point for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

It must return exactly the bits kvd_decode_attention returns with a caller
workspace (same kernels, same automatic partitions), call after call on the
same shared array.  This file is named to run last,
so a run that stops at the first failure has run every other test before it.
"""
import pytest
import torch

from synth import build_workload, step_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    return m


CASES = [
    # B, H_q, H_kv, d, dtype, lens
    (4, 32, 8, 128, "bf16", [700, 33, 1200, 5]),
    (3, 16, 16, 64, "f16", [1, 400, 129]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_d{c[3]}_{c[4]}")
def test_static_entry_point_matches_workspace_entry_point(kvd, case):
    B, H_q, H_kv, d, dtype, lens = case
    w = build_workload("noalloc", B, H_q, H_kv, d, dtype, lens, seed=900 + CASES.index(case))
    kc, vc, bt = w.k_cache.cuda(), w.v_cache.cuda(), w.block_table.cuda()
    need = kvd.kvd_workspace_size(B, H_q, H_kv, d, 0)
    assert 0 < need <= kvd.KVD_STATIC_WORKSPACE_BYTES
    for step in range(2):                        # two calls in a row on the shared array
        si = step_inputs(w, step)
        q, sl = si["q"].cuda(), si["seq_lens"].cuda()
        kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
        ref_lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
        ref = kvd.kvd_decode_attention(q, kc, vc, bt, sl, w.scale, lse_out=ref_lse)
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, H_q), float("nan"), dtype=torch.float32, device="cuda")
        kvd.kvd_decode_attention_static(q, kc, vc, bt, sl, w.scale, out=out, lse_out=lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        # same kernels, same shape, same automatic partitions: the same bits
        err = torch.max(torch.abs(out.float() - ref.float())).item()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), \
            f"step {step}: differs from the workspace entry point (max abs {err})"
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32)), f"step {step}: lse differs"


def test_static_entry_point_rejects_oversized_shapes(kvd):
    # 4096 sequences x 8 KV heads x group 8 needs far more than the fixed array
    B, H_q, H_kv, d = 4096, 64, 8, 128
    need = kvd.kvd_workspace_size(B, H_q, H_kv, d, 0)
    assert need > kvd.KVD_STATIC_WORKSPACE_BYTES
    q = torch.zeros((B, H_q, d), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, H_kv, 16, d), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((B, 1), dtype=torch.int32, device="cuda")
    sl = torch.ones((B,), dtype=torch.int32, device="cuda")
    with pytest.raises(kvd.KvdError) as e:
        kvd.kvd_decode_attention_static(q, kc, kc, bt, sl, 0.1, out=torch.empty_like(q))
    assert e.value.status == kvd.KVD_ERR_UNSUPPORTED
    assert "fixed" in kvd.kvd_last_error()

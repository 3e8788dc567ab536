"""GPU parity of the shared-prefix decode over quantised caches (E4M3, INT8,
INT4; d = 128 on the tensor-memory prefix pass, d = 64 on the warp-level one)
against the oracle.

The oracle's pools are its own quantisation of the 16-bit pool plus its own
quantising append of the step; the GPU's pools after the fused append must
equal them bit for bit on every slot holding data, and the output must be
within the dtype tolerance of the oracle's attention over them.  The output
is also compared with the plain quantised decode (kvd_decode_step_{fmt}),
which reads every member's prefix pages itself: the two differ only in fp32
summation order and in the prefix pass's head-plus-remainder operands.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (LSE_TOL, TOL, assert_out_close, assert_pools_equal, data_rows, odt, oracle_q8,
                         oracle_q8_rows, uneven_groups_case)
from synth import build_workload, named_config, step_inputs, to_words

pytestmark = pytest.mark.gpu

FMTS = ["fp8", "int8", "int4"]


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    return m


def q_state(kvd, w, fmt):
    quant = getattr(kvd, "kvd_quantize_" + fmt)
    k8, ks = quant(w.k_cache.cuda())
    v8, vs = quant(w.v_cache.cuda())
    torch.cuda.synchronize()
    return [k8, v8, ks, vs]


def groups_of(w):
    per = w.B // w.groups
    start = torch.arange(0, w.B + 1, per, dtype=torch.int32)
    pages = torch.full((w.groups,), w.prefix_tokens // 16, dtype=torch.int32)
    return start.cuda(), pages.cuda(), per


def oracle_attend(w, si, pools, fmt, rows=None):
    hk, hv, hks, hvs = pools
    q = si["q"].cpu() if rows is None else si["q"].cpu()[torch.tensor(rows)]
    return getattr(oracle, "attend_" + fmt)(to_words(q), hk, hv, hks, hvs, w.block_table.numpy(),
                                            si["seq_lens"].cpu().numpy(), w.scale, odt(w))


CASES = [
    # B, H_q, H_kv, d, dtype, lens, groups, prefix tokens, partitions
    (8, 32, 8, 128, "f16", [300, 257, 520, 999, 290, 400, 700, 266], 2, 256, 0),
    (6, 64, 8, 128, "bf16", [40, 33, 90, 49, 34, 70], 3, 32, 0),
    (4, 16, 1, 128, "bf16", [200, 145, 160, 300], 2, 144, 5),                 # MQA, group 16
    # one group of 40 members x 4 rows = 160 query rows: two 128-row blocks
    (40, 32, 8, 128, "f16", [530 + 7 * i for i in range(40)], 1, 512, 0),
    # a long shared prefix: several 64-token steps per chunk and a ragged last step
    (16, 64, 8, 128, "bf16", [2100 + 13 * i for i in range(16)], 2, 2048, 0),
    # the prefix pass outweighs the suffixes (the decode keeps few SMs)
    (64, 32, 8, 128, "f16", [2049 + (7 * i) % 40 for i in range(64)], 8, 2048, 0),
    # d = 64: the warp-level prefix pass
    (8, 16, 4, 64, "f16", [300, 257, 520, 999, 290, 400, 700, 266], 2, 256, 0),
    (4, 8, 8, 64, "f16", [600, 513, 530, 1000], 1, 512, 5),                  # MHA
    (6, 32, 8, 64, "bf16", [40, 33, 90, 49, 34, 70], 3, 32, 0),
    (40, 32, 8, 64, "bf16", [530 + 7 * i for i in range(40)], 1, 512, 0),    # two row blocks
]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_d{c[3]}_{c[4]}_g{c[6]}_p{c[7]}")
def test_fused_shared_prefix_matches_oracle_and_plain_step(kvd, fmt, case):
    B, H_q, H_kv, hd, dtype, lens, groups, prefix, parts = case
    w = build_workload("spq", B, H_q, H_kv, hd, dtype, lens, seed=2100 + CASES.index(case),
                       prefix_groups=groups, prefix_tokens=prefix)
    si = step_inputs(w, 0)
    pools = q_state(kvd, w, fmt)
    plain = [t.clone() for t in pools]
    bt = w.block_table.cuda()
    d = {k: v.cuda() for k, v in si.items()}
    gs, gp, per = groups_of(w)
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    out = getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt)(
        d["q"], *pools, bt, d["seq_lens"], gs, gp, per, w.scale, k_new=d["k_new"], v_new=d["v_new"],
        num_partitions=parts, lse_out=lse)
    ref_plain = getattr(kvd, "kvd_decode_step_" + fmt)(d["q"], d["k_new"], d["v_new"], *plain, bt,
                                                        d["seq_lens"], w.scale, num_partitions=parts)
    torch.cuda.synchronize()
    orc = oracle_q8(w, fmt, si)
    assert_pools_equal(pools, orc, data_rows(w.k_cache, w.v_cache, w.block_table, si))
    for a, b in zip(pools, plain):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    ref, ref_lse = oracle_attend(w, si, orc, fmt)
    assert_out_close(out, ref, w.dtype)
    gl = lse.cpu().double().numpy()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.max(np.abs(gl[fin] - ref_lse[fin])) <= LSE_TOL
    assert torch.max(torch.abs(out.float() - ref_plain.float())).item() <= TOL[w.dtype]
    assert kvd.kvd_read_device_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_shared_prefix_attention_only_after_append(kvd, fmt):
    # without k_new/v_new the call only reads: after kvd_append_{fmt} it must
    # agree with kvd_decode_attention_{fmt} and leave the pools untouched
    lens = [300, 257, 520, 999, 290, 400, 700, 266]
    w = build_workload("spqa", 8, 32, 8, 128, "f16", lens, seed=2151, prefix_groups=2, prefix_tokens=256)
    si = step_inputs(w, 0)
    pools = q_state(kvd, w, fmt)
    bt = w.block_table.cuda()
    d = {k: v.cuda() for k, v in si.items()}
    getattr(kvd, "kvd_append_" + fmt)(*pools, bt, d["slot"], d["k_new"], d["v_new"])
    before = [t.clone() for t in pools]
    gs, gp, per = groups_of(w)
    out = getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt)(d["q"], *pools, bt, d["seq_lens"], gs,
                                                                     gp, per, w.scale)
    ref_plain = getattr(kvd, "kvd_decode_attention_" + fmt)(d["q"], *pools, bt, d["seq_lens"], w.scale)
    torch.cuda.synchronize()
    for a, b in zip(pools, before):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    ref, _ = oracle_attend(w, si, oracle_q8(w, fmt, si), fmt)
    assert_out_close(out, ref, w.dtype)
    assert torch.max(torch.abs(out.float() - ref_plain.float())).item() <= TOL[w.dtype]
    assert kvd.kvd_read_device_error() == 0


@pytest.mark.parametrize("hd", [128, 64])
@pytest.mark.parametrize("fmt", FMTS)
def test_shared_prefix_bad_page_is_flagged_and_contained(kvd, fmt, hd):
    # a block-table entry inside group 0's shared prefix points outside the
    # pool: the prefix pass skips that page (d = 128: its tiles hold stale
    # values, masked; d = 64: no warp attends it), the error word says so, and
    # group 1 is still right
    lens = [300, 257, 520, 999, 290, 400, 700, 266]
    w = build_workload("spqbad", 8, 32, 8, hd, "f16", lens, seed=2161, prefix_groups=2, prefix_tokens=256)
    si = step_inputs(w, 0)
    pools = q_state(kvd, w, fmt)
    bt = w.block_table.cuda()
    d = {k: v.cuda() for k, v in si.items()}
    getattr(kvd, "kvd_append_" + fmt)(*pools, bt, d["slot"], d["k_new"], d["v_new"])
    gs, gp, per = groups_of(w)
    bt_bad = bt.clone()
    bt_bad[0, 5] = w.num_blocks + 3
    kvd.kvd_read_device_error(clear=True)
    out = getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt)(d["q"], *pools, bt_bad, d["seq_lens"],
                                                                     gs, gp, per, w.scale)
    torch.cuda.synchronize()
    assert kvd.kvd_read_device_error(clear=True) & kvd.KVD_DEVERR_BLOCK_TABLE
    ref, _ = oracle_attend(w, si, oracle_q8(w, fmt, si), fmt)
    assert_out_close(out[per:], ref[per:], w.dtype)


@pytest.mark.parametrize("hd,dtype,H_q,H_kv", [(128, "f16", 32, 8), (64, "bf16", 16, 4)])
@pytest.mark.parametrize("fmt", FMTS)
def test_uneven_groups(kvd, fmt, hd, dtype, H_q, H_kv):
    # groups of 5, 40, 1, 3 and 7 members sharing 4, 10, 2, 0 and 6 pages:
    # different page counts and row blocks per unit, one member exactly as
    # long as its prefix, one shorter than it (attended whole).  The step's
    # rows are appended through each member's own pages, attention runs on
    # the shared table; the oracle does the same
    w, bt2, gs, gpg, maxg = uneven_groups_case(hd, dtype, H_q, H_kv, seed=2201)
    si = step_inputs(w, 0)
    pools = q_state(kvd, w, fmt)
    d = {k: v.cuda() for k, v in si.items()}
    getattr(kvd, "kvd_append_" + fmt)(*pools, w.block_table.cuda(), d["slot"], d["k_new"], d["v_new"])
    kvd.kvd_read_device_error(clear=True)
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
    out = getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt)(
        d["q"], *pools, bt2.cuda(), d["seq_lens"], gs.cuda(), gpg.cuda(), maxg, w.scale, lse_out=lse)
    torch.cuda.synchronize()
    assert kvd.kvd_read_device_error() == 0
    hk, hv, hks, hvs = oracle_q8(w, fmt, si)
    ref, ref_lse = getattr(oracle, "attend_" + fmt)(to_words(si["q"]), hk, hv, hks, hvs, bt2.numpy(),
                                                    si["seq_lens"].numpy(), w.scale, odt(w))
    assert_out_close(out, ref, w.dtype)
    assert float(np.max(np.abs(lse.cpu().double().numpy() - ref_lse))) <= LSE_TOL


@pytest.mark.parametrize("fmt", FMTS)
def test_group_larger_than_declared_is_flagged_and_attended_whole(kvd, fmt):
    # max_group_size below the 40-member group: that group is invalid (its
    # members are attended whole, the error word says so), the others share
    w, bt2, gs, gpg, maxg = uneven_groups_case(128, "f16", 32, 8, seed=2202)
    si = step_inputs(w, 0)
    pools = q_state(kvd, w, fmt)
    d = {k: v.cuda() for k, v in si.items()}
    getattr(kvd, "kvd_append_" + fmt)(*pools, w.block_table.cuda(), d["slot"], d["k_new"], d["v_new"])
    kvd.kvd_read_device_error(clear=True)
    out = getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt)(
        d["q"], *pools, bt2.cuda(), d["seq_lens"], gs.cuda(), gpg.cuda(), 8, w.scale)
    torch.cuda.synchronize()
    assert kvd.kvd_read_device_error(clear=True) & kvd.KVD_DEVERR_SEQ_LEN
    hk, hv, hks, hvs = oracle_q8(w, fmt, si)
    ref, _ = getattr(oracle, "attend_" + fmt)(to_words(si["q"]), hk, hv, hks, hvs, bt2.numpy(),
                                              si["seq_lens"].numpy(), w.scale, odt(w))
    assert_out_close(out, ref, w.dtype)


@pytest.mark.parametrize("fmt", FMTS)
def test_full_size_cbatch_shared_prefix(kvd, fmt):
    # the continuous-batching workload (8 groups x 32 members sharing a
    # 4096-token prefix, fp16) over the quantised cache: every row against
    # the plain quantised step, sampled sequences against the oracle
    w = named_config("cbatch", device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    pools = q_state(kvd, w, fmt)
    plain = [t.clone() for t in pools]
    bt = w.block_table.cuda()
    gs, gp, per = groups_of(w)
    out = getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt)(
        si["q"], *pools, bt, si["seq_lens"], gs, gp, per, w.scale, k_new=si["k_new"], v_new=si["v_new"])
    ref_plain = getattr(kvd, "kvd_decode_step_" + fmt)(si["q"], si["k_new"], si["v_new"], *plain, bt,
                                                        si["seq_lens"], w.scale)
    torch.cuda.synchronize()
    for a, b in zip(pools, plain):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    del plain
    assert torch.max(torch.abs(out.float() - ref_plain.float())).item() <= TOL[w.dtype]
    lens = si["seq_lens"].cpu().numpy()
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 0, 37, 255})
    (hk, hv, hks, hvs), bts, pages = oracle_q8_rows(w, fmt, si, rows)
    sel = torch.tensor(rows, dtype=torch.long)
    ref, _ = getattr(oracle, "attend_" + fmt)(to_words(si["q"].cpu()[sel]), hk, hv, hks, hvs, bts,
                                              si["seq_lens"].cpu()[sel].numpy(), w.scale, odt(w))
    assert_out_close(out.cpu()[sel], ref, w.dtype)
    assert kvd.kvd_read_device_error() == 0

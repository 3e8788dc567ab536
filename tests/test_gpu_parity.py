"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Append must be bit-exact over the whole pool; attention must be within the
max-abs tolerance (2e-3 fp16, 1e-2 bf16) of the oracle.  Inputs are seeded
synthetic workloads whose unused pool slots hold NaN canaries.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (LSE_TOL, TOL, gpu_state, gpu_step, max_err, max_lse_err, oracle_step,
                         uneven_groups_case, words)
from synth import CANARY_WORD, build_workload, step_inputs, to_words

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvd():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kv_cache_decode_scatters_b200 as m
    m.kvd_read_device_error(clear=True)
    return m


def run_case(kvd, w, step=0, num_partitions=0):
    si = step_inputs(w, step)
    kc, vc, bt = gpu_state(w)
    out, lse = gpu_step(kvd, w, si, kc, vc, bt, num_partitions=num_partitions)
    okc, ovc, ref = oracle_step(w, si)
    return si, kc, vc, out, lse, okc, ovc, ref


# ------------------------------------------------------------------ append

@pytest.mark.parametrize("d,dtype", [(64, "f16"), (128, "bf16"), (128, "f16")])
def test_append_bit_exact_whole_pool(kvd, d, dtype):
    w = build_workload("app", 6, 8, 4, d, dtype, [1, 15, 16, 17, 33, 0], seed=501, spare_pages=5)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    torch.cuda.synchronize()
    okc, ovc = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    oracle.append(okc, ovc, w.block_table.numpy(), si["slot"].numpy(), to_words(si["k_new"]),
                  to_words(si["v_new"]))
    assert np.array_equal(to_words(kc), okc)
    assert np.array_equal(to_words(vc), ovc)
    assert kvd.kvd_read_device_error() == 0


def test_append_out_of_range_is_flagged_not_written(kvd):
    w = build_workload("app", 3, 4, 4, 128, "f16", [5, 9, 20], seed=502)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    slot = si["slot"].clone()
    slot[1] = 16 * w.max_blocks + 3          # beyond the table
    bt_bad = bt.clone()
    bt_bad[2, 1] = w.num_blocks + 100        # page outside the pool
    before_k = to_words(kc).copy()
    kvd.kvd_append(kc, vc, bt_bad, slot.cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    flags = kvd.kvd_read_device_error(clear=True)
    assert flags & kvd.KVD_DEVERR_SLOT and flags & kvd.KVD_DEVERR_BLOCK_TABLE
    okc = before_k.copy()
    ovc = to_words(w.v_cache).copy()
    s0 = si["slot"].numpy().copy()
    s0[1:] = -1
    oracle.append(okc, ovc, w.block_table.numpy(), s0, to_words(si["k_new"]), to_words(si["v_new"]))
    assert np.array_equal(to_words(kc), okc), "only sequence 0 may have been written"


# --------------------------------------------------------------- attention

CASES = [
    # B, H_q, H_kv, d, dtype, lens
    (1, 8, 8, 64, "f16", [1024]),                  # the pages' (1, 8, 1024, 64) example
    (3, 4, 4, 128, "f16", [1, 15, 16]),
    (4, 8, 8, 128, "f16", [17, 31, 32, 33]),
    (2, 8, 1, 128, "bf16", [100, 257]),            # MQA, group 8
    (2, 16, 1, 128, "bf16", [40, 130]),            # MQA, group 16
    (3, 16, 8, 64, "f16", [64, 1, 300]),           # group 2
    (3, 32, 8, 128, "bf16", [500, 77, 1000]),      # group 4
    (4, 64, 8, 128, "bf16", [513, 2049, 16, 999]), # group 8 (70B shape)
    (2, 32, 2, 128, "f16", [1500, 31]),            # group 16
    (2, 12, 4, 64, "bf16", [48, 95]),              # group 3 (padded n-tile)
    (5, 8, 2, 128, "f16", [3, 0, 45, 0, 200]),     # empty sequences in the batch
]


def test_maximum_batch(kvd):
    # B = KVD_MAX_BATCH ragged sequences (0..80 tokens, some empty): eight
    # sequences per prologue thread in the prefix sums, thousands of short
    # pairs per partition, every partition edge inside a short pair
    B = 4096
    g = np.random.default_rng(1234)
    lens = g.integers(0, 81, size=B)
    lens[::97] = 0
    w = build_workload("maxb", B, 8, 2, 128, "f16", [int(x) for x in lens], seed=705, spare_pages=4)
    si, kc, vc, out, lse, okc, ovc, ref = run_case(kvd, w)
    assert np.array_equal(to_words(kc), okc) and np.array_equal(to_words(vc), ovc)
    assert max_err(out, ref) <= TOL[w.dtype]
    for b in np.flatnonzero(lens == 0):
        assert torch.all(out[b] == 0)
    assert kvd.kvd_read_device_error() == 0


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_d{c[3]}_{c[4]}")
def test_decode_matches_oracle(kvd, case):
    B, H_q, H_kv, d, dtype, lens = case
    w = build_workload("par", B, H_q, H_kv, d, dtype, lens, seed=700 + CASES.index(case), spare_pages=3)
    si, kc, vc, out, lse, okc, ovc, ref = run_case(kvd, w)
    assert np.array_equal(to_words(kc), okc) and np.array_equal(to_words(vc), ovc)
    err = max_err(out, ref)
    assert err <= TOL[w.dtype], f"max abs error {err}"
    assert max_lse_err(lse, ref) <= LSE_TOL
    for b, n in enumerate(lens):
        if n == 0:
            assert torch.all(out[b] == 0) and torch.all(torch.isneginf(lse[b]))
    assert kvd.kvd_read_device_error() == 0


@pytest.mark.parametrize("parts", [1, 2, 3, 7, 64, 1000, 0])
def test_partition_counts_agree(kvd, parts):
    w = build_workload("parts", 3, 32, 8, 128, "bf16", [700, 33, 1200], seed=601)
    si, kc, vc, out, lse, okc, ovc, ref = run_case(kvd, w, num_partitions=parts)
    assert max_err(out, ref) <= TOL[w.dtype]
    assert max_lse_err(lse, ref) <= LSE_TOL


@pytest.mark.parametrize("parts", [9, 10])
def test_both_ring_shapes_match_the_oracle(kvd, parts):
    # 64 (sequence, KV head) pairs at d = 128: 9 partitions give more pairs
    # than 7 warps x 9 CTAs, so the launch takes 16 warps x 1 stage; 10 give
    # at most one pair per warp, so 7 warps x 2 stages.  Both sides of that
    # choice match the oracle on the same inputs, every row.
    lens = [257 + 97 * i for i in range(8)]
    w = build_workload("shape", 8, 64, 8, 128, "bf16", lens, seed=613)
    si, kc, vc, out, lse, okc, ovc, ref = run_case(kvd, w, num_partitions=parts)
    assert max_err(out, ref) <= TOL[w.dtype]
    assert max_lse_err(lse, ref) <= LSE_TOL


def test_single_token_returns_v0_exactly(kvd):
    w = build_workload("one", 3, 8, 2, 128, "f16", [1, 1, 1], seed=611)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    out, _ = gpu_step(kvd, w, si, kc, vc, bt)
    v = si["v_new"].cuda().repeat_interleave(4, dim=1)
    assert torch.equal(out, v)


def test_constant_values_give_that_constant(kvd):
    w = build_workload("const", 2, 4, 4, 64, "bf16", [200, 17], seed=612)
    si = step_inputs(w, 0)
    c = torch.randn(4, 64, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    vw = w.v_cache
    for b, n in enumerate([200, 17]):
        for j in range(n - 1):
            vw[int(w.block_table[b, j // 16]), :, j % 16, :] = c
    si["v_new"][:] = c
    kc, vc, bt = gpu_state(w)
    out, _ = gpu_step(kvd, w, si, kc, vc, bt)
    ref = c.float().cuda()[None].expand(2, 4, 64)
    assert torch.max(torch.abs(out.float() - ref)).item() <= 2 ** -7 * ref.abs().max().item()


def test_paged_equals_contiguous_placement(kvd):
    lens = [300, 47, 129]
    a = build_workload("pl", 3, 16, 4, 128, "f16", lens, seed=621, placement="shuffle")
    si = step_inputs(a, 0)
    # same logical content, pages handed out in logical order
    b = build_workload("pl", 3, 16, 4, 128, "f16", lens, seed=621, placement="identity")
    kb = b.k_cache.clone()
    vb = b.v_cache.clone()
    for s in range(3):
        for i in range((lens[s] + 15) // 16):
            kb[int(b.block_table[s, i])] = a.k_cache[int(a.block_table[s, i])]
            vb[int(b.block_table[s, i])] = a.v_cache[int(a.block_table[s, i])]
    b.k_cache, b.v_cache = kb, vb
    outs = []
    for w in (a, b):
        kc, vc, bt = gpu_state(w)
        o, _ = gpu_step(kvd, w, si, kc, vc, bt, num_partitions=37)
        outs.append(o)
    assert torch.equal(outs[0], outs[1]), "physical placement changed the result"


def test_shared_prefix_equals_private_copies(kvd):
    lens = [90, 130, 70, 64 + 1]
    w = build_workload("pre", 4, 8, 2, 128, "bf16", lens, seed=631, prefix_groups=2, prefix_tokens=64)
    assert w.block_table[0, 0] == w.block_table[1, 0]
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    o1, _ = gpu_step(kvd, w, si, kc, vc, bt, num_partitions=5)
    pages, rows = [], torch.full_like(w.block_table, -1)
    for b, n in enumerate(lens):
        for i in range((n + 15) // 16):
            rows[b, i] = len(pages)
            pages.append(int(w.block_table[b, i]))
    idx = torch.tensor(pages)
    kc2, vc2 = w.k_cache[idx].cuda(), w.v_cache[idx].cuda()
    o2, _ = gpu_step(kvd, w, si, kc2, vc2, rows.cuda(), num_partitions=5)
    assert torch.equal(o1, o2)


def test_bad_block_table_entry_is_flagged_and_contained(kvd):
    w = build_workload("bad", 3, 8, 8, 128, "f16", [64, 64, 64], seed=641)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    bt_bad = bt.clone()
    bt_bad[1, 2] = -5
    out = kvd.kvd_decode_attention(si["q"].cuda(), kc, vc, bt_bad, si["seq_lens"].cuda(), w.scale,
                                   num_partitions=3)
    flags = kvd.kvd_read_device_error(clear=True)
    assert flags & kvd.KVD_DEVERR_BLOCK_TABLE
    _, _, ref = oracle_step(w, si)
    g = out.float().cpu().double().numpy()
    for b in (0, 2):
        assert np.max(np.abs(g[b] - ref[b][0])) <= TOL[w.dtype]
    assert np.all(np.isfinite(g[1]))


def test_bad_seq_len_is_flagged(kvd):
    w = build_workload("badlen", 2, 4, 4, 64, "f16", [20, 20], seed=651)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    sl = si["seq_lens"].clone()
    sl[0] = 16 * w.max_blocks + 1
    sl[1] = -4
    kvd.kvd_decode_attention(si["q"].cuda(), kc, vc, bt, sl.cuda(), w.scale)
    assert kvd.kvd_read_device_error(clear=True) & kvd.KVD_DEVERR_SEQ_LEN


def test_generic_merge_matches_oracle(kvd):
    rng = np.random.default_rng(5)
    for d, dt in ((128, torch.float16), (64, torch.bfloat16)):
        B, H_q, S = 3, 4, 6
        po = rng.standard_normal((B, H_q, S, d))
        pl = rng.standard_normal((B, H_q, S)) * 3
        pl[0, 1, 2] = -np.inf
        pl[2, :, :] = -np.inf                     # sequence 2: everything empty
        counts = np.array([6, 4, 5], np.int32)
        po32, pl32 = po.astype(np.float32), pl.astype(np.float32)
        ref, ref_lse = oracle.merge(po32.astype(np.float64), pl32.astype(np.float64), counts)
        lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
        out = kvd.kvd_merge_lse(torch.from_numpy(po32).cuda(), torch.from_numpy(pl32).cuda(),
                                torch.from_numpy(counts).cuda(), lse_out=lse, dtype=dt)
        torch.cuda.synchronize()
        err = np.max(np.abs(out.float().cpu().double().numpy() - ref))
        assert err <= TOL[dt] * 2, err
        fin = np.isfinite(ref_lse)
        got = lse.cpu().double().numpy()
        assert np.array_equal(np.isfinite(got), fin)
        assert np.max(np.abs(got[fin] - ref_lse[fin])) <= LSE_TOL
        assert torch.all(out[2] == 0)


def test_repeated_calls_are_deterministic(kvd):
    w = build_workload("det", 4, 32, 8, 128, "bf16", [900, 40, 1500, 333], seed=661)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    q, sl = si["q"].cuda(), si["seq_lens"].cuda()
    a = kvd.kvd_decode_attention(q, kc, vc, bt, sl, w.scale)
    b = kvd.kvd_decode_attention(q, kc, vc, bt, sl, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ------------------------------------------------------- fused decode step

STEP_CASES = [
    (4, 32, 8, 128, "bf16", [700, 33, 1200, 0], 0),
    (5, 8, 8, 64, "f16", [1, 16, 17, 300, 47], 0),
    (3, 16, 1, 128, "bf16", [200, 64, 129], 7),
    (2, 32, 2, 128, "f16", [513, 31], 3),
]


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_d{c[3]}_{c[4]}_N{c[6]}")
def test_fused_step_equals_append_then_attend(kvd, case):
    B, H_q, H_kv, d, dtype, lens, parts = case
    w = build_workload("step", B, H_q, H_kv, d, dtype, lens, seed=800 + STEP_CASES.index(case),
                       spare_pages=2)
    si = step_inputs(w, 0)
    kc1, vc1, bt = gpu_state(w)
    o1, l1 = gpu_step(kvd, w, si, kc1, vc1, bt, num_partitions=parts)
    kc2, vc2, _ = gpu_state(w)
    l2 = torch.empty_like(l1)
    o2 = kvd.kvd_decode_step(si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), kc2, vc2, bt,
                             si["seq_lens"].cuda(), w.scale, num_partitions=parts, lse_out=l2)
    torch.cuda.synchronize()
    assert torch.equal(kc1.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc1.view(torch.int16), vc2.view(torch.int16))
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)
    _, _, ref = oracle_step(w, si)
    assert max_err(o2, ref) <= TOL[w.dtype]
    assert kvd.kvd_read_device_error() == 0


def test_fused_steps_continuous_batching(kvd):
    # 4 consecutive fused steps with a shared prefix, against the oracle
    lens = [40, 47, 33, 64 + 5]
    w = build_workload("steps", 4, 8, 2, 128, "f16", lens, seed=851, steps=4, prefix_groups=2,
                       prefix_tokens=32)
    kc, vc, bt = gpu_state(w)
    okc, ovc = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    for step in range(4):
        si = step_inputs(w, step)
        out = kvd.kvd_decode_step(si["q"].cuda(), si["k_new"].cuda(), si["v_new"].cuda(), kc, vc,
                                  bt, si["seq_lens"].cuda(), w.scale)
        torch.cuda.synchronize()
        okc, ovc, ref = oracle_step(w, si, okc, ovc)
        assert max_err(out, ref) <= TOL[w.dtype]
    assert np.array_equal(to_words(kc), okc) and np.array_equal(to_words(vc), ovc)


def test_cuda_graph_of_16_steps_matches_eager(kvd):
    # continuous batching: 16 fused append+attend steps captured once in a CUDA
    # graph; replaying it must give the eager steps' caches and outputs exactly
    lens = [40, 47, 33, 69, 52, 38, 90, 61]
    w = build_workload("graph", 8, 16, 4, 128, "bf16", lens, seed=871, steps=16, prefix_groups=2,
                       prefix_tokens=32)
    steps = [step_inputs(w, s) for s in range(16)]
    dev = [{k: v.cuda() for k, v in si.items()} for si in steps]
    ws = kvd.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, 0)

    kc_e, vc_e, bt = gpu_state(w)
    outs_e = [torch.empty_like(d["q"]) for d in dev]
    for d, o in zip(dev, outs_e):
        kvd.kvd_decode_step(d["q"], d["k_new"], d["v_new"], kc_e, vc_e, bt, d["seq_lens"], w.scale,
                            out=o, workspace=ws)
    torch.cuda.synchronize()

    kc_g, vc_g, _ = gpu_state(w)
    outs_g = [torch.empty_like(d["q"]) for d in dev]
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for d, o in zip(dev, outs_g):
                kvd.kvd_decode_step(d["q"], d["k_new"], d["v_new"], kc_g, vc_g, bt, d["seq_lens"],
                                    w.scale, out=o, workspace=ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs_e, outs_g):
        assert torch.equal(a, b)
    assert torch.equal(kc_e.view(torch.int16), kc_g.view(torch.int16))
    assert torch.equal(vc_e.view(torch.int16), vc_g.view(torch.int16))
    # a second replay rewrites the same rows and recomputes the same outputs
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs_e, outs_g):
        assert torch.equal(a, b)
    del g


# --------------------------------------------------- shared-prefix decode

def groups_of(w):
    per = w.B // w.groups
    start = torch.arange(0, w.B + 1, per, dtype=torch.int32)
    pages = torch.full((w.groups,), w.prefix_tokens // 16, dtype=torch.int32)
    return start.cuda(), pages.cuda(), per


SP_CASES = [
    # B, H_q, H_kv, d, dtype, lens, groups, prefix tokens, partitions
    (8, 32, 8, 128, "f16", [300, 257, 520, 999, 290, 400, 700, 266], 2, 256, 0),
    (6, 64, 8, 128, "bf16", [40, 33, 90, 49, 34, 70], 3, 32, 0),
    (4, 8, 8, 64, "f16", [600, 513, 530, 1000], 1, 512, 5),
    (4, 16, 1, 128, "bf16", [200, 145, 160, 300], 2, 144, 0),   # MQA, group 16
    # one group of 40 members x 4 rows = 160 query rows: two 128-row blocks
    (40, 32, 8, 128, "f16", [530 + 7 * i for i in range(40)], 1, 512, 0),
    # a long shared prefix: several 64-token steps per chunk and a ragged last step
    (16, 64, 8, 128, "bf16", [2100 + 13 * i for i in range(16)], 2, 2048, 0),
    # the prefix pass outweighs the suffixes: the suffix decode keeps a few
    # SMs and the prefix pass runs beside it on the rest
    (64, 32, 8, 128, "f16", [2049 + (7 * i) % 40 for i in range(64)], 8, 2048, 0),
]


@pytest.mark.parametrize("case", SP_CASES, ids=lambda c: f"B{c[0]}_Hq{c[1]}_Hkv{c[2]}_d{c[3]}_{c[4]}_g{c[6]}")
def test_shared_prefix_matches_oracle_and_plain_decode(kvd, case):
    B, H_q, H_kv, d, dtype, lens, groups, prefix, parts = case
    w = build_workload("sp", B, H_q, H_kv, d, dtype, lens, seed=900 + SP_CASES.index(case),
                       prefix_groups=groups, prefix_tokens=prefix)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    ref_gpu, _ = gpu_step(kvd, w, si, kc, vc, bt, num_partitions=parts)   # append + plain decode
    gs, gp, per = groups_of(w)
    lse = torch.empty((B, H_q), dtype=torch.float32, device="cuda")
    out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt, si["seq_lens"].cuda(),
                                                 gs, gp, per, w.scale, num_partitions=parts,
                                                 lse_out=lse)
    torch.cuda.synchronize()
    _, _, ref = oracle_step(w, si)
    assert max_err(out, ref) <= TOL[w.dtype]
    assert max_lse_err(lse, ref) <= LSE_TOL
    assert torch.max(torch.abs(out.float() - ref_gpu.float())).item() <= TOL[w.dtype]
    assert kvd.kvd_read_device_error() == 0


def test_shared_prefix_side_by_side_is_bit_reproducible(kvd):
    # The prefix pass runs beside the suffix decode, and the split of the SMs
    # between them is computed on the device.  Neither the split nor the
    # order in which the two passes finish may change a bit of the output.
    B = 64
    w = build_workload("spr", B, 32, 8, 128, "f16", [2049 + (13 * i) % 300 for i in range(B)],
                       seed=1404, prefix_groups=8, prefix_tokens=2048)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    gs, gp, per = groups_of(w)
    outs = []
    for _ in range(3):
        lse = torch.empty((B, 32), dtype=torch.float32, device="cuda")
        out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt, si["seq_lens"].cuda(),
                                                     gs, gp, per, w.scale, lse_out=lse)
        outs.append((out, lse))
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(l, outs[0][1])
    assert kvd.kvd_read_device_error() == 0


@pytest.mark.parametrize("scale", [-0.09, 0.0])
def test_shared_prefix_any_scale(kvd, scale):
    # a negative scale turns the row maximum into a minimum of the raw scores;
    # a zero scale gives uniform weights (the mean of V over the sequence)
    lens = [300, 257, 520, 999, 290, 400, 700, 266]
    w = build_workload("spscale", 8, 32, 8, 128, "f16", lens, seed=981, prefix_groups=2,
                       prefix_tokens=256, scale=scale)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    gs, gp, per = groups_of(w)
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
    out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt, si["seq_lens"].cuda(),
                                                 gs, gp, per, w.scale, k_new=si["k_new"].cuda(),
                                                 v_new=si["v_new"].cuda(), lse_out=lse)
    torch.cuda.synchronize()
    _, _, ref = oracle_step(w, si)
    assert max_err(out, ref) <= TOL[w.dtype]
    assert max_lse_err(lse, ref) <= LSE_TOL
    assert kvd.kvd_read_device_error() == 0


def test_shared_prefix_bad_page_is_flagged_and_contained(kvd):
    # a block-table entry of group 0's shared prefix points outside the pool:
    # the error word says so and group 1 is still exact
    lens = [300, 257, 520, 999, 290, 400, 700, 266]
    w = build_workload("spbad", 8, 32, 8, 128, "f16", lens, seed=971, prefix_groups=2,
                       prefix_tokens=256)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    gs, gp, per = groups_of(w)
    bt_bad = bt.clone()
    bt_bad[0, 5] = w.num_blocks + 3
    kvd.kvd_read_device_error(clear=True)
    out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt_bad, si["seq_lens"].cuda(),
                                                 gs, gp, per, w.scale)
    torch.cuda.synchronize()
    assert kvd.kvd_read_device_error(clear=True) & kvd.KVD_DEVERR_BLOCK_TABLE
    _, _, ref = oracle_step(w, si)
    for b in range(per, w.B):
        assert np.max(np.abs(out[b].float().cpu().double().numpy() - ref[b][0])) <= TOL[w.dtype]


def test_shared_prefix_fused_append_matches_decode_step(kvd):
    lens = [300, 257, 520, 999, 290, 400, 700, 266]
    w = build_workload("spf", 8, 32, 8, 128, "bf16", lens, seed=951, steps=3, prefix_groups=4,
                       prefix_tokens=256)
    gs, gp, per = groups_of(w)
    kc1, vc1, bt = gpu_state(w)
    kc2, vc2, _ = gpu_state(w)
    okc, ovc = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    for step in range(3):
        si = step_inputs(w, step)
        d = {k: v.cuda() for k, v in si.items()}
        o1 = kvd.kvd_decode_step(d["q"], d["k_new"], d["v_new"], kc1, vc1, bt, d["seq_lens"], w.scale)
        o2 = kvd.kvd_decode_attention_shared_prefix(d["q"], kc2, vc2, bt, d["seq_lens"], gs, gp, per,
                                                    w.scale, k_new=d["k_new"], v_new=d["v_new"])
        torch.cuda.synchronize()
        okc, ovc, ref = oracle_step(w, si, okc, ovc)
        assert max_err(o2, ref) <= TOL[w.dtype]
        assert torch.max(torch.abs(o1.float() - o2.float())).item() <= TOL[w.dtype]
    assert torch.equal(kc1.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(vc1.view(torch.int16), vc2.view(torch.int16))
    assert np.array_equal(to_words(kc2), okc)
    assert kvd.kvd_read_device_error() == 0


def test_shared_prefix_member_shorter_than_prefix_is_attended_whole(kvd):
    # group claims 4 shared pages, but member 1 has only 40 tokens: it must
    # fall back to plain attention and still match the oracle
    lens = [90, 40, 100, 120]
    w = build_workload("spshort", 4, 8, 2, 128, "f16", lens, seed=961)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    # make sequences 0 and 1 share sequence 0's first 4 pages in the table
    bt2 = bt.clone()
    bt2[1, :3] = bt[0, :3]
    kc_h, vc_h = kc.cpu(), vc.cpu()
    gs = torch.tensor([0, 2, 4], dtype=torch.int32).cuda()
    gp = torch.tensor([4, 0], dtype=torch.int32).cuda()
    out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt2, si["seq_lens"].cuda(),
                                                 gs, gp, 2, w.scale)
    torch.cuda.synchronize()
    q = to_words(si["q"])
    ref, _ = oracle.attend(q, to_words(kc_h), to_words(vc_h), bt2.cpu().numpy(),
                           si["seq_lens"].numpy(), w.scale, oracle.F16)
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype]


@pytest.mark.parametrize("d,dtype,H_q,H_kv", [(128, "f16", 32, 8), (128, "bf16", 64, 8), (64, "f16", 16, 4)])
def test_shared_prefix_uneven_groups(kvd, d, dtype, H_q, H_kv):
    # groups of 5, 40, 1, 3 and 7 members sharing 4, 10, 2, 0 and 6 pages:
    # units of different page counts and row blocks, one member exactly as
    # long as its prefix, one shorter than it
    w, bt2, gs, gpg, maxg = uneven_groups_case(d, dtype, H_q, H_kv, seed=1401)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    kvd.kvd_read_device_error(clear=True)
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda")
    out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt2.cuda(), si["seq_lens"].cuda(),
                                                 gs.cuda(), gpg.cuda(), maxg, w.scale, lse_out=lse)
    torch.cuda.synchronize()
    assert kvd.kvd_read_device_error() == 0
    ref, ref_lse = oracle.attend(to_words(si["q"]), to_words(kc), to_words(vc), bt2.numpy(),
                                 si["seq_lens"].numpy(), w.scale,
                                 oracle.BF16 if w.dtype == torch.bfloat16 else oracle.F16)
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"
    assert float(np.max(np.abs(lse.cpu().double().numpy() - ref_lse))) <= LSE_TOL


@pytest.mark.parametrize("starts", [[4, 8, 0, 4], [0, 4, 4, 8]], ids=["unordered", "empty_group"])
def test_shared_prefix_group_starts_in_any_order(kvd, starts):
    # Decreasing group starts make the plan walk the groups in order instead
    # of searching them: [4, 8, 0, 4] names the workload's two groups in
    # reverse order around an invalid group [8, 0), which is flagged.  With
    # [0, 4, 4, 8] the search skips the empty middle group.
    w = build_workload("spo", 8, 32, 8, 128, "f16", [300, 257, 520, 999, 290, 400, 700, 266],
                       seed=1403, prefix_groups=2, prefix_tokens=256)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    kvd.kvd_read_device_error(clear=True)
    gs = torch.tensor(starts, dtype=torch.int32, device="cuda")
    gp = torch.full((3,), 16, dtype=torch.int32, device="cuda")
    out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt, si["seq_lens"].cuda(),
                                                 gs, gp, 4, w.scale)
    torch.cuda.synchronize()
    flagged = kvd.kvd_read_device_error(clear=True)
    assert bool(flagged & kvd.KVD_DEVERR_SEQ_LEN) == (starts[1] > starts[2])
    _, _, ref = oracle_step(w, si)
    assert max_err(out, ref) <= TOL[w.dtype]


def test_shared_prefix_group_larger_than_declared_is_flagged_and_attended_whole(kvd):
    # max_group_size below the 40-member group: that group is invalid (its
    # members are attended whole, the error word says so), the others share
    w, bt2, gs, gpg, maxg = uneven_groups_case(128, "f16", 32, 8, seed=1402)
    si = step_inputs(w, 0)
    kc, vc, bt = gpu_state(w)
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    kvd.kvd_read_device_error(clear=True)
    out = kvd.kvd_decode_attention_shared_prefix(si["q"].cuda(), kc, vc, bt2.cuda(), si["seq_lens"].cuda(),
                                                 gs.cuda(), gpg.cuda(), 8, w.scale)
    torch.cuda.synchronize()
    assert kvd.kvd_read_device_error(clear=True) & kvd.KVD_DEVERR_SEQ_LEN
    ref, _ = oracle.attend(to_words(si["q"]), to_words(kc), to_words(vc), bt2.numpy(),
                           si["seq_lens"].numpy(), w.scale, oracle.F16)
    err = float(np.max(np.abs(out.float().cpu().double().numpy() - ref)))
    assert err <= TOL[w.dtype], f"max abs error {err}"

"""Host-side pieces of bench.py that need no GPU: the hash-keyed lookup of a
profile's DRAM traffic and the bounded CPU-oracle sampler of the reference arm."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _summary(tmp, name, workload, mode, digest, nbytes):
    (tmp / name).write_text(
        f"# test\n\nworkload: {workload}\ncache_mode: {mode}\n"
        f"decode_source_sha256_16: {digest}\ndram_bytes_per_launch: {nbytes}\n", encoding="utf-8")


def test_profile_traffic_is_keyed_by_source_hash_workload_and_mode(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))
    now = bench.source_hash()
    _summary(tmp_path, "decode_kernel_a.md", "mha7b", "fused", now, 111)
    _summary(tmp_path, "decode_kernel_b.md", "mha7b", "fp8", now, 222)
    _summary(tmp_path, "decode_kernel_c.md", "gqa70b", "fused", "0" * 16, 333)  # stale source
    _summary(tmp_path, "other_kernel.md", "gqa70b", "fused", now, 444)          # not a decode summary
    assert bench.profile_traffic("mha7b", "fused") == 111
    assert bench.profile_traffic("mha7b", "fp8") == 222
    assert bench.profile_traffic("mha7b", "int8") is None
    assert bench.profile_traffic("gqa70b", "fused") is None


def test_committed_profiles_parse():
    # every committed decode summary carries the machine-readable lines
    for name in sorted(os.listdir(os.path.join(ROOT, "profiles"))):
        if not (name.startswith("decode_kernel") and name.endswith(".md")):
            continue
        text = open(os.path.join(ROOT, "profiles", name), encoding="utf-8").read()
        if "dram_bytes_per_launch:" in text:
            for key in ("workload:", "cache_mode:", "decode_source_sha256_16:"):
                assert key in text, f"{name} lacks {key}"


def test_oracle_sampler_bounds_and_reuses_inputs():
    smp = bench.OracleSampler("tiny")
    gbs, spent, done = smp.run(0.0)             # at least one unit even with no budget
    assert done == 1 and gbs > 0 and spent > 0
    gbs2, _, done2 = smp.run(0.0, min_units=3)
    assert done2 == 3 and gbs2 > 0
    assert len(smp.cache) == 1                  # one sequence in the tiny shape, built once
    assert "4 append+attend units over 1 of the 1 sequences of the tiny shape" in smp.describe()


def test_long_sequences_are_sampled_by_kv_head():
    smp = bench.OracleSampler("long")
    c = smp._inputs(0)
    # 131072 tokens x 2 x 128 x 2 B = 64 MiB per KV head: one KV head and its 8 query heads
    assert c["heads"] == (8, 1)


def test_reference_arm_prints_one_json_line(capsys):
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "4",
                             "--warmup", "3", "--ref-budget", "0.5"])
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["steps"] == 4 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def _full_oracle(w, si):
    import oracle
    from synth import to_words
    kc, vc = to_words(w.k_cache).copy(), to_words(w.v_cache).copy()
    oracle.append(kc, vc, w.block_table.numpy(), si["slot"].numpy(), to_words(si["k_new"]),
                  to_words(si["v_new"]))
    dt = oracle.BF16 if w.dtype.is_floating_point and w.dtype == bench.torch.bfloat16 else oracle.F16
    out, _ = oracle.attend(to_words(si["q"]), kc, vc, w.block_table.numpy(), si["seq_lens"].numpy(),
                           w.scale, dt)
    return out


def test_row_snapshot_renumbers_pages_and_feeds_the_oracle():
    # the parity sample's compact copy (shared prefix pages, shuffled pool,
    # sampled rows) must give the oracle exactly the rows of the whole batch
    from synth import build_workload, step_inputs
    w = build_workload("snap", 8, 8, 2, 64, "f16", [70, 33, 90, 37, 64, 65, 100, 34], seed=31,
                       prefix_groups=2, prefix_tokens=32, spare_pages=3)
    si = step_inputs(w, 0)
    rows = bench.sample_sequences(w, 3, 5)
    assert 1 in rows and 6 in rows            # shortest and longest are always sampled
    snap = bench.RowSnapshot(w, si, rows)
    assert snap.k.shape[0] < w.num_blocks      # only the sampled sequences' pages
    full = _full_oracle(w, si)
    err, spent, gbs, threads = bench.oracle_parity(snap, full[rows])
    assert err == 0.0 and spent > 0 and threads >= 1
    # a wrong row is seen
    wrong = full[rows].copy()
    wrong[-1, 0, 0] += 0.01
    assert abs(bench.oracle_parity(snap, wrong)[0] - 0.01) < 1e-9


@pytest.mark.parametrize("fmt", ["fp8", "int8", "int4"])
def test_row_snapshot_quantised_parity_uses_the_oracles_quantisation(fmt):
    import oracle
    from synth import build_workload, step_inputs, to_words
    w = build_workload("snap8", 3, 8, 2, 128, "bf16", [40, 17, 33], seed=32, spare_pages=2)
    si = step_inputs(w, 0)
    snap = bench.RowSnapshot(w, si, [0, 1, 2])
    quant = getattr(oracle, "quantize_" + fmt)
    k8, ks = quant(to_words(w.k_cache), oracle.BF16)
    v8, vs = quant(to_words(w.v_cache), oracle.BF16)
    getattr(oracle, "append_" + fmt)(k8, v8, ks, vs, w.block_table.numpy(), si["slot"].numpy(),
                                     to_words(si["k_new"]), to_words(si["v_new"]), oracle.BF16)
    ref, _ = getattr(oracle, "attend_" + fmt)(to_words(si["q"]), k8, v8, ks, vs, w.block_table.numpy(),
                                              si["seq_lens"].numpy(), w.scale, oracle.BF16)
    assert bench.oracle_parity(snap, ref, fmt=fmt)[0] == 0.0


def test_quantised_byte_counts():
    # a d = 128 row: 128 code bytes (64 for INT4) + 4 fp32 scales
    assert bench.quant_row_bytes("fp8", 128) == 144
    assert bench.quant_row_bytes("int8", 128) == 144
    assert bench.quant_row_bytes("int4", 128) == 80
    assert bench.quant_row_bytes("int4", 64) == 40
    from synth import build_workload, step_inputs
    w = build_workload("bytes4", 2, 8, 2, 128, "bf16", [40, 17], seed=33, spare_pages=2)
    si = step_inputs(w, 0)
    toks = int(si["seq_lens"].sum())
    assert bench.quant_attention_bytes(w, si["seq_lens"], "int4") == toks * 2 * 2 * 80 + 2 * 2 * 8 * 128 * 2
    rows = int((si["slot"] >= 0).sum()) * 2
    assert bench.quant_append_bytes(w, si["slot"], "int4") == rows * 2 * (256 + 80)
    snap = bench.RowSnapshot(w, si, [0, 1])
    assert snap.nbytes_q("int4") == (bench.quant_attention_bytes(w, si["seq_lens"], "int4")
                                     + bench.quant_append_bytes(w, si["slot"], "int4"))

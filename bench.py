"""Benchmark of one paged-KV decode step (append + decode attention + merge).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mha7b]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

Prints ONE JSON line (rank 0).  Metric: achieved HBM GB/s of the decode step
= algorithmic bytes of one step (K/V pages of every (sequence, KV head) pair,
q, out, and the appended K/V rows read and written) / device time of one step.
Inputs are resident in HBM when timing starts; the KV pool (2.1 GB for the
7B-shape workload) is far larger than the 126 MB L2, so no flush is needed
between steps.

Multi-GPU (torchrun): every rank runs the same workload on its own GPU with no
data-path collective (the decode step of independent sequences shards by
batch); value = bytes of all ranks / slowest rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth import build_workload, config_spec, named_config, step_inputs, to_words  # noqa: E402

METRIC = "paged decode-attention achieved HBM GB/s (% of B200 peak); us per decode step"
FALLBACK_HBM_GBS = 6650.0
PROFILE_DIR = os.path.join(ROOT, "profiles")
DECODE_SOURCES = [os.path.join(ROOT, "kv_cache_decode_scatters_b200", "csrc", f)
                  for f in ("decode.cu", "tile.cuh", "common.cuh", "quant.cuh")]


# ------------------------------------------------------------------ helpers

def attention_bytes(w, seq_lens) -> int:
    """K/V pages read + q read + out written (algorithmic, per step)."""
    s = 2  # fp16 / bf16 bytes
    kv = int(seq_lens.to(torch.int64).sum().item()) * w.H_kv * 2 * w.d * s
    return kv + 2 * w.B * w.H_q * w.d * s


# quantised cache formats: the name of the code type, and the bytes of one
# stored row of d channels (codes, then its fp32 scale per 32 channels)
QUANT_NAMES = {"fp8": "E4M3", "int8": "INT8", "int4": "INT4"}


def quant_row_bytes(fmt, d) -> int:
    return (d // 2 if fmt == "int4" else d) + (d // 32) * 4


def quant_attention_bytes(w, seq_lens, fmt) -> int:
    """Attention bytes over a quantised cache: codes + fp32 group scales + q + out."""
    per_tok = w.H_kv * 2 * quant_row_bytes(fmt, w.d)
    return int(seq_lens.to(torch.int64).sum().item()) * per_tok + 2 * w.B * w.H_q * w.d * 2


def quant_append_bytes(w, slot, fmt) -> int:
    """Quantising append: each K and V row read in 16 bits, written as codes + scales."""
    rows = int((slot >= 0).sum().item()) * w.H_kv
    return rows * 2 * (w.d * 2 + quant_row_bytes(fmt, w.d))


def append_bytes(w, slot) -> int:
    rows = int((slot >= 0).sum().item()) * w.H_kv
    return rows * w.d * 2 * 2 * 2          # K and V rows, read from k_new/v_new and written


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def read_only_peak_gbs(kvd, nbytes=4 << 30, reps=5):
    """Read-only HBM bandwidth of this device, measured by the library's
    streaming kernels (kvd_read_stream) over a buffer far larger than L2:
    best of `reps` launches of each form, CUDA events on the launching
    stream.  Returns {form: GB/s}."""
    x = torch.ones(nbytes // 4, dtype=torch.int32, device="cuda")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    res = {}
    for name, mode in (("vector", kvd.KVD_READ_VECTOR), ("bulk", kvd.KVD_READ_BULK)):
        kvd.kvd_read_stream(x, mode, sink=sink, stream=stream)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            kvd.kvd_read_stream(x, mode, sink=sink, stream=stream)
            b.record(stream)
            torch.cuda.synchronize()
            best = min(best, a.elapsed_time(b))
        res[name] = nbytes / (best * 1e-3) / 1e9
    del x
    torch.cuda.empty_cache()
    return res


def source_hash() -> str:
    """Hash of the decode kernel's sources (kernel, tile, shared helpers)."""
    h = hashlib.sha256()
    for path in DECODE_SOURCES:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_traffic(workload: str, mode: str):
    """DRAM bytes per decode launch from a committed ncu summary under
    profiles/, if one was taken on the current decode kernel sources for this
    workload and step mode ("fused", "separate_append", "shared_prefix", or a
    quantised format "fp8" / "int8" / "int4", optionally with
    "_separate_append")."""
    try:
        names = sorted(os.listdir(PROFILE_DIR))
    except OSError:
        return None
    want = source_hash()
    for name in names:
        if not (name.startswith("decode_kernel") and name.endswith(".md")):
            continue
        with open(os.path.join(PROFILE_DIR, name), encoding="utf-8") as f:
            text = f.read()
        m_src = re.search(r"decode_source_sha256_16:\s*([0-9a-f]+)", text)
        m_wl = re.search(r"workload:\s*(\S+)", text)
        m_mode = re.search(r"cache_mode:\s*(\S+)", text)
        m_b = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
        if not (m_src and m_b and m_wl and m_mode):
            continue
        if m_src.group(1) == want and m_wl.group(1) == workload and m_mode.group(1) == mode:
            return int(m_b.group(1))
    return None


def sample_sequences(w, k, seed):
    """k seeded random sequences of w plus its longest and its shortest."""
    g = torch.Generator().manual_seed(seed)
    pick = set(torch.randperm(w.B, generator=g)[:min(k, w.B)].tolist())
    pick.add(int(torch.argmax(w.seq_lens0)))
    pick.add(int(torch.argmin(w.seq_lens0)))
    return sorted(pick)


class RowSnapshot:
    """Host copy of what a few sequences of a workload read -- their pages
    (renumbered compactly, storage words) and their step inputs -- taken
    before any kernel writes the pool.  It is the input of the CPU-baseline
    leg's oracle run, whose result the GPU's output rows are compared with."""

    def __init__(self, w, si, rows):
        bt = w.block_table.cpu()
        n = si["seq_lens"].cpu()
        npg = [(int(n[b]) + 15) // 16 for b in rows]
        pages = sorted({int(p) for b, m in zip(rows, npg) for p in bt[b, :m].tolist()})
        idx = torch.tensor(pages or [0], dtype=torch.long, device=w.k_cache.device)
        self.k = to_words(w.k_cache.index_select(0, idx)).copy()
        self.v = to_words(w.v_cache.index_select(0, idx)).copy()
        remap = {p: i for i, p in enumerate(pages)}
        self.bt = np.zeros((len(rows), max(npg + [1])), dtype=np.int32)
        for i, (b, m) in enumerate(zip(rows, npg)):
            self.bt[i, :m] = [remap[p] for p in bt[b, :m].tolist()]
        sel = torch.tensor(rows, dtype=torch.long)
        self.rows = rows
        self.q = to_words(si["q"].cpu()[sel])
        self.k_new = to_words(si["k_new"].cpu()[sel])
        self.v_new = to_words(si["v_new"].cpu()[sel])
        self.seq_lens = n[sel].numpy().astype(np.int32)
        self.slot = si["slot"].cpu()[sel].numpy().astype(np.int32)
        self.scale = w.scale
        self.bf16 = w.dtype == torch.bfloat16
        tokens = int(self.seq_lens.astype(np.int64).sum())
        appended = int((self.slot >= 0).sum()) * w.H_kv
        self.nbytes = (tokens * w.H_kv * 2 * w.d * 2 + 2 * len(rows) * w.H_q * w.d * 2
                       + appended * w.d * 2 * 2 * 2)
        self._q = (tokens * w.H_kv * 2, 2 * len(rows) * w.H_q * w.d * 2, appended * 2, w.d)

    def nbytes_q(self, fmt):
        """The bytes over a quantised cache: codes + per-32-channel fp32 scales."""
        kv_rows, qo, app_rows, d = self._q
        return kv_rows * quant_row_bytes(fmt, d) + qo + app_rows * (d * 2 + quant_row_bytes(fmt, d))

    def describe(self, w):
        return (f"sequences {self.rows} of {w.B} (lengths {self.seq_lens.tolist()}), all "
                f"{w.H_q} query heads each")

    def describe_short(self):
        return f"sequences {self.rows} (lengths {self.seq_lens.tolist()}), all query heads"


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"]
        except Exception:
            sel = []
        self.cmd = ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "100"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, dist.get_rank(), world, local
    if n_gpus > 1:
        raise SystemExit("--gpus N > 1 must be launched with torchrun (one rank per GPU)")
    return None, 0, 1, 0


def max_over_ranks(dist, x: float) -> float:
    """Largest x over all ranks (host timing bookkeeping, not a data-path collective)."""
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(dist, world, steps, total_ms, attn_ms, step_bytes):
    """Whole-job numbers from per-rank device times: the slowest rank sets the
    step time; value counts the bytes every rank processed (weak scaling)."""
    total_ms = max_over_ranks(dist, total_ms)
    attn_ms = max_over_ranks(dist, attn_ms)
    ms_step = total_ms / steps
    value = world * step_bytes / (ms_step * 1e-3) / 1e9
    return ms_step, attn_ms, value


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ------------------------------------------------------------ CPU (oracle)

class OracleSampler:
    """The fp64 CPU oracle (append + attend) timed on units of a workload's
    shape: one sequence with all its heads, or, for a sequence too long to
    time often (more than 64 MB of K/V), the sequence with a subset of its KV
    heads and their query heads.  Inputs are built once per sequence and
    reused, so each timed step is oracle work only."""

    UNIT_BYTES = 64 << 20
    MAX_SEQS = 16  # distinct sequences prepared (cycled; bounds host memory)

    def __init__(self, w_name, threads=0):
        import oracle
        self.oracle = oracle
        self.name = w_name
        self.spec = config_spec(w_name)
        self.threads = threads if threads > 0 else oracle.max_threads()
        self.cache = {}
        self.next = 0
        self.units = []

    def _inputs(self, b):
        if b not in self.cache:
            sp = self.spec
            n = sp["lens"][b]
            per_head = n * 2 * sp["d"] * 2
            hkv = max(1, min(sp["H_kv"], self.UNIT_BYTES // max(1, per_head)))
            G = sp["H_q"] // sp["H_kv"]
            w = build_workload("cpu_sample", 1, G * hkv, hkv, sp["d"], sp["dtype"], [n],
                               seed=4242 + b, placement="shuffle")
            si = step_inputs(w, 0)
            self.cache[b] = dict(
                scale=w.scale, kc=to_words(w.k_cache).copy(), vc=to_words(w.v_cache).copy(),
                bt=w.block_table.numpy(), q=to_words(si["q"]), kn=to_words(si["k_new"]),
                vn=to_words(si["v_new"]), sl=si["seq_lens"].numpy(), slot=si["slot"].numpy(),
                dt=self.oracle.BF16 if w.dtype == torch.bfloat16 else self.oracle.F16,
                nbytes=attention_bytes(w, si["seq_lens"]) + append_bytes(w, si["slot"]),
                heads=(G * hkv, hkv))
        return self.cache[b]

    def run(self, budget_s, min_units=1):
        """Units one after another until about budget_s seconds of oracle time.
        Returns (GB/s, seconds, units)."""
        done, spent, nbytes = 0, 0.0, 0
        while spent < budget_s or done < min_units:
            b = self.next % min(self.spec["B"], self.MAX_SEQS)
            self.next += 1
            c = self._inputs(b)
            t0 = time.perf_counter()
            self.oracle.append(c["kc"], c["vc"], c["bt"], c["slot"], c["kn"], c["vn"])
            self.oracle.attend(c["q"], c["kc"], c["vc"], c["bt"], c["sl"], c["scale"], c["dt"],
                               nthreads=self.threads)
            spent += time.perf_counter() - t0
            nbytes += c["nbytes"]
            done += 1
            self.units.append(b)
        return nbytes / spent / 1e9, spent, done

    def describe(self):
        sp = self.spec
        seen = sorted(set(self.units))
        shapes = {self._inputs(b)["heads"] for b in seen}
        heads = ", ".join(f"{hq} query / {hk} KV heads" for hq, hk in sorted(shapes))
        return (f"{len(self.units)} append+attend units over {len(seen)} of the {sp['B']} sequences "
                f"of the {self.name} shape ({heads} per unit; lengths "
                f"{[sp['lens'][b] for b in seen[:8]]}{' ...' if len(seen) > 8 else ''}), "
                f"fp64 oracle, {self.threads} OpenMP threads")


def oracle_parity(snap, gpu_rows, threads=0, fmt=None):
    """CPU-baseline leg: the oracle's append + attend on a RowSnapshot (for an
    8-bit cache, after the oracle's own quantisation of the snapshot's pages),
    timed, and the largest |GPU - oracle| over the snapshot's output rows.
    gpu_rows: float64 [rows, H_q, d] of the GPU's output for those sequences.
    Returns (max_abs_err, seconds, GB/s of the oracle, threads)."""
    import oracle
    dt = oracle.BF16 if snap.bf16 else oracle.F16
    threads = threads if threads > 0 else oracle.max_threads()
    if fmt is None:
        t0 = time.perf_counter()
        kc, vc = snap.k.copy(), snap.v.copy()
        oracle.append(kc, vc, snap.bt, snap.slot, snap.k_new, snap.v_new)
        ref, _ = oracle.attend(snap.q, kc, vc, snap.bt, snap.seq_lens, snap.scale, dt, nthreads=threads)
    else:
        # the 8-bit pool is quantised once (setup, as on the GPU), then timed
        quant = getattr(oracle, "quantize_" + fmt)
        k8, ks = quant(snap.k, dt)
        v8, vs = quant(snap.v, dt)
        t0 = time.perf_counter()
        getattr(oracle, "append_" + fmt)(k8, v8, ks, vs, snap.bt, snap.slot, snap.k_new, snap.v_new, dt)
        ref, _ = getattr(oracle, "attend_" + fmt)(snap.q, k8, v8, ks, vs, snap.bt, snap.seq_lens,
                                                  snap.scale, dt, nthreads=threads)
    spent = time.perf_counter() - t0
    err = float(np.max(np.abs(gpu_rows - ref))) if ref.size else 0.0
    return err, spent, (snap.nbytes if fmt is None else snap.nbytes_q(fmt)) / spent / 1e9, threads


ONE_THREAD_WORKLOADS = ("tiny", "long")


def oracle_sample(w_name, budget_s=12.0, threads=0):
    """The CPU baseline: the oracle timed for about budget_s seconds, on all
    host threads (threads=0) or on `threads`.
    Returns (GB/s, seconds, units, threads, description)."""
    smp = OracleSampler(w_name, threads)
    gbs, spent, done = smp.run(budget_s)
    return gbs, spent, done, smp.threads, smp.describe()


def run_reference(args):
    dist, rank, world, local = (None, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0)
    if rank != 0:
        return 0
    # the whole run (warm-up + timed steps) takes about --ref-budget seconds of
    # oracle time, shared evenly by its steps; each step runs at least one unit
    smp = OracleSampler(args.workload)
    per_step = args.ref_budget / (args.warmup + args.steps)
    vals = []
    for i in range(args.warmup + args.steps):
        gbs, spent, done = smp.run(per_step)
        if i >= args.warmup:
            vals.append((gbs, spent))
    threads, desc = smp.threads, smp.describe()
    gbs = sum(v for v, _ in vals) / len(vals)
    spec = config_spec(args.workload)
    line = {
        "metric": METRIC, "value": round(gbs, 6), "unit": "GB/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(s for _, s in vals) / len(vals), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, **{k: spec[k] for k in ("B", "H_q", "H_kv", "d")},
                   "kv_dtype": spec["dtype"], "sample": "see cpu_baseline"},
        "cpu_baseline": {"value": round(gbs, 6), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(gbs, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU path

# The workloads reported beside the headline one in a default run (workload,
# shared-prefix mode): every synthetic configuration of the method's benchmark.
PER_WORKLOADS = (("tiny", False, None), ("gqa70b", False, None), ("long", False, None),
                 ("cbatch", False, None), ("cbatch", True, None), ("mha7b", False, "fp8"),
                 ("gqa70b", False, "fp8"), ("mha7b", False, "int8"), ("gqa70b", False, "int8"),
                 ("mha7b", False, "int4"), ("gqa70b", False, "int4"), ("cbatch", True, "fp8"),
                 ("cbatch", True, "int8"), ("cbatch", True, "int4"))


def measure_workload(kvd, name, shared_prefix, dev, steps, warmup, fmt=None):
    """Time one workload's decode step through the call the headline uses
    (kvd_decode_step, the shared-prefix call with its fused append, or, with
    fmt "fp8" / "int8" / "int4", kvd_decode_step_{fmt} over the pool
    quantised to that cache) with automatic partitions: `warmup` untimed steps, then
    `steps` calls each bracketed by CUDA events on the launching stream.
    Returns (report dict, RowSnapshot of sampled sequences taken before any
    kernel ran, the GPU's output rows of those sequences as float64)."""
    w = named_config(name, device="cuda", gen_device="cuda")
    si = step_inputs(w, 0)
    snap = RowSnapshot(w, si, sample_sequences(w, 3, 77))
    kc, vc, bt = w.k_cache, w.v_cache, w.block_table.to(dev)
    q8 = None
    if fmt is not None:
        quant = getattr(kvd, "kvd_quantize_" + fmt)
        k8, ks = quant(kc)
        v8, vs = quant(vc)
        q8 = (k8, v8, ks, vs, getattr(kvd, "kvd_decode_step_" + fmt),
              getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt))
    q, k_new, v_new, seq_lens = si["q"], si["k_new"], si["v_new"], si["seq_lens"].to(dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    sp = None
    if shared_prefix:
        per = w.B // w.groups
        sp = {"start": torch.arange(0, w.B + 1, per, dtype=torch.int32, device=dev),
              "pages": torch.full((w.groups,), w.prefix_tokens // 16, dtype=torch.int32, device=dev),
              "max": per}
        n = kvd.kvd_shared_prefix_workspace_size(w.B, w.H_q, w.H_kv, w.d, w.groups, per, 0)
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
    else:
        ws = kvd.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, 0, dev)

    def call(x_q, x_k, x_v, x_len):
        if q8 is not None and sp is not None:
            q8[5](x_q, q8[0], q8[1], q8[2], q8[3], bt, x_len, sp["start"], sp["pages"], sp["max"], w.scale,
                  out=out, k_new=x_k, v_new=x_v, workspace=ws, stream=stream)
        elif q8 is not None:
            q8[4](x_q, x_k, x_v, q8[0], q8[1], q8[2], q8[3], bt, x_len, w.scale, out=out, workspace=ws,
                  stream=stream)
        elif sp is not None:
            kvd.kvd_decode_attention_shared_prefix(x_q, kc, vc, bt, x_len, sp["start"], sp["pages"],
                                                   sp["max"], w.scale, out=out, k_new=x_k, v_new=x_v,
                                                   workspace=ws, stream=stream)
        else:
            kvd.kvd_decode_step(x_q, x_k, x_v, kc, vc, bt, x_len, w.scale, out=out, workspace=ws,
                                stream=stream)

    for _ in range(warmup):
        call(q, k_new, v_new, seq_lens)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for a, b in evs:
        a.record(stream)
        call(q, k_new, v_new, seq_lens)
        b.record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    flags = kvd.kvd_read_device_error()
    gpu_rows = out[snap.rows].float().cpu().double().numpy()
    times = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)
    call_us = sum(times) / len(times)
    step_us = t0.elapsed_time(t1) * 1e3 / steps

    # the HBM bytes count each shared prefix page once per group (members'
    # block tables point at the same physical pages), with or without the
    # shared-prefix call; the logical bytes (every member's own view) beside
    a_b = attention_bytes(w, si["seq_lens"].cpu())
    a_logical = a_b
    if w.groups:
        a_b -= w.groups * (w.B // w.groups - 1) * w.prefix_tokens * w.H_kv * 2 * w.d * 2
    nbytes = a_b + append_bytes(w, si["slot"].cpu())
    if q8 is not None:  # codes + scales read; appended rows read in 16 bits, written as codes + scales
        a_b = quant_attention_bytes(w, si["seq_lens"].cpu(), fmt)
        a_logical = a_b
        if w.groups:
            a_b -= (w.groups * (w.B // w.groups - 1) * w.prefix_tokens * w.H_kv * 2
                    * quant_row_bytes(fmt, w.d))
        nbytes = a_b + quant_append_bytes(w, si["slot"].cpu(), fmt)
    rep = {
        "workload": name + (" --shared-prefix" if shared_prefix else "") + (f" --kv-{fmt}" if fmt else ""),
        "call": (f"kvd_decode_attention_shared_prefix_{fmt} (fused quantising append) over the "
                 f"{QUANT_NAMES[fmt]} cache" if sp is not None and q8 is not None
                 else "kvd_decode_attention_shared_prefix (fused append)" if sp is not None
                 else f"kvd_decode_step_{fmt} over the {QUANT_NAMES[fmt]} cache"
                 if q8 is not None else "kvd_decode_step"),
        "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
        "kv_dtype": w.dtype_name if q8 is None else f"{fmt} codes, {w.dtype_name} q/out",
        "seq_lens": _lens_desc(w), "steps": steps, "warmup": warmup,
        "bytes_per_step": nbytes,
        "us_per_step": round(step_us, 2),
        "timed_call_us": round(call_us, 2),
        "timed_call_us_median": round(times[len(times) // 2], 2),
        "gbs": round(nbytes / (call_us * 1e-6) / 1e9, 2),
        "device_error_flags": flags,
    }
    if w.groups:
        rep["logical_attention_bytes"] = a_logical
    if w.steps > 1:
        # the workload's consecutive steps, each with its own inputs (lengths
        # +1 per step), back to back; one warm pass, then one timed pass
        sets = [step_inputs(w, i, device=dev) for i in range(w.steps)]
        for x in sets:
            call(x["q"], x["k_new"], x["v_new"], x["seq_lens"])
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for x in sets:
            call(x["q"], x["k_new"], x["v_new"], x["seq_lens"])
        c1.record(stream)
        torch.cuda.synchronize()
        rep["consecutive_steps"] = {"steps": w.steps,
                                    "us_per_step": round(c0.elapsed_time(c1) * 1e3 / w.steps, 2)}
        del sets
    rep["fmt"] = fmt
    return rep, snap, gpu_rows


def run_ours(args):
    import kv_cache_decode_scatters_b200 as kvd

    dist, rank, world, local = dist_setup(args.gpus)
    if world != args.gpus and dist is not None:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    # each rank decodes its own batch of the workload (rank 0: the standard one)
    w = named_config(args.workload, device="cuda", gen_device="cuda", scale_down=args.scale_down,
                     shard=rank)
    si = step_inputs(w, 0)
    # the parity sample: host copy of a few sequences' pages before any kernel runs
    snap = None
    if world == 1 and not args.no_cpu_baseline and not args.graph:
        snap = RowSnapshot(w, si, sample_sequences(w, 3, 77))
    kc, vc, bt = w.k_cache, w.v_cache, w.block_table.to(dev)
    q, k_new, v_new = si["q"], si["k_new"], si["v_new"]
    slot, seq_lens = si["slot"].to(dev), si["seq_lens"].to(dev)
    out = torch.empty_like(q)
    ws = kvd.alloc_workspace(w.B, w.H_q, w.H_kv, w.d, args.partitions, dev)
    stream = torch.cuda.current_stream()
    stream0 = stream

    f8 = None
    if args.kv_fp8 or args.kv_int8 or args.kv_int4:
        # the pool stored as codes (E4M3, INT8 or packed INT4) + per-32-channel fp32 scales
        fmt = "fp8" if args.kv_fp8 else "int8" if args.kv_int8 else "int4"
        k8, ks = getattr(kvd, "kvd_quantize_" + fmt)(kc)
        v8, vs = getattr(kvd, "kvd_quantize_" + fmt)(vc)
        f8 = {"fmt": fmt, "k8": k8, "v8": v8, "ks": ks, "vs": vs,
              "append": getattr(kvd, "kvd_append_" + fmt),
              "decode": getattr(kvd, "kvd_decode_attention_" + fmt),
              "step": getattr(kvd, "kvd_decode_step_" + fmt),
              "shared": getattr(kvd, "kvd_decode_attention_shared_prefix_" + fmt),
              "name": QUANT_NAMES[fmt]}

    sp = None
    if args.shared_prefix:
        if not w.groups:
            raise SystemExit("--shared-prefix needs a workload with prefix groups (cbatch)")
        per = w.B // w.groups
        sp = {"start": torch.arange(0, w.B + 1, per, dtype=torch.int32, device=dev),
              "pages": torch.full((w.groups,), w.prefix_tokens // 16, dtype=torch.int32, device=dev),
              "max": per}
        n = kvd.kvd_shared_prefix_workspace_size(w.B, w.H_q, w.H_kv, w.d, w.groups, per, args.partitions)
        ws = torch.empty(n, dtype=torch.uint8, device=dev)

    def step(ev_a=None, ev_b=None):
        if f8 is not None and sp is not None:
            if ev_a is not None:
                ev_a.record(stream)
            f8["shared"](q, f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt, seq_lens, sp["start"], sp["pages"],
                         sp["max"], w.scale, out=out, k_new=k_new, v_new=v_new,
                         num_partitions=args.partitions, workspace=ws, stream=stream)
            if ev_b is not None:
                ev_b.record(stream)
            return
        if f8 is not None and not args.separate_append:
            if ev_a is not None:
                ev_a.record(stream)
            f8["step"](q, k_new, v_new, f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt, seq_lens, w.scale,
                       out=out, num_partitions=args.partitions, workspace=ws, stream=stream)
            if ev_b is not None:
                ev_b.record(stream)
            return
        if f8 is not None:
            f8["append"](f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt, slot, k_new, v_new, stream=stream)
            if ev_a is not None:
                ev_a.record(stream)
            f8["decode"](q, f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt, seq_lens, w.scale, out=out,
                         num_partitions=args.partitions, workspace=ws, stream=stream)
            if ev_b is not None:
                ev_b.record(stream)
            return
        if sp is not None:
            if ev_a is not None:
                ev_a.record(stream)
            kvd.kvd_decode_attention_shared_prefix(q, kc, vc, bt, seq_lens, sp["start"], sp["pages"],
                                                   sp["max"], w.scale, out=out, k_new=k_new,
                                                   v_new=v_new, num_partitions=args.partitions,
                                                   workspace=ws, stream=stream)
            if ev_b is not None:
                ev_b.record(stream)
            return
        if args.separate_append:
            kvd.kvd_append(kc, vc, bt, slot, k_new, v_new, stream=stream)
        if ev_a is not None:
            ev_a.record(stream)
        if args.separate_append:
            kvd.kvd_decode_attention(q, kc, vc, bt, seq_lens, w.scale, out=out,
                                     num_partitions=args.partitions, workspace=ws, stream=stream)
        else:
            kvd.kvd_decode_step(q, k_new, v_new, kc, vc, bt, seq_lens, w.scale, out=out,
                                num_partitions=args.partitions, workspace=ws, stream=stream)
        if ev_b is not None:
            ev_b.record(stream)

    def bytes_of(x):
        """(attention bytes, logical attention bytes, append bytes) of a step.
        With shared prefixes the HBM bytes count each shared page once per
        group (the metric's bytes); the logical bytes (every member's own
        view) are reported beside them."""
        a_b = attention_bytes(w, x["seq_lens"])
        p_b = append_bytes(w, x["slot"])
        kv_tok = w.H_kv * 2 * w.d * 2  # K and V bytes per token of one sequence
        if f8 is not None:
            a_b = quant_attention_bytes(w, x["seq_lens"], f8["fmt"])
            p_b = quant_append_bytes(w, x["slot"], f8["fmt"])
            kv_tok = w.H_kv * 2 * quant_row_bytes(f8["fmt"], w.d)
        a_logical = a_b
        if w.groups:
            a_b -= w.groups * (w.B // w.groups - 1) * w.prefix_tokens * kv_tok
        return a_b, a_logical, p_b

    a_bytes, a_bytes_logical, p_bytes = bytes_of(si)
    step_bytes = a_bytes + p_bytes
    # bytes of the call the roofline times (events bracket it)
    timed_bytes = a_bytes if args.separate_append else step_bytes

    graph = None
    if args.graph:
        # one CUDA graph holding args.graph_steps consecutive steps; timing
        # replays it (launch overhead of the host removed)
        gs = torch.cuda.Stream()
        gs.wait_stream(stream)
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        # consecutive steps with their own inputs where the workload provisions
        # pages for them (continuous batching: lengths grow by one per step),
        # else the same step repeated
        sets = [step_inputs(w, s if s < w.steps else 0, device=dev) for s in range(args.graph_steps)]
        step_bytes = sum(attention_bytes(w, x["seq_lens"].cpu()) + append_bytes(w, x["slot"].cpu())
                         for x in sets) // len(sets)
        timed_bytes = step_bytes
        outs = [torch.empty_like(q) for _ in sets]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gs):
            with torch.cuda.graph(graph, stream=gs):
                for x, o in zip(sets, outs):
                    kvd.kvd_decode_step(x["q"], x["k_new"], x["v_new"], kc, vc, bt, x["seq_lens"],
                                        w.scale, out=o, num_partitions=args.partitions,
                                        workspace=ws, stream=gs)
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all(), "non-finite output"
    assert kvd.kvd_read_device_error() == 0, "device error flagged during warm-up"

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist)
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.__enter__()
    t_start.record(stream)
    if graph is not None:
        for i in range(args.steps):
            evs[i][0].record(stream)
            graph.replay()
            evs[i][1].record(stream)
    else:
        for i in range(args.steps):
            step(*evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if sampler:
        sampler.__exit__(None, None, None)
    barrier(dist)
    head_rows = out[snap.rows].float().cpu().double().numpy() if snap is not None else None
    per = args.graph_steps if graph is not None else 1      # decode steps per timed iteration
    call_median_us = sorted(a.elapsed_time(b) for a, b in evs)[args.steps // 2] * 1e3 / per
    ms_step, attn_ms, value = aggregate(dist, world, args.steps * per, t_start.elapsed_time(t_end),
                                        sum(a.elapsed_time(b) for a, b in evs) / (args.steps * per),
                                        step_bytes)

    def run_step(x, st=None):
        """One step of the selected mode on the inputs x (q, k_new, v_new,
        seq_lens and, for the two-call paths, slot), on stream st (default:
        the bench's stream)."""
        stream = st if st is not None else stream0
        if f8 is not None and sp is not None:
            f8["shared"](x["q"], f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt, x["seq_lens"], sp["start"],
                         sp["pages"], sp["max"], w.scale, out=out, k_new=x["k_new"], v_new=x["v_new"],
                         num_partitions=args.partitions, workspace=ws, stream=stream)
        elif f8 is not None and not args.separate_append:
            f8["step"](x["q"], x["k_new"], x["v_new"], f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt,
                       x["seq_lens"], w.scale, out=out, num_partitions=args.partitions, workspace=ws,
                       stream=stream)
        elif f8 is not None:
            f8["append"](f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt, x["slot"], x["k_new"], x["v_new"],
                         stream=stream)
            f8["decode"](x["q"], f8["k8"], f8["v8"], f8["ks"], f8["vs"], bt, x["seq_lens"], w.scale,
                         out=out, num_partitions=args.partitions, workspace=ws, stream=stream)
        elif sp is not None:
            kvd.kvd_decode_attention_shared_prefix(x["q"], kc, vc, bt, x["seq_lens"], sp["start"],
                                                   sp["pages"], sp["max"], w.scale, out=out,
                                                   k_new=x["k_new"], v_new=x["v_new"],
                                                   num_partitions=args.partitions, workspace=ws,
                                                   stream=stream)
        elif args.separate_append:
            kvd.kvd_append(kc, vc, bt, x["slot"], x["k_new"], x["v_new"], stream=stream)
            kvd.kvd_decode_attention(x["q"], kc, vc, bt, x["seq_lens"], w.scale, out=out,
                                     num_partitions=args.partitions, workspace=ws, stream=stream)
        else:
            kvd.kvd_decode_step(x["q"], x["k_new"], x["v_new"], kc, vc, bt, x["seq_lens"], w.scale,
                                out=out, num_partitions=args.partitions, workspace=ws, stream=stream)

    # ---- a workload's consecutive steps (continuous batching: every length
    # grows by one per step), each with its own inputs, back to back
    multi = None
    if w.steps > 1 and graph is None:
        sets = [step_inputs(w, s, device=dev) for s in range(w.steps)]
        for x in sets:
            run_step(x)
        reps = 5
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        m0.record(stream)
        for _ in range(reps):
            for x in sets:
                run_step(x)
        m1.record(stream)
        torch.cuda.synchronize()
        tot_ms = m0.elapsed_time(m1) / reps
        nb = sum(sum(bytes_of({k: v.cpu() for k, v in x.items()})[::2]) for x in sets)
        multi = {"steps": w.steps, "total_us": round(tot_ms * 1e3, 2),
                 "us_per_step": round(tot_ms * 1e3 / w.steps, 2),
                 "gbs": round(nb / (tot_ms * 1e-3) / 1e9, 2), "repeats": reps,
                 "how": "the workload's consecutive steps (lengths +1 per step, own inputs), "
                        "back to back on one stream, CUDA events; mean over the repeats"}
        del sets

    # ---- end to end through the public API with pinned host buffers
    inputs = [("q", q), ("k_new", k_new), ("v_new", v_new), ("seq_lens", seq_lens)]
    if args.separate_append:
        inputs.append(("slot", slot))
    # a step's inputs sit in one pinned staging buffer, copied by one H2D copy
    # into one device buffer (each input a 256-byte aligned view of it)
    offs, total = [], 0
    for _, t in inputs:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_buf = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    d_buf = torch.empty(total, dtype=torch.uint8, device=dev)

    def views(buf):
        return {n: buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                for (n, t), o in zip(inputs, offs)}

    h_in, d_in = views(h_buf), views(d_buf)
    for n, t in inputs:
        h_in[n].copy_(t.cpu())
    h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = total                      # bytes of the one H2D copy (inputs + alignment padding)
    d2h = h_out.numel() * h_out.element_size()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))

    def e2e_step():
        d_buf.copy_(h_buf, non_blocking=True)
        run_step(d_in)
        h_out.copy_(out, non_blocking=True)
        stream.synchronize()

    def e2e_time(fn):
        for _ in range(3):
            fn()
        barrier(dist)
        t0 = time.perf_counter()
        for _ in range(e2e_steps):
            fn()
        e2e_s = max_over_ranks(dist, time.perf_counter() - t0)
        barrier(dist)
        return e2e_s

    e2e_eager_s = e2e_time(e2e_step)
    # the same step as one CUDA graph: the H2D copy of the step's inputs from
    # the pinned buffer, the library call, the D2H copy of out; each step
    # replays it and waits for it (a decode loop refills h_buf between steps)
    e2e_graph_s, e2e_graph_err = None, None
    try:
        gstream = torch.cuda.Stream()
        gstream.wait_stream(stream)
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(gstream):
            run_step(d_in, gstream)          # warm this stream once outside the capture
            gstream.synchronize()
            with torch.cuda.graph(e2e_graph, stream=gstream):
                d_buf.copy_(h_buf, non_blocking=True)
                run_step(d_in, gstream)
                h_out.copy_(out, non_blocking=True)
        torch.cuda.synchronize()

        def e2e_graph_step():
            e2e_graph.replay()
            stream.synchronize()

        with torch.cuda.stream(stream):
            e2e_graph_s = e2e_time(e2e_graph_step)
    except Exception as exc:  # capture unsupported for this mode: report the eager figure only
        e2e_graph_err = f"{type(exc).__name__}: {exc}"[:200]
    e2e_s = e2e_graph_s if e2e_graph_s is not None else e2e_eager_s
    e2e_val = world * step_bytes * e2e_steps / e2e_s / 1e9
    e2e_eager_val = world * step_bytes * e2e_steps / e2e_eager_s / 1e9

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    # ---- every other configuration of the benchmark, through the same call
    per_wl = []
    default_run = (args.workload == "mha7b" and f8 is None and sp is None and not args.separate_append
                   and graph is None and args.scale_down == 1)
    if world == 1 and (args.per_workload == "on" or (args.per_workload == "auto" and default_run)):
        for name, shared, fmt in PER_WORKLOADS:
            per_wl.append(measure_workload(kvd, name, shared, dev, args.per_workload_steps, 5, fmt))
            torch.cuda.empty_cache()

    peak, peak_kind = peaks()
    achieved = timed_bytes / (attn_ms * 1e-3) / 1e9
    read_peaks = read_only_peak_gbs(kvd)
    read_peak = max(read_peaks.values())
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        gbs, spent, done, threads, desc = oracle_sample(args.workload, budget_s=args.cpu_budget)
        cpu = {"value": round(gbs, 6), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": desc}
        if args.workload in ONE_THREAD_WORKLOADS:
            # the single-thread figure of the smallest and the longest shapes
            g1, _, _, _, d1 = oracle_sample(args.workload, budget_s=args.cpu_budget / 3, threads=1)
            cpu["one_thread"] = {"value": round(g1, 6), "unit": "GB/s", "cores": 1, "sample": d1}
    # ---- parity of the timed call against the oracle (CPU-baseline leg)
    tol = 1e-2 if w.dtype == torch.bfloat16 else 2e-3
    parity = None
    if snap is not None:
        err, spent, ogbs, othr = oracle_parity(snap, head_rows, fmt=f8["fmt"] if f8 else None)
        parity = {"max_abs_err": err, "tol": tol, "ok": err <= tol, "sample": snap.describe(w),
                  "against": "fp64 oracle" + (" over the oracle's own %s quantisation" % f8["name"]
                                               if f8 else "")}
    per_report = []
    for rep, psnap, prows in per_wl:
        ptol = 1e-2 if psnap.bf16 else 2e-3
        perr, pspent, pgbs, pthr = oracle_parity(psnap, prows, fmt=rep["fmt"])
        ach = rep["bytes_per_step"] / (rep["timed_call_us"] * 1e-6) / 1e9
        rep["roofline"] = {"achieved": round(ach, 2), "frac": round(ach / peak, 4),
                           "frac_of_read_only_peak": round(ach / read_peak, 4)}
        rep["max_abs_err"] = perr
        rep["tol"] = ptol
        rep["parity_ok"] = perr <= ptol
        rep["parity_sample"] = psnap.describe_short()
        rep["cpu_baseline"] = {"value": round(pgbs, 4), "unit": "GB/s", "cores": pthr, "kind": "oracle",
                               "sample": "append + attend of the parity sample, one run"}
        per_report.append(rep)
    clocks = sampler.summary() if sampler else None
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": (f8["fmt"] + " cache, " + w.dtype_name + " q/out") if f8 is not None else w.dtype_name,
        "data": "synthetic",
        "config": {
            "workload": w.name if args.scale_down == 1 else f"{w.name}/scale_down={args.scale_down}",
            "B": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "d": w.d,
            "seq_lens": _lens_desc(w), "page_tokens": 16, "pages_in_pool": w.num_blocks,
            "placement": "shuffled pages", "partitions": args.partitions or kvd.kvd_auto_partitions(),
            "bytes_per_step": step_bytes, "attention_bytes": a_bytes, "append_bytes": p_bytes,
            "l2": "inputs larger than L2 (KV pool %.2f GB >> 126 MB); no flush" % (
                2 * w.k_cache.numel() * 2 / 1e9),
            "step": ("kvd_decode_attention_shared_prefix_%s with fused quantising append over an %s "
                     "cache (plan, decode, prefix tensor-core pass with dequantised tiles beside it, merge kernels)"
                     % (f8["fmt"], f8["name"]) if f8 is not None and sp is not None else
                     "kvd_append_%s + kvd_decode_attention_%s over an %s cache "
                     "(quantising append, decode, merge kernels)" % (f8["fmt"], f8["fmt"], f8["name"])
                     if f8 is not None and args.separate_append else
                     "kvd_decode_step_%s over an %s cache (decode kernel with fused quantising "
                     "append, merge kernel)" % (f8["fmt"], f8["name"])
                     if f8 is not None else
                     "kvd_decode_attention_shared_prefix with fused append (plan, decode, prefix pass beside it, "
                     "merge kernels)"
                     if sp is not None else
                     "kvd_append + kvd_decode_attention (append, decode, merge kernels)"
                     if args.separate_append else
                     "kvd_decode_step (decode kernel with fused append, merge kernel)"),
        },
        "us_per_step": round(ms_step * 1e3, 2),
        "timed_call_us": round(attn_ms * 1e3, 2),
        "timed_call_us_median": round(call_median_us, 2),
        "consecutive_steps": multi,
        "roofline": {
            "bound": "hbm",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "peak_kind": peak_kind,
            "kernel": ("kvd_decode_attention_shared_prefix_%s call (prefix_plan_kernel + decode_kernel over "
                       "%s pages with fused quantising append + prefix_tcq_kernel + merge)"
                       % (f8["fmt"], f8["name"])
                       if f8 is not None and sp is not None else
                       "kvd_decode_attention_%s call (decode_kernel over %s pages + merge)"
                       % (f8["fmt"], f8["name"]) if f8 is not None and args.separate_append else
                       "kvd_decode_step_%s call (decode_kernel over %s pages with fused quantising "
                       "append + merge)" % (f8["fmt"], f8["name"]) if f8 is not None else
                       "kvd_decode_attention_shared_prefix call (prefix_plan_kernel + decode_kernel with "
                       "fused append + prefix_tc_kernel + merge)" if sp is not None else
                       "kvd_decode_attention call (decode_kernel + decode_merge_kernel)"
                       if args.separate_append else
                       "kvd_decode_step call (decode_kernel with fused append + decode_merge_kernel)")
                      + ", CUDA events on the launching stream; achieved = its algorithmic bytes / mean duration",
            "bytes_per_launch": timed_bytes,
            "traffic": profile_traffic(w.name, (f8["fmt"] + ("_shared_prefix" if sp is not None else
                                                             "_separate_append" if args.separate_append
                                                             else ""))
                                      if f8 is not None else "shared_prefix" if sp is not None
                                      else "separate_append" if args.separate_append else "fused"),
        },
        "frac_of_8000_spec": round(achieved / 8000.0, 4),
        "shared_prefix": ({"logical_attention_bytes": a_bytes_logical,
                           "value_logical_gbs": round(
                               world * (step_bytes + a_bytes_logical - a_bytes) / (ms_step * 1e-3) / 1e9, 2),
                           "achieved_logical_gbs": round(
                               (timed_bytes + a_bytes_logical - a_bytes) / (attn_ms * 1e-3) / 1e9, 2),
                           "note": ("value, roofline and e2e count each shared prefix page once per "
                                    "group; the logical figures count it once per member")}
                          if w.groups else None),
        "read_only_peak": {"value": round(read_peak, 1), "unit": "GB/s",
                           "frac": round(achieved / read_peak, 4),
                           "forms": {k: round(v, 1) for k, v in read_peaks.items()},
                           "how": "kvd_read_stream over 4 GiB (vector: 16-byte loads; bulk: the decode "
                                  "kernel's 16-warp bulk-copy pipeline with no arithmetic), best of 5 "
                                  "each, CUDA events, this run; value = the faster form"},
        "parity": parity,
        "per_workload": per_report or None,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "us_per_step": round(e2e_s / e2e_steps * 1e6, 2),
                "mode": "cuda graph" if e2e_graph_s is not None else "eager",
                "eager": {"value": round(e2e_eager_val, 2), "unit": "GB/s",
                          "us_per_step": round(e2e_eager_s / e2e_steps * 1e6, 2)},
                "graph_error": e2e_graph_err,
                "how": "per step: the step's inputs in one pinned host buffer -> one H2D copy, the "
                       "timed call, D2H of out, stream sync; wall clock, max over ranks.  mode "
                       "'cuda graph': those three captured once as a CUDA graph and replayed each "
                       "step (eager: issued from Python each step)"},
        "gpu_launches": (4 if sp is not None else 3 if args.separate_append else 2) * args.steps * per,
        "graph": ({"steps_per_graph": args.graph_steps, "replays": args.steps} if graph is not None
                  else None),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def _lens_desc(w):
    l = w.seq_lens0
    if bool((l == l[0]).all()):
        return int(l[0])
    return {"min": int(l.min()), "max": int(l.max()), "mean": round(float(l.float().mean()), 1)}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="mha7b",
                   choices=["tiny", "mha7b", "gqa70b", "long", "cbatch"])
    p.add_argument("--partitions", type=int, default=0, help="0 = automatic")
    p.add_argument("--separate-append", action="store_true",
                   help="time kvd_append[_fp8|_int8|_int4] + kvd_decode_attention[_fp8|_int8|_int4] "
                        "instead of the fused kvd_decode_step[_fp8|_int8|_int4]")
    p.add_argument("--e2e-steps", type=int, default=300)
    p.add_argument("--kv-fp8", action="store_true",
                   help="store the cache as FP8 E4M3 codes with per-32-channel scales (d=128)")
    p.add_argument("--kv-int8", action="store_true",
                   help="store the cache as INT8 codes with per-32-channel scales (d=128)")
    p.add_argument("--kv-int4", action="store_true",
                   help="store the cache as packed INT4 codes with per-32-channel scales (d=128)")
    p.add_argument("--shared-prefix", action="store_true",
                   help="read each group's shared prefix pages once (kvd_decode_attention_shared_prefix)")
    p.add_argument("--graph", action="store_true",
                   help="capture --graph-steps fused steps in one CUDA graph and time its replays")
    p.add_argument("--graph-steps", type=int, default=16)
    p.add_argument("--cpu-budget", type=float, default=12.0,
                   help="seconds of oracle work for the CPU baseline sample")
    p.add_argument("--ref-budget", type=float, default=90.0,
                   help="seconds of oracle work for the whole reference-arm run")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--per-workload", choices=["auto", "on", "off"], default="auto",
                   help="also time (and parity-check) every other configuration; auto = only in the "
                        "default single-GPU run")
    p.add_argument("--per-workload-steps", type=int, default=50)
    p.add_argument("--scale-down", type=int, default=1,
                   help="shrink batch and lengths by this factor (profiling small cases only)")
    args = p.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.graph and (args.separate_append or args.shared_prefix or args.kv_fp8 or args.kv_int8
                       or args.kv_int4):
        raise SystemExit("--graph times the fused step only")
    if args.kv_fp8 + args.kv_int8 + args.kv_int4 > 1:
        raise SystemExit("--kv-fp8, --kv-int8 and --kv-int4 are exclusive")
    if args.shared_prefix and args.separate_append:
        raise SystemExit("--shared-prefix always fuses the append")
    return args


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

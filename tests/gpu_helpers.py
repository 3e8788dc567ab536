"""Shared pieces of the GPU parity tests: run one decode step through the
C-ABI (via the Python binding) and through the oracle on the same inputs."""
import numpy as np
import torch

import oracle
from synth import build_workload, step_inputs, to_words

TOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}   # max-abs error vs the fp64 oracle
LSE_TOL = 1e-3

# (workload, call, rows checked, max-abs error, lse error, tolerance) of the
# full-size parity tests; the session prints them (see conftest.py)
ERROR_REPORT = []


def record_error(workload, call, rows, err, lse_err, tol):
    ERROR_REPORT.append((workload, call, rows, err, lse_err, tol))


def odt(w):
    return oracle.BF16 if w.dtype == torch.bfloat16 else oracle.F16


def gpu_state(w):
    """Device copies of the workload's pool and block table."""
    return (w.k_cache.cuda().clone(), w.v_cache.cuda().clone(), w.block_table.cuda())


def gpu_step(kvd, w, si, kc, vc, bt, num_partitions=0, with_lse=True, out=None):
    q = si["q"].cuda()
    kvd.kvd_append(kc, vc, bt, si["slot"].cuda(), si["k_new"].cuda(), si["v_new"].cuda())
    lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device="cuda") if with_lse else None
    out = kvd.kvd_decode_attention(q, kc, vc, bt, si["seq_lens"].cuda(), w.scale, out=out,
                                   num_partitions=num_partitions, lse_out=lse)
    torch.cuda.synchronize()
    return out, lse


def oracle_step(w, si, kc_words=None, vc_words=None, rows=None):
    """Oracle append + attend.  rows: optional list of sequence indices to
    attend (others are skipped); returns dict b -> (out [H_q,d], lse [H_q])."""
    kc = to_words(w.k_cache).copy() if kc_words is None else kc_words
    vc = to_words(w.v_cache).copy() if vc_words is None else vc_words
    bt = w.block_table.numpy()
    oracle.append(kc, vc, bt, si["slot"].cpu().numpy(), to_words(si["k_new"]), to_words(si["v_new"]))
    q = to_words(si["q"])
    sl = si["seq_lens"].cpu().numpy()
    if rows is None:
        out, lse = oracle.attend(q, kc, vc, bt, sl, w.scale, odt(w))
        return kc, vc, {b: (out[b], lse[b]) for b in range(w.B)}
    res = {}
    for b in rows:
        o, l = oracle.attend(q[b:b + 1], kc, vc, bt[b:b + 1], sl[b:b + 1], w.scale, odt(w))
        res[b] = (o[0], l[0])
    return kc, vc, res


def host(t):
    """Device tensor -> numpy copy; 8-bit codes as their bytes (uint8)."""
    a = t.cpu().numpy().copy()
    return a.view(np.uint8) if a.dtype == np.int8 else a


def oracle_q8(w, fmt, si=None):
    """The oracle's own 8-bit pools: its quantisation of the workload's whole
    16-bit pool and, with step inputs si, its quantising append of the step's
    rows -- no input from the GPU."""
    k8, ks = getattr(oracle, "quantize_" + fmt)(to_words(w.k_cache), odt(w))
    v8, vs = getattr(oracle, "quantize_" + fmt)(to_words(w.v_cache), odt(w))
    if si is not None:
        getattr(oracle, "append_" + fmt)(k8, v8, ks, vs, w.block_table.numpy(), si["slot"].cpu().numpy(),
                              to_words(si["k_new"]), to_words(si["v_new"]), odt(w))
    return k8, v8, ks, vs


def oracle_q8_rows(w, fmt, si, rows):
    """oracle_q8 for a few sequences of a large workload: only the pages
    they use, renumbered (returns the pools, their block table and the page
    list, so the GPU's pools can be compared page for page)."""
    bt = w.block_table.cpu()
    n = si["seq_lens"].cpu()
    npg = [(int(n[b]) + 15) // 16 for b in rows]
    pages = sorted({int(p) for b, m in zip(rows, npg) for p in bt[b, :m].tolist()})
    remap = {p: i for i, p in enumerate(pages)}
    bts = np.zeros((len(rows), max(npg)), dtype=np.int32)
    for i, (b, m) in enumerate(zip(rows, npg)):
        bts[i, :m] = [remap[p] for p in bt[b, :m].tolist()]
    idx = torch.tensor(pages, dtype=torch.long, device=w.k_cache.device)
    kw, vw = to_words(w.k_cache.index_select(0, idx)), to_words(w.v_cache.index_select(0, idx))
    k8, ks = getattr(oracle, "quantize_" + fmt)(kw, odt(w))
    v8, vs = getattr(oracle, "quantize_" + fmt)(vw, odt(w))
    sel = torch.tensor(rows, dtype=torch.long)
    getattr(oracle, "append_" + fmt)(k8, v8, ks, vs, bts, si["slot"].cpu()[sel].numpy(),
                          to_words(si["k_new"].cpu()[sel]), to_words(si["v_new"].cpu()[sel]), odt(w))
    return (k8, v8, ks, vs), bts, pages


def data_rows(k_cache, v_cache, block_table=None, si=None):
    """Bool [NB, H_kv, 16]: pool rows holding data -- rows of the 16-bit pool
    that are not the NaN canary of never-written slots, plus the rows the
    step appends.  The canary's 8-bit encoding (which NaN code, which NaN
    scale) is a convention nothing reads, so pools are compared on these."""
    m = (torch.isfinite(k_cache.float()).all(-1) & torch.isfinite(v_cache.float()).all(-1)).cpu().numpy()
    if si is not None:
        slot = si["slot"].cpu().numpy()
        bt = block_table.cpu().numpy() if torch.is_tensor(block_table) else block_table
        for b, pos in enumerate(slot):
            if pos >= 0:
                m[bt[b, pos // 16], :, pos % 16] = True
    return m


def assert_pools_equal(gpu, orc, rows):
    """8-bit codes and fp32 scales, bit for bit, on the rows holding data."""
    for g, o in zip(gpu, orc):
        g = host(g) if torch.is_tensor(g) else g
        if g.dtype == np.float32:
            g, o = g.view(np.uint32), o.view(np.uint32)
        assert np.array_equal(g[rows], o[rows])




def max_err(gpu_out, ref, rows=None):
    g = gpu_out.float().cpu().double().numpy()
    errs = []
    for b, (o, _) in ref.items():
        if rows is not None and b not in rows:
            continue
        errs.append(np.max(np.abs(g[b] - o)) if o.size else 0.0)
    return float(max(errs)) if errs else 0.0


def max_lse_err(gpu_lse, ref):
    g = gpu_lse.cpu().double().numpy()
    errs = []
    for b, (_, l) in ref.items():
        fin = np.isfinite(l)
        assert np.array_equal(np.isfinite(g[b]), fin), "lse finiteness differs"
        if fin.any():
            errs.append(np.max(np.abs(g[b][fin] - l[fin])))
    return float(max(errs)) if errs else 0.0


def assert_out_close(gpu_out, ref, dtype):
    """out within TOL[dtype] (max-abs) of the fp64 oracle wherever a value of
    the output dtype can be that close.  Where |ref| is so large that half an
    ulp of the dtype exceeds TOL (bf16 from |ref| >= 2.56: half an ulp is
    1/256 of the value), even the correctly rounded output misses the
    absolute bound, so there the output must be within one ulp of ref.
    Returns the max abs error over all outputs."""
    g = gpu_out.float().cpu().double().numpy() if torch.is_tensor(gpu_out) else gpu_out
    err = np.abs(g - ref)
    mant = 8 if dtype == torch.bfloat16 else 11               # significant bits
    mag = np.abs(ref)
    ulp = np.exp2(np.floor(np.log2(np.maximum(mag, 2.0 ** -14))) - (mant - 1))
    near = ulp / 2 <= TOL[dtype]
    if near.any():
        assert float(err[near].max()) <= TOL[dtype], f"max abs error {float(err[near].max())}"
    if (~near).any():
        worst = float((err[~near] / ulp[~near]).max())
        assert worst <= 1.0, f"error of {worst} ulp where |out| >= {float(mag[~near].min())}"
    return float(err.max()) if err.size else 0.0


def uneven_groups_case(d, dtype, H_q, H_kv, seed):
    """Groups of different sizes and shared page counts, made by pointing
    each member's first pages at its group's first member's pages."""
    sizes = [5, 40, 1, 3, 7]
    gpages = [4, 10, 2, 0, 6]
    rng = np.random.default_rng(seed)
    lens, starts = [], [0]
    for sz, gp in zip(sizes, gpages):
        for i in range(sz):
            lens.append(int(gp * 16 + 1 + rng.integers(0, 90)))
        starts.append(starts[-1] + sz)
    lens[starts[1] + 3] = 10 * 16      # exactly the shared prefix: no private page
    lens[starts[4] + 2] = 40           # shorter than its group's 6 shared pages
    w = build_workload("spu", len(lens), H_q, H_kv, d, dtype, lens, seed=seed, spare_pages=4)
    bt2 = w.block_table.clone()
    for g, gp in enumerate(gpages):
        s0, s1 = starts[g], starts[g + 1]
        for b in range(s0 + 1, s1):
            bt2[b, :gp] = w.block_table[s0, :gp]
    gs = torch.tensor(starts, dtype=torch.int32)
    gpg = torch.tensor(gpages, dtype=torch.int32)
    return w, bt2, gs, gpg, max(sizes)


def words(t):
    return to_words(t)


__all__ = ["TOL", "LSE_TOL", "ERROR_REPORT", "record_error", "assert_out_close", "uneven_groups_case", "host", "oracle_q8", "oracle_q8_rows",
           "data_rows", "assert_pools_equal", "odt", "gpu_state", "gpu_step", "oracle_step", "max_err", "max_lse_err",
           "words", "step_inputs"]

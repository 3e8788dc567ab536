"""Shared pieces of the GPU parity tests: run one decode step through the
C-ABI (via the Python binding) and through the oracle on the same inputs."""
import numpy as np
import torch

import oracle
from synth import step_inputs, to_words

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


def words(t):
    return to_words(t)


__all__ = ["TOL", "LSE_TOL", "ERROR_REPORT", "record_error", "gpu_state", "gpu_step", "oracle_step", "max_err", "max_lse_err",
           "words", "step_inputs"]

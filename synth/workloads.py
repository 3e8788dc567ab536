"""Seeded synthetic workloads for one paged-KV decode step.

Layout conventions (the ones the library's C interface documents):
  k_cache, v_cache : [num_blocks, H_kv, 16, d]  fp16 / bf16 (the physical pool)
  block_table      : int32 [B, max_blocks]      logical page -> physical page
  seq_lens         : int32 [B]                  tokens attended, including the
                                                token appended in the same step
  slot             : int32 [B]                  logical position of the new token
  q                : [B, H_q, d];  k_new, v_new : [B, H_kv, d]

Value recipe: every K, V, q, k_new, v_new value is drawn as float32 N(0, 1)
from a torch.Generator seeded per workload, optionally scaled (key outlier
channels), then rounded once to the storage dtype.  Token slots of the pool
that no sequence has written yet (the slot the step will append into, page
tails, spare pages) hold the canary word 0xFFFF, a NaN in fp16 and bf16, so a
kernel that reads them pollutes its output visibly.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

PAGE_TOKENS = 16
CANARY_WORD = 0xFFFF

_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


def to_words(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit storage words of an fp16/bf16 tensor, as a numpy uint16 array."""
    assert t.dtype in (torch.float16, torch.bfloat16)
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@dataclass
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    d: int
    dtype: torch.dtype
    scale: float
    seq_lens0: torch.Tensor          # int32 [B] lengths at step 0 (incl. its appended token)
    block_table: torch.Tensor        # int32 [B, max_blocks]
    k_cache: torch.Tensor            # [NB, H_kv, 16, d] state before the step-0 append
    v_cache: torch.Tensor
    steps: int
    seed: int
    outlier_channels: list = field(default_factory=list)   # (head, dim) pairs scaled in K
    outlier_scale: float = 1.0
    prefix_tokens: int = 0
    groups: int = 0
    device: str = "cpu"
    gen_device: str = "cpu"

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def dtype_name(self) -> str:
        return "bf16" if self.dtype == torch.bfloat16 else "f16"

    def seq_lens_at(self, step: int) -> torch.Tensor:
        s = self.seq_lens0.clone()
        s[s > 0] += step
        return s


def _gen(seed: int, device: str) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, gen_device, out_device, dtype, outliers=None, outlier_scale=1.0,
           head_axis=None, dim_axis=None):
    x = torch.randn(shape, generator=g, device=gen_device, dtype=torch.float32)
    if outliers:
        for (h, dd) in outliers:
            idx = [slice(None)] * len(shape)
            idx[head_axis] = h
            idx[dim_axis] = dd
            x[tuple(idx)] *= outlier_scale
    return x.to(dtype).to(out_device)


def build_workload(name, B, H_q, H_kv, d, dtype, seq_lens, *, seed, steps=1,
                   placement="shuffle", spare_pages=0, outlier_frac=0.0,
                   outlier_scale=20.0, prefix_groups=0, prefix_tokens=0, scale=None,
                   device="cpu", gen_device=None, max_blocks=None,
                   chunk_pages=4096) -> Workload:
    """Build the paged pool and block table for a decode workload.

    seq_lens: step-0 lengths (each includes the token appended at step 0);
      a length of 0 means the sequence is idle (no append, empty attention).
    placement: "shuffle" places pages by a seeded permutation of the pool,
      "identity" hands out physical pages in logical order.
    prefix_groups / prefix_tokens: sequences are split into prefix_groups
      equal groups whose members map their first prefix_tokens tokens
      (a whole number of pages) onto the same physical pages.
    steps: pages are provisioned for steps consecutive appends.
    """
    if isinstance(dtype, str):
        dtype = _DTYPES[dtype]
    gen_device = gen_device or device
    sl = torch.as_tensor(seq_lens, dtype=torch.int64).cpu()
    assert sl.numel() == B and (sl >= 0).all()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    g_host = _gen(seed, "cpu")

    # ---- page accounting
    final_len = torch.where(sl > 0, sl + (steps - 1), sl)
    need = (final_len + PAGE_TOKENS - 1) // PAGE_TOKENS
    pp = 0
    group_of = [None] * B
    if prefix_groups:
        assert prefix_tokens % PAGE_TOKENS == 0 and B % prefix_groups == 0
        pp = prefix_tokens // PAGE_TOKENS
        per = B // prefix_groups
        for b in range(B):
            assert sl[b] >= prefix_tokens + 1, "shared-prefix members must extend the prefix"
            group_of[b] = b // per
    shared_total = prefix_groups * pp
    private_need = [int(need[b]) - (pp if group_of[b] is not None else 0) for b in range(B)]
    total = shared_total + sum(private_need)
    NB = max(1, total + spare_pages)
    if placement == "shuffle":
        ids = torch.randperm(NB, generator=g_host).to(torch.int32)
    elif placement == "identity":
        ids = torch.arange(NB, dtype=torch.int32)
    else:
        raise ValueError(placement)
    mb = int(need.max()) if B else 1
    mb = max(mb, 1)
    if max_blocks is not None:
        assert max_blocks >= mb
        mb = max_blocks
    bt = torch.full((B, mb), -1, dtype=torch.int32)
    ptr = 0
    shared = []
    for gi in range(prefix_groups):
        shared.append(ids[ptr:ptr + pp])
        ptr += pp
    for b in range(B):
        col = 0
        if group_of[b] is not None:
            bt[b, :pp] = shared[group_of[b]]
            col = pp
        k = private_need[b]
        bt[b, col:col + k] = ids[ptr:ptr + k]
        ptr += k

    # ---- outlier channels (K only), chosen from the H_kv * d channels
    outliers = []
    if outlier_frac > 0:
        n_out = max(1, int(round(outlier_frac * H_kv * d)))
        pick = torch.randperm(H_kv * d, generator=g_host)[:n_out].tolist()
        outliers = sorted((c // d, c % d) for c in pick)

    # ---- pool values, generated chunk by chunk of pages
    g = _gen(seed * 2 + 1, gen_device)
    k_cache = torch.empty((NB, H_kv, PAGE_TOKENS, d), dtype=dtype, device=device)
    v_cache = torch.empty_like(k_cache)
    for c0 in range(0, NB, chunk_pages):
        c1 = min(NB, c0 + chunk_pages)
        shp = (c1 - c0, H_kv, PAGE_TOKENS, d)
        k_cache[c0:c1] = _randn(shp, g, gen_device, device, dtype, outliers, outlier_scale, 1, 3)
        v_cache[c0:c1] = _randn(shp, g, gen_device, device, dtype)

    # ---- canary every token slot that holds no written token yet
    written = torch.zeros((NB, PAGE_TOKENS), dtype=torch.bool)
    for b in range(B):
        n_written = int(sl[b]) - 1 if sl[b] > 0 else 0      # step 0 appends position n-1
        if n_written <= 0:
            continue
        full = n_written // PAGE_TOKENS
        if full:
            written[bt[b, :full].long()] = True
        rem = n_written % PAGE_TOKENS
        if rem:
            written[int(bt[b, full]), :rem] = True
    free = (~written).nonzero(as_tuple=False)
    if free.numel():
        kw = k_cache.view(torch.int16)
        vw = v_cache.view(torch.int16)
        pages = free[:, 0].to(device)
        toks = free[:, 1].to(device)
        canary = torch.tensor(CANARY_WORD, dtype=torch.int32).to(torch.int16).item()
        kw[pages, :, toks, :] = canary
        vw[pages, :, toks, :] = canary

    return Workload(name=name, B=B, H_q=H_q, H_kv=H_kv, d=d, dtype=dtype, scale=float(scale),
                    seq_lens0=sl.to(torch.int32), block_table=bt, k_cache=k_cache,
                    v_cache=v_cache, steps=steps, seed=seed, outlier_channels=outliers,
                    outlier_scale=outlier_scale if outliers else 1.0,
                    prefix_tokens=prefix_tokens if prefix_groups else 0,
                    groups=prefix_groups, device=device, gen_device=gen_device)


def step_inputs(w: Workload, step: int = 0, device=None):
    """q, k_new, v_new, slot and seq_lens for decode step `step` of workload w."""
    device = device or w.device
    g = _gen(w.seed * 7919 + 104729 * (step + 1), w.gen_device)
    q = _randn((w.B, w.H_q, w.d), g, w.gen_device, device, w.dtype)
    k_new = _randn((w.B, w.H_kv, w.d), g, w.gen_device, device, w.dtype,
                   w.outlier_channels, w.outlier_scale, 1, 2)
    v_new = _randn((w.B, w.H_kv, w.d), g, w.gen_device, device, w.dtype)
    n = w.seq_lens_at(step)
    slot = torch.where(n > 0, n - 1, torch.full_like(n, -1)).to(torch.int32)
    return {"q": q, "k_new": k_new, "v_new": v_new,
            "slot": slot.to(device), "seq_lens": n.to(torch.int32).to(device)}


# --------------------------------------------------------------- named configs

def _lognormal_suffix(B, g, median=1000.0, sigma=1.0):
    x = torch.empty(B, dtype=torch.float64).log_normal_(mean=math.log(median), std=sigma, generator=g)
    return torch.round(x).to(torch.int64)


def config_spec(name: str, scale_down: int = 1, shard: int = 0) -> dict:
    """Shapes, lengths and build options of a named workload (no pool).

    The five synthetic decode workloads of this method's benchmark; seeds are
    1000 + config index.  scale_down > 1 shrinks batch and lengths with the
    same structure, for quick tests.  shard > 0 draws another batch of the
    same workload (other seeds), e.g. the sequences of another GPU.
    """
    s = max(1, int(scale_down))
    spec = _config_spec(name, s)
    if shard:
        off = 7919 * int(shard)
        spec["seed"] += off
        if name in ("gqa70b", "cbatch"):
            spec = _config_spec(name, s, seed_offset=off)
            spec["seed"] += off
    return spec


def _config_spec(name: str, s: int, seed_offset: int = 0) -> dict:
    if name == "tiny":
        # 1 sequence, 8 heads, d=64, fp16, 1023 cached + 1 appended = 1024
        # tokens on pages 0..63 in order.
        return dict(B=1, H_q=8, H_kv=8, d=64, dtype="f16", lens=[max(1, 1024 // s)], seed=1001,
                    opts=dict(placement="identity"))
    if name == "mha7b":
        B = max(1, 32 // s)
        return dict(B=B, H_q=32, H_kv=32, d=128, dtype="f16", lens=[max(1, 4096 // s)] * B,
                    seed=1002, opts=dict(placement="shuffle"))
    if name == "gqa70b":
        B = max(1, 64 // s)
        g = _gen(1003 + seed_offset, "cpu")
        lo, hi = 512 // s, 32768 // s
        lens = torch.randint(max(1, lo), hi + 1, (B,), generator=g).tolist()
        return dict(B=B, H_q=64, H_kv=8, d=128, dtype="bf16", lens=lens, seed=1003,
                    opts=dict(placement="shuffle", outlier_frac=0.01, outlier_scale=20.0))
    if name == "long":
        return dict(B=1, H_q=64, H_kv=8, d=128, dtype="bf16", lens=[max(1, 131072 // s)],
                    seed=1004, opts=dict(placement="shuffle"))
    if name == "cbatch":
        groups, per = 8, max(1, 32 // s)
        B = groups * per
        prefix = max(PAGE_TOKENS, (4096 // s) // PAGE_TOKENS * PAGE_TOKENS)
        cap = 16384 // s - 16
        g = _gen(1005 + seed_offset, "cpu")
        suf = _lognormal_suffix(B, g, median=1000.0 / s)
        suf = suf.clamp(min=1, max=max(1, cap - prefix))
        return dict(B=B, H_q=32, H_kv=8, d=128, dtype="f16", lens=(prefix + suf).tolist(),
                    seed=1005, opts=dict(placement="shuffle", steps=16, prefix_groups=groups,
                                         prefix_tokens=prefix))
    raise KeyError(name)


def named_config(name: str, device="cpu", gen_device=None, scale_down: int = 1,
                 shard: int = 0) -> Workload:
    """Build the named workload's pool, block table and lengths (see config_spec)."""
    c = config_spec(name, scale_down, shard)
    return build_workload(name, c["B"], c["H_q"], c["H_kv"], c["d"], c["dtype"], c["lens"],
                          seed=c["seed"], device=device, gen_device=gen_device, **c["opts"])


NAMED_CONFIGS = ("tiny", "mha7b", "gqa70b", "long", "cbatch")

"""KV memory utilisation of paged vs contiguous allocation over a stream of
chat completions (host-side simulation).

"KV缓存与Flash注意力", section "练习" (hard exercise): a toy PagedAttention
with fixed 16-token blocks and a free list, simulating 1,000 chat
completions of different lengths and comparing memory fragmentation with
contiguous allocation.  "KV Cache:推理慢的真正原因", section PagedAttention:
contiguous allocation reserves max_len per sequence and wastes what it does
not use; paging lifts utilisation from 20-40% to over 90%.

Both allocators serve the same arrival stream with the same KV budget
(tokens).  Contiguous allocation reserves max_len tokens per request up
front; paged allocation takes 16-token pages as the sequence grows, and when
the pool runs dry it preempts the most recently admitted sequence (frees its
pages and requeues it at the front; on readmission it needs its whole current
length again).  Utilisation = tokens actually stored / tokens reserved,
sampled at every decode step and averaged.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .allocator import PAGE_TOKENS, BlockAllocator, OutOfPages


@dataclass
class SimResult:
    completed: int
    mean_utilisation: float
    peak_concurrency: int
    mean_concurrency: float
    steps: int
    preemptions: int = 0


def _requests(n, seed, max_len, prompt_median=300, output_median=250):
    rng = np.random.default_rng(seed)
    prompt = np.clip(np.round(rng.lognormal(np.log(prompt_median), 0.8, n)), 1, max_len // 2).astype(int)
    out = np.clip(np.round(rng.lognormal(np.log(output_median), 0.9, n)), 1, max_len // 2).astype(int)
    return list(zip(prompt.tolist(), out.tolist()))


def simulate(mode: str, n_requests=1000, budget_tokens=1 << 17, max_len=4096, seed=0) -> SimResult:
    """Run the arrival stream through one allocator ("paged" or "contiguous").

    Each step admits waiting requests while memory allows (FIFO), then every
    running sequence decodes one token; finished sequences free their memory.
    """
    reqs = _requests(n_requests, seed, max_len)
    waiting = list(range(n_requests))
    running = {}          # id -> [length, remaining output tokens]
    alloc = BlockAllocator(budget_tokens // PAGE_TOKENS) if mode == "paged" else None
    reserved_contig = 0
    progress = {}         # preempted id -> [length, remaining]
    done = steps = 0
    util_sum = conc_sum = 0.0
    peak = 0
    order = []            # running ids in admission order (preemption victims from the end)
    preemptions = 0
    while done < n_requests:
        # admit
        while waiting:
            rid = waiting[0]
            prompt, out = reqs[rid]
            length = prompt if rid not in progress else progress[rid][0]
            if mode == "paged":
                try:
                    alloc.add(rid, length)
                except OutOfPages:
                    break
            else:
                if reserved_contig + max_len > budget_tokens:
                    break
                reserved_contig += max_len
            waiting.pop(0)
            running[rid] = progress.pop(rid) if rid in progress else [prompt, out]
            order.append(rid)
        if not running:
            raise RuntimeError("budget too small for a single request")
        # one decode step
        steps += 1
        finished = []
        for rid in list(order):
            if rid not in running:
                continue
            st = running[rid]
            if mode == "paged":
                while True:
                    try:
                        alloc.grow(rid, 1)
                        break
                    except OutOfPages:
                        victim = order[-1]
                        order.pop()
                        progress[victim] = running.pop(victim)
                        alloc.release(victim)
                        waiting.insert(0, victim)
                        preemptions += 1
                        if victim == rid:
                            break
                if rid not in running:
                    continue
            st[0] += 1
            st[1] -= 1
            if st[1] == 0:
                finished.append(rid)
        stored = sum(st[0] for st in running.values())
        reserved = alloc.used_pages * PAGE_TOKENS if mode == "paged" else reserved_contig
        util_sum += stored / reserved if reserved else 1.0
        conc_sum += len(running)
        peak = max(peak, len(running))
        for rid in finished:
            del running[rid]
            order.remove(rid)
            if mode == "paged":
                alloc.release(rid)
            else:
                reserved_contig -= max_len
            done += 1
    return SimResult(done, util_sum / steps, peak, conc_sum / steps, steps, preemptions)

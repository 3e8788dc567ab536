"""Toy one-layer decoder used to pin the oracle's append + paged gather (TEST ONLY).

[LES] "KV缓存与Flash注意力", section "步骤3": a naive incremental decoder that
re-encodes the whole prefix at every step and a cached decoder that projects
only the new token must give the same outputs; for a 100-token generation the
naive one does 5050 token projections and the cached one 100.  [BLOG]
"KV Cache:推理慢的真正原因", section "为什么需要 KV Cache": step i processes i
tokens, so the naive total is n(n+1)/2.

Exactness by construction: embeddings and projection weights are small
integers, so every projected K/V value is an integer of magnitude <= 16, which
binary16 stores exactly and binary64 sums exactly in any order.  The two
decoders therefore feed bit-identical K/V to the oracle and the comparison is
exact equality, which pins the oracle's append and block-table gather.
"""
import numpy as np

from . import F16, PAGE_TOKENS, append, attend


def _proj(x, w):
    # x: [d_model] ints, w: [d_model, H*d] ints -> exact integers
    return (x.astype(np.int64) @ w.astype(np.int64)).astype(np.float64)


def run(n_tokens=100, d_model=8, heads=2, d=8, seed=7):
    rng = np.random.default_rng(seed)
    X = rng.integers(-2, 3, size=(n_tokens, d_model))
    Wq = rng.integers(-1, 2, size=(d_model, heads * d))
    Wk = rng.integers(-1, 2, size=(d_model, heads * d))
    Wv = rng.integers(-1, 2, size=(d_model, heads * d))
    scale = 1.0 / np.sqrt(d)

    def words(a):
        return np.asarray(a, dtype=np.float16).view(np.uint16)

    max_pages = (n_tokens + PAGE_TOKENS - 1) // PAGE_TOKENS

    # ---- naive: re-project the whole prefix every step, contiguous placement
    naive_ops = 0
    naive_out = []
    for t in range(n_tokens):
        n = t + 1
        K = np.zeros((max_pages, heads, PAGE_TOKENS, d), dtype=np.float64)
        V = np.zeros_like(K)
        for j in range(n):                      # recompute every prefix token
            naive_ops += 1
            k = _proj(X[j], Wk).reshape(heads, d)
            v = _proj(X[j], Wv).reshape(heads, d)
            K[j // PAGE_TOKENS, :, j % PAGE_TOKENS, :] = k
            V[j // PAGE_TOKENS, :, j % PAGE_TOKENS, :] = v
        q = _proj(X[t], Wq).reshape(1, heads, d)
        bt = np.arange(max_pages, dtype=np.int32).reshape(1, max_pages)
        o, _ = attend(words(q), words(K), words(V), bt, np.array([n], np.int32), scale, F16)
        naive_out.append(o[0])

    # ---- cached: project only the new token, append into shuffled pages
    perm = rng.permutation(max_pages + 3).astype(np.int32)   # spare physical pages
    nb = max_pages + 3
    k_pool = np.full((nb, heads, PAGE_TOKENS, d), 0x7E00, dtype=np.uint16)  # NaN canary
    v_pool = np.full_like(k_pool, 0x7E00)
    bt = perm[:max_pages].reshape(1, max_pages).copy()
    cached_ops = 0
    cached_out = []
    for t in range(n_tokens):
        cached_ops += 1
        k = words(_proj(X[t], Wk).reshape(1, heads, d))
        v = words(_proj(X[t], Wv).reshape(1, heads, d))
        append(k_pool, v_pool, bt, np.array([t], np.int32), k, v)
        q = _proj(X[t], Wq).reshape(1, heads, d)
        o, _ = attend(words(q), k_pool, v_pool, bt, np.array([t + 1], np.int32), scale, F16)
        cached_out.append(o[0])

    return {
        "naive_ops": naive_ops,
        "cached_ops": cached_ops,
        "naive_out": np.stack(naive_out),
        "cached_out": np.stack(cached_out),
    }

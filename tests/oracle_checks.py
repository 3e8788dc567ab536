"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each check_* function raises AssertionError on a mismatch.  They are run
against the real oracle by test_oracle_pins.py and against deliberately broken
copies of it by test_oracle_mutants.py (every planted mistake must trip at
least one check).  Nothing here calls the CUDA library.
"""
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from oracle import toy_decoder
from synth import CANARY_WORD, PAGE_TOKENS, build_workload, step_inputs, to_words

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers

def f64(words, dtype):
    """Independent decoding of storage words with library conversions."""
    words = np.asarray(words, dtype=np.uint16)
    if dtype == oracle.F16:
        return words.view(np.float16).astype(np.float64)
    t = torch.from_numpy(words.astype(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def np_append(k_pool, v_pool, bt, slot, k_new, v_new):
    """Scatter written directly with numpy indexing (not via the oracle)."""
    for b in range(len(slot)):
        pos = int(slot[b])
        if pos < 0:
            continue
        page = bt[b, pos // PAGE_TOKENS]
        k_pool[page, :, pos % PAGE_TOKENS, :] = k_new[b]
        v_pool[page, :, pos % PAGE_TOKENS, :] = v_new[b]


def case(B, H_q, H_kv, d, dtype, lens, seed, placement="shuffle", **kw):
    """A small workload with the step's token already appended (by numpy)."""
    w = build_workload("pin", B, H_q, H_kv, d, dtype, lens, seed=seed,
                       placement=placement, **kw)
    si = step_inputs(w, 0)
    kc = to_words(w.k_cache).copy()
    vc = to_words(w.v_cache).copy()
    np_append(kc, vc, w.block_table.numpy(), si["slot"].numpy(),
              to_words(si["k_new"]), to_words(si["v_new"]))
    dt = oracle.BF16 if w.dtype == torch.bfloat16 else oracle.F16
    return dict(w=w, q=to_words(si["q"]), kc=kc, vc=vc, bt=w.block_table.numpy(),
                sl=si["seq_lens"].numpy(), slot=si["slot"].numpy(),
                k_new=to_words(si["k_new"]), v_new=to_words(si["v_new"]),
                scale=w.scale, dt=dt)


def logical(pool, bt, b, g, n):
    """[n, d] words of KV head g of sequence b in logical token order."""
    j = np.arange(n)
    return pool[bt[b, j // PAGE_TOKENS], g, j % PAGE_TOKENS, :]


def run(c, **kw):
    return oracle.attend(c["q"], c["kc"], c["vc"], c["bt"], c["sl"], c["scale"], c["dt"], **kw)


def close(a, b, rtol, atol, what):
    a = np.asarray(a)
    b = np.asarray(b)
    if not np.allclose(a, b, rtol=rtol, atol=atol, equal_nan=False):
        err = np.max(np.abs(a - b)) if a.shape == b.shape else "shape"
        raise AssertionError(f"{what}: max abs diff {err}")


# ------------------------------------------------------------- the checks

def check_f16_decoder():
    words = np.arange(65536, dtype=np.uint16)
    ref = words.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(w) for w in words])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "f16 NaN set differs"
    assert np.array_equal(got[~nan], ref[~nan]), "f16 decoding differs from numpy"
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan])), "f16 sign of zero"


def check_bf16_decoder():
    words = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(words.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(w) for w in words])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "bf16 NaN set differs"
    assert np.array_equal(got[~nan], ref[~nan]), "bf16 decoding differs from torch"


def check_kv_bytes_golden():
    n = 0
    with open(os.path.join(GOLDEN, "kv_bytes.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.split("|")[0].strip()
            if not line or line.startswith("#"):
                continue
            L, H, dh, s, tokens, batch, expect = (int(x) for x in line.split())
            got = oracle.kv_bytes_per_token(L, H, dh, s) * tokens * batch
            assert got == expect, f"kv bytes {L,H,dh,s,tokens,batch}: {got} != {expect}"
            n += 1
    assert n >= 5


def check_toy_decoder_golden():
    with open(os.path.join(GOLDEN, "op_counts.txt"), encoding="utf-8") as f:
        rows = [l.split("|")[0].split() for l in f if l.strip() and not l.startswith("#")]
    (tokens, naive, cached), = [tuple(int(x) for x in r) for r in rows]
    r = toy_decoder.run(n_tokens=tokens)
    assert r["naive_ops"] == naive, (r["naive_ops"], naive)
    assert r["cached_ops"] == cached, (r["cached_ops"], cached)
    assert np.array_equal(r["naive_out"], r["cached_out"]), "cached decode != naive recompute"


def check_against_sdpa():
    """Special case of a library routine: CPU float64 SDPA on gathered K/V."""
    cases = [
        (2, 4, 4, 64, "f16", [37, 64], 11),
        (2, 8, 2, 64, "bf16", [16, 53], 12),     # GQA group 4
        (1, 8, 1, 128, "f16", [100], 13),       # MQA
        (3, 6, 3, 32, "bf16", [1, 17, 33], 14),
    ]
    for (B, H_q, H_kv, d, dt, lens, seed) in cases:
        c = case(B, H_q, H_kv, d, dt, lens, seed)
        out, lse = run(c)
        G = H_q // H_kv
        for b in range(B):
            n = int(c["sl"][b])
            K = np.stack([f64(logical(c["kc"], c["bt"], b, g, n), c["dt"]) for g in range(H_kv)])
            V = np.stack([f64(logical(c["vc"], c["bt"], b, g, n), c["dt"]) for g in range(H_kv)])
            K = torch.from_numpy(K).repeat_interleave(G, dim=0)[None]
            V = torch.from_numpy(V).repeat_interleave(G, dim=0)[None]
            q = torch.from_numpy(f64(c["q"][b], c["dt"]))[None, :, None, :]
            ref = F.scaled_dot_product_attention(q, K, V, scale=c["scale"])[0, :, 0, :].numpy()
            close(out[b], ref, 1e-12, 1e-12, f"sdpa case {B,H_q,H_kv,d,dt} b={b}")
            s = (torch.einsum("hd,hnd->hn", q[0, :, 0, :], K[0]) * c["scale"]).numpy()
            ref_lse = np.log(np.sum(np.exp(s - s.max(1, keepdims=True)), 1)) + s.max(1)
            close(lse[b], ref_lse, 1e-12, 1e-12, "lse vs logsumexp")


def _brute(q, K, V, scale):
    """Plain triple loop with Python floats (written apart from the oracle)."""
    n, d = len(K), len(q)
    s = []
    for j in range(n):
        acc = 0.0
        for i in range(d):
            acc += q[i] * K[j][i]
        s.append(acc * scale)
    m = max(s)
    w = [math.exp(x - m) for x in s]
    tot = sum(w)
    return [sum(w[j] * V[j][i] for j in range(n)) / tot for i in range(d)]


def check_bruteforce_sweep():
    seed = 100
    for (B, H_q, H_kv) in [(1, 1, 1), (2, 2, 1), (1, 4, 2), (2, 8, 4), (1, 8, 8)]:
        for d in (2, 4, 8):
            for lens in ([1], [15], [16], [17], [31, 32], [33, 40], [3, 24]):
                lens = (lens * B)[:B]
                seed += 1
                c = case(B, H_q, H_kv, d, "f16" if seed % 2 else "bf16", lens, seed,
                         scale=0.37)
                out, _ = run(c)
                G = H_q // H_kv
                for b in range(B):
                    n = int(c["sl"][b])
                    for hq in range(H_q):
                        g = hq // G
                        K = f64(logical(c["kc"], c["bt"], b, g, n), c["dt"]).tolist()
                        V = f64(logical(c["vc"], c["bt"], b, g, n), c["dt"]).tolist()
                        q = f64(c["q"][b, hq], c["dt"]).tolist()
                        ref = _brute(q, K, V, c["scale"])
                        close(out[b, hq], ref, 1e-12, 1e-13, f"brute {B,H_q,H_kv,d,lens}")


def check_closed_forms():
    # n = 1: the only weight is exp(0) = 1, out is v_0 exactly, lse = s_0
    c = case(2, 4, 2, 64, "f16", [1, 1], 21)
    out, lse = run(c)
    for b in range(2):
        for hq in range(4):
            v0 = f64(c["v_new"][b, hq // 2], c["dt"])
            assert np.array_equal(out[b, hq], v0), "n=1 must return v_0 exactly"
            s0 = np.dot(f64(c["q"][b, hq], c["dt"]), f64(c["k_new"][b, hq // 2], c["dt"])) * c["scale"]
            close(lse[b, hq], s0, 1e-14, 1e-14, "n=1 lse")
    # constant V -> that constant
    c = case(1, 2, 2, 64, "bf16", [45], 22)
    const = to_words(torch.randn(2, 64, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16))
    n = int(c["sl"][0])
    j = np.arange(n)
    for g in range(2):
        c["vc"][c["bt"][0, j // 16], g, j % 16, :] = const[g]
    out, _ = run(c)
    for hq in range(2):
        close(out[0, hq], f64(const[hq], c["dt"]), 1e-13, 0, "constant V")
    # identical keys -> mean of V
    c = case(1, 1, 1, 64, "f16", [50], 23)
    n = int(c["sl"][0])
    j = np.arange(n)
    c["kc"][c["bt"][0, j // 16], 0, j % 16, :] = c["kc"][c["bt"][0, 0], 0, 0, :]
    out, _ = run(c)
    V = f64(logical(c["vc"], c["bt"], 0, 0, n), c["dt"])
    close(out[0, 0], V.mean(0), 1e-13, 1e-14, "identical keys")
    # one key dominating (k_j parallel to q, large) -> v_j
    c = case(1, 1, 1, 64, "f16", [40], 24)
    qv = f64(c["q"][0, 0], c["dt"])
    jstar = 29
    c["kc"][c["bt"][0, jstar // 16], 0, jstar % 16, :] = np.asarray(8.0 * qv, np.float16).view(np.uint16)
    out, _ = run(c)
    vstar = f64(c["vc"][c["bt"][0, jstar // 16], 0, jstar % 16, :], c["dt"])
    close(out[0, 0], vstar, 1e-12, 1e-12, "dominant key")
    # empty sequence -> 0 and lse = -inf
    c = case(2, 2, 1, 64, "f16", [0, 5], 25)
    out, lse = run(c)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0])), "empty sequence"
    assert np.all(np.isfinite(out[1])), "non-empty sequence after an empty one"


def check_gqa_equals_repeated_mha():
    c = case(2, 8, 2, 64, "bf16", [30, 47], 31)
    out, lse = run(c)
    G = 4
    c2 = dict(c)
    c2["kc"] = np.repeat(c["kc"], G, axis=1)
    c2["vc"] = np.repeat(c["vc"], G, axis=1)
    out2, lse2 = run(c2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2), "GQA != repeated-head MHA"


def check_tiled_equals_one_shot():
    c = case(2, 4, 2, 64, "f16", [70, 33], 41)
    out, _ = run(c)
    for tile in (1, 4, 16, 70, 1000):
        t = oracle.attend_tiled(c["q"], c["kc"], c["vc"], c["bt"], c["sl"], c["scale"], c["dt"], tile)
        close(t, out, 1e-12, 1e-13, f"tiled tile={tile}")


def check_merge():
    c = case(2, 4, 1, 64, "bf16", [90, 61], 51)
    full, full_lse = run(c)
    rng = np.random.default_rng(3)
    S = 5
    B = 2
    po = np.zeros((B, 4, S, 64))
    pl = np.full((B, 4, S), -np.inf)
    counts = np.zeros(B, np.int32)
    for b in range(B):
        n = int(c["sl"][b])
        cuts = np.sort(rng.choice(np.arange(1, n), size=3, replace=False))
        bounds = [0, *cuts.tolist(), n]
        lo = np.zeros(B, np.int32)
        hi = np.zeros(B, np.int32)
        for s in range(len(bounds) - 1):
            lo[:] = 0
            hi[:] = 0
            lo[b], hi[b] = bounds[s], bounds[s + 1]
            o, l = run(c, lo=lo, hi=hi)
            po[b, :, s] = o[b]
            pl[b, :, s] = l[b]
        counts[b] = len(bounds) - 1
    out, lse = oracle.merge(po, pl, counts)
    close(out, full, 1e-12, 1e-13, "merge of partitions")
    close(lse, full_lse, 1e-12, 1e-13, "merged lse")
    # one partition: identity
    o1, l1 = oracle.merge(full[:, :, None, :], full_lse[:, :, None])
    assert np.array_equal(o1, full) and np.array_equal(l1, full_lse), "S=1 merge is not the identity"
    # empty partitions (lse = -inf, garbage o) carry no weight
    po2 = np.concatenate([po, np.full((B, 4, 2, 64), np.nan)], axis=2)
    pl2 = np.concatenate([pl, np.full((B, 4, 2), -np.inf)], axis=2)
    out2, lse2 = oracle.merge(po2, pl2, counts + 2)
    close(out2, out, 1e-15, 0, "empty partitions")
    # all empty -> 0, -inf
    o3, l3 = oracle.merge(np.full((1, 1, 3, 8), np.nan), np.full((1, 1, 3), -np.inf))
    assert np.all(o3 == 0) and np.all(np.isneginf(l3)), "all-empty merge"


def check_paging_invariance():
    c = case(3, 4, 2, 64, "f16", [40, 16, 77], 61)
    out, lse = run(c)
    # same logical content on identity-placed pages
    bt, kc, vc = c["bt"], c["kc"], c["vc"]
    nb_used = [(int(n) + 15) // 16 for n in c["sl"]]
    tot = sum(nb_used)
    kc2 = np.full((tot,) + kc.shape[1:], CANARY_WORD, np.uint16)
    vc2 = np.full_like(kc2, CANARY_WORD)
    bt2 = np.full_like(bt, -1)
    p = 0
    for b, k in enumerate(nb_used):
        for i in range(k):
            kc2[p] = kc[bt[b, i]]
            vc2[p] = vc[bt[b, i]]
            bt2[b, i] = p
            p += 1
    c2 = dict(c, kc=kc2, vc=vc2, bt=bt2)
    out2, lse2 = run(c2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2), "placement changed the result"


def check_shared_prefix_equals_private():
    c = case(4, 4, 2, 64, "bf16", [40, 55, 33, 70], 71, prefix_groups=2, prefix_tokens=32)
    assert c["bt"][0, 0] == c["bt"][1, 0] and c["bt"][2, 1] == c["bt"][3, 1]
    out, lse = run(c)
    bt, kc, vc = c["bt"], c["kc"], c["vc"]
    pages = []
    bt2 = np.full_like(bt, -1)
    for b in range(4):
        for i in range((int(c["sl"][b]) + 15) // 16):
            bt2[b, i] = len(pages)
            pages.append(bt[b, i])
    c2 = dict(c, kc=kc[pages].copy(), vc=vc[pages].copy(), bt=bt2)
    out2, lse2 = run(c2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2), "shared prefix != private copies"


def check_append():
    w = build_workload("pin", 5, 4, 2, 64, "f16", [1, 16, 17, 40, 0], seed=81)
    si = step_inputs(w, 0)
    kc0 = to_words(w.k_cache).copy()
    vc0 = to_words(w.v_cache).copy()
    kc, vc = kc0.copy(), vc0.copy()
    oracle.append(kc, vc, w.block_table.numpy(), si["slot"].numpy(),
                  to_words(si["k_new"]), to_words(si["v_new"]))
    kr, vr = kc0.copy(), vc0.copy()
    np_append(kr, vr, w.block_table.numpy(), si["slot"].numpy(),
              to_words(si["k_new"]), to_words(si["v_new"]))
    assert np.array_equal(kc, kr) and np.array_equal(vc, vr), "append differs from the scatter"
    changed = np.any(kc != kc0, axis=(1, 3))            # [page, token]
    expect = np.zeros_like(changed)
    bt = w.block_table.numpy()
    for b, pos in enumerate(si["slot"].numpy()):
        if pos >= 0:
            expect[bt[b, pos // 16], pos % 16] = True
    assert np.array_equal(changed, expect), "append touched other rows"
    # paged append then gather == the contiguous KVCache of the blog
    # ("缓存的是什么": k[:, :, start:end] = k_new at start = length)
    b = 3
    n = int(si["seq_lens"][b])
    contiguous = np.full((2, 64, 64), CANARY_WORD, np.uint16)     # [H, max_len, d]
    contiguous[:, : n - 1] = logical(kc0, bt, b, slice(None), n - 1).transpose(1, 0, 2)
    contiguous[:, n - 1: n] = to_words(si["k_new"])[b][:, None, :]
    got = logical(kc, bt, b, slice(None), n).transpose(1, 0, 2)
    assert np.array_equal(got, contiguous[:, :n]), "paged append != contiguous append"


# ------------------------------------------------------------ 8-bit cache

def _torch_e4m3(x32):
    """float32 array -> E4M3 codes via torch's float8_e4m3fn conversion."""
    return torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def _torch_e4m3_value(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def check_e4m3_decoder():
    codes = np.arange(256, dtype=np.uint8)
    ref = _torch_e4m3_value(codes)
    got = np.array([oracle.e4m3_decode(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "E4M3 NaN codes differ"
    assert np.array_equal(got[~nan], ref[~nan]), "E4M3 decoding differs from torch"
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def check_e4m3_encoder():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-12, 6, 20000))).astype(np.float32)
    x = np.clip(x, -448, 448)
    # every midpoint between neighbouring finite values: ties go to the even code
    vals = np.unique(np.abs(_torch_e4m3_value(np.arange(0x7F, dtype=np.uint8))))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, vals.astype(np.float32)])
    got = np.array([oracle.e4m3_encode(v) for v in x], dtype=np.uint8)
    ref = _torch_e4m3(x)
    assert np.array_equal(got, ref), f"{int(np.sum(got != ref))} E4M3 encodings differ from torch"
    # saturation (torch turns these into NaN; the kernels' conversion saturates)
    assert oracle.e4m3_encode(449.0) == 0x7E and oracle.e4m3_encode(-1000.0) == 0xFE


def _quantize_numpy(rows_f32):
    """Independent re-derivation: fp32 scale max|x|/448 per 32 channels, codes by torch."""
    n, d = rows_f32.shape
    g = rows_f32.reshape(n, d // 32, 32)
    mx = np.abs(g).max(axis=2).astype(np.float32)
    s = (mx / np.float32(448.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        qv = np.where(s[..., None] > 0, g / s[..., None], 0).astype(np.float32)
    codes = _torch_e4m3(qv.reshape(n, d)).reshape(n, d)
    return codes, s


def check_quantize_fp8():
    rng = np.random.default_rng(12)
    for dt, tdt in ((oracle.F16, torch.float16), (oracle.BF16, torch.bfloat16)):
        x = torch.from_numpy(rng.standard_normal((64, 128)).astype(np.float32))
        x[3, 17] = 40.0                        # an outlier channel in group 0 of row 3
        x[5, 64:96] = 0.0                      # an all-zero group
        xq = x.to(tdt)
        words = to_words(xq)
        codes, scales = oracle.quantize_fp8(words, dt)
        rows32 = xq.to(torch.float32).numpy()
        rc, rs = _quantize_numpy(rows32)
        assert np.array_equal(codes, rc), "codes differ from the numpy/torch re-derivation"
        assert np.array_equal(scales, rs), "scales differ from the numpy re-derivation"
        deq = _torch_e4m3_value(codes).reshape(64, 4, 32) * scales[..., None]
        err = np.abs(deq.reshape(64, 128) - rows32)
        # half an E4M3 ulp at the largest binade (448 -> ulp 32), in units of s;
        # the tiny slack covers ties landing exactly on the half ulp
        bound = scales.repeat(32, axis=1).astype(np.float64) * 16.0 * (1 + 1e-6) + 1e-30
        assert np.all(err <= bound), "round trip exceeds half an E4M3 ulp"
        assert scales[5, 2] == 0 and np.all(codes[5, 64:96] == 0)
        # the outlier only coarsens its own group
        assert scales[3, 0] > 10 * np.median(scales[:, 0]) and scales[3, 1] < 3 * np.median(scales[:, 1])


def _fp8_case(B, H_q, H_kv, d, dt, lens, seed):
    c = case(B, H_q, H_kv, d, dt, lens, seed)
    k8, ks = oracle.quantize_fp8(c["kc"], c["dt"])
    v8, vs = oracle.quantize_fp8(c["vc"], c["dt"])
    c.update(k8=k8, ks=ks, v8=v8, vs=vs)
    return c


def check_attend_fp8_against_sdpa():
    for (B, H_q, H_kv, d, dt, lens, seed) in [(2, 8, 2, 128, "bf16", [40, 77], 31),
                                              (1, 4, 4, 64, "f16", [33], 32)]:
        c = _fp8_case(B, H_q, H_kv, d, dt, lens, seed)
        out, lse = oracle.attend_fp8(c["q"], c["k8"], c["v8"], c["ks"], c["vs"], c["bt"], c["sl"],
                                     c["scale"], c["dt"])
        G = H_q // H_kv
        for b in range(B):
            n = int(c["sl"][b])
            j = np.arange(n)
            pages, rows = c["bt"][b, j // 16], j % 16
            Kd = _torch_e4m3_value(c["k8"][pages, :, rows, :]) * np.repeat(c["ks"][pages, :, rows, :], 32, axis=-1)
            Vd = _torch_e4m3_value(c["v8"][pages, :, rows, :]) * np.repeat(c["vs"][pages, :, rows, :], 32, axis=-1)
            K = torch.from_numpy(Kd.transpose(1, 0, 2)).repeat_interleave(G, dim=0)[None]
            V = torch.from_numpy(Vd.transpose(1, 0, 2)).repeat_interleave(G, dim=0)[None]
            q = torch.from_numpy(f64(c["q"][b], c["dt"]))[None, :, None, :]
            ref = F.scaled_dot_product_attention(q, K, V, scale=c["scale"])[0, :, 0, :].numpy()
            close(out[b], ref, 1e-12, 1e-12, "fp8 attention vs SDPA on dequantised K/V")
        # quantisation error against the unquantised cache stays small
        full, _ = run(c)
        assert np.max(np.abs(out - full)) < 0.1, "fp8 attention far from fp16/bf16 attention"


def check_append_fp8():
    w = build_workload("pin8", 4, 4, 2, 128, "bf16", [1, 16, 17, 40], seed=83)
    si = step_inputs(w, 0)
    kc, vc = to_words(w.k_cache), to_words(w.v_cache)
    k8, ks = oracle.quantize_fp8(kc, oracle.BF16)
    v8, vs = oracle.quantize_fp8(vc, oracle.BF16)
    k8_0, ks_0 = k8.copy(), ks.copy()
    oracle.append_fp8(k8, v8, ks, vs, w.block_table.numpy(), si["slot"].numpy(),
                      to_words(si["k_new"]), to_words(si["v_new"]), oracle.BF16)
    kn8, kns = oracle.quantize_fp8(to_words(si["k_new"]), oracle.BF16)
    bt = w.block_table.numpy()
    changed = np.any(k8 != k8_0, axis=(1, 3))
    for b, pos in enumerate(si["slot"].numpy()):
        p, r = bt[b, pos // 16], pos % 16
        assert np.array_equal(k8[p, :, r, :], kn8[b]) and np.array_equal(ks[p, :, r, :], kns[b])
        changed[p, r] = False
    assert not changed.any(), "fp8 append touched other rows"


# ------------------------------------------------------------ INT8 cache

def _i8(codes):
    return np.ascontiguousarray(codes, dtype=np.uint8).view(np.int8).astype(np.float64)


def check_int8_decoder():
    codes = np.arange(256, dtype=np.uint8)
    got = np.array([oracle.int8_decode(c) for c in codes])
    assert np.array_equal(got, codes.view(np.int8).astype(np.float64)), "INT8 decoding differs"


def check_int8_encoder():
    # closed forms: nearest integer, ties to the even one, clamp at +-127, NaN -> 0
    cases = {2.5: 2, 3.5: 4, -2.5: -2, 0.5: 0, 1.5: 2, -0.5: 0, 126.5: 126, 127.4: 127,
             127.5: 127, 200.0: 127, -1e9: -127, -127.6: -127, 63.49: 63, -63.51: -64, 0.0: 0}
    for x, want in cases.items():
        got = np.uint8(oracle.int8_encode(x)).view(np.int8)
        assert got == want, f"INT8 encode({x}) = {got}, expected {want}"
    assert oracle.int8_encode(float("nan")) == 0
    rng = np.random.default_rng(14)
    x = rng.uniform(-127.4, 127.4, 5000).astype(np.float32)
    got = _i8(np.array([oracle.int8_encode(v) for v in x], dtype=np.uint8))
    assert np.all(np.abs(got - x.astype(np.float64)) <= 0.5), "INT8 encode is not the nearest integer"


def check_quantize_int8():
    rng = np.random.default_rng(15)
    for dt, tdt in ((oracle.F16, torch.float16), (oracle.BF16, torch.bfloat16)):
        x = torch.from_numpy(rng.standard_normal((64, 128)).astype(np.float32))
        x[3, 17] = 40.0                        # an outlier channel in group 0 of row 3
        x[5, 64:96] = 0.0                      # an all-zero group
        x[9, 40] = float("nan")                # a NaN element (group 1 of row 9)
        xq = x.to(tdt)
        codes, scales = oracle.quantize_int8(to_words(xq), dt)
        rows32 = xq.to(torch.float32).numpy().astype(np.float64)
        deq = (_i8(codes).reshape(64, 4, 32) * scales[..., None]).reshape(64, 128)
        fin = np.isfinite(rows32)
        # every value within half a quantisation step of its group, plus the
        # rounding of the fp32 quotient x / s the code is taken from (at most
        # 127 * 2^-24 of a step: a quotient just below a half can round onto it)
        step = scales.repeat(32, axis=1).astype(np.float64)
        bound = step * (0.5 + 128 * 2.0 ** -24)
        assert np.all(np.abs(deq - rows32)[fin] <= bound[fin]), "INT8 round trip exceeds half a step"
        # the largest magnitude of each group is the extreme code, with its sign
        g = np.where(fin, rows32, 0).reshape(64, 4, 32)
        i = np.abs(g).argmax(axis=2)
        ext = np.take_along_axis(_i8(codes).reshape(64, 4, 32), i[..., None], 2)[..., 0]
        sgn = np.sign(np.take_along_axis(g, i[..., None], 2)[..., 0])
        nz = scales > 0
        assert np.array_equal(ext[nz], 127 * sgn[nz]), "a group's extreme is not +-127"
        assert scales[5, 2] == 0 and np.all(codes[5, 64:96] == 0)
        assert codes[9, 40] == 0 and np.isfinite(scales[9, 1]) and scales[9, 1] > 0
        # the outlier only coarsens its own group
        assert scales[3, 0] > 10 * np.median(scales[:, 0]) and scales[3, 1] < 3 * np.median(scales[:, 1])


def check_attend_int8_against_sdpa():
    for (B, H_q, H_kv, d, dt, lens, seed) in [(2, 8, 2, 128, "bf16", [40, 77], 41),
                                              (1, 4, 4, 64, "f16", [33], 42)]:
        c = case(B, H_q, H_kv, d, dt, lens, seed)
        k8, ks = oracle.quantize_int8(c["kc"], c["dt"])
        v8, vs = oracle.quantize_int8(c["vc"], c["dt"])
        out, lse = oracle.attend_int8(c["q"], k8, v8, ks, vs, c["bt"], c["sl"], c["scale"], c["dt"])
        G = H_q // H_kv
        for b in range(B):
            n = int(c["sl"][b])
            j = np.arange(n)
            pages, rows = c["bt"][b, j // 16], j % 16
            Kd = _i8(k8[pages, :, rows, :]) * np.repeat(ks[pages, :, rows, :], 32, axis=-1)
            Vd = _i8(v8[pages, :, rows, :]) * np.repeat(vs[pages, :, rows, :], 32, axis=-1)
            K = torch.from_numpy(Kd.transpose(1, 0, 2)).repeat_interleave(G, dim=0)[None]
            V = torch.from_numpy(Vd.transpose(1, 0, 2)).repeat_interleave(G, dim=0)[None]
            q = torch.from_numpy(f64(c["q"][b], c["dt"]))[None, :, None, :]
            ref = F.scaled_dot_product_attention(q, K, V, scale=c["scale"])[0, :, 0, :].numpy()
            close(out[b], ref, 1e-12, 1e-12, "int8 attention vs SDPA on dequantised K/V")
        full, _ = run(c)
        assert np.max(np.abs(out - full)) < 0.05, "int8 attention far from fp16/bf16 attention"


def check_append_int8():
    w = build_workload("pin8i", 4, 4, 2, 128, "bf16", [1, 16, 17, 40], seed=84)
    si = step_inputs(w, 0)
    kc, vc = to_words(w.k_cache), to_words(w.v_cache)
    k8, ks = oracle.quantize_int8(kc, oracle.BF16)
    v8, vs = oracle.quantize_int8(vc, oracle.BF16)
    k8_0, v8_0 = k8.copy(), v8.copy()
    oracle.append_int8(k8, v8, ks, vs, w.block_table.numpy(), si["slot"].numpy(),
                       to_words(si["k_new"]), to_words(si["v_new"]), oracle.BF16)
    kn8, kns = oracle.quantize_int8(to_words(si["k_new"]), oracle.BF16)
    vn8, vns = oracle.quantize_int8(to_words(si["v_new"]), oracle.BF16)
    bt = w.block_table.numpy()
    changed = np.any(k8 != k8_0, axis=(1, 3)) | np.any(v8 != v8_0, axis=(1, 3))
    for b, pos in enumerate(si["slot"].numpy()):
        p, r = bt[b, pos // 16], pos % 16
        assert np.array_equal(k8[p, :, r, :], kn8[b]) and np.array_equal(ks[p, :, r, :], kns[b])
        assert np.array_equal(v8[p, :, r, :], vn8[b]) and np.array_equal(vs[p, :, r, :], vns[b])
        changed[p, r] = False
    assert not changed.any(), "int8 append touched other rows"


# ------------------------------------------------------------ INT4 cache

def _unpack4(codes):
    """Packed INT4 bytes [..., d/2] -> code values [..., d] in float64: channel
    2i is the low nibble of byte i, 2i+1 its high nibble, two's complement
    (numpy only, independent of the oracle)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    lo = (c & 15).astype(np.int64)
    hi = (c >> 4).astype(np.int64)
    v = np.stack([lo, hi], axis=-1).reshape(c.shape[:-1] + (2 * c.shape[-1],))
    return np.where(v >= 8, v - 16, v).astype(np.float64)


def check_int4_decoder():
    got = np.array([oracle.int4_decode(n) for n in range(16)])
    assert np.array_equal(got, np.array([0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1.0])), \
        "INT4 decoding differs from 4-bit two's complement"


def check_int4_encoder():
    # closed forms: nearest integer, ties to the even one, clamp at +-7, NaN -> 0
    cases = {2.5: 2, 3.5: 4, -2.5: -2, 0.5: 0, -0.5: 0, 1.5: 2, 6.5: 6, 6.6: 7, 7.4: 7, 7.5: 7,
             100.0: 7, -100.0: -7, -7.6: -7, -6.5: -6, 4.49: 4, -4.51: -5, 0.0: 0}
    for x, want in cases.items():
        n = oracle.int4_encode(x)
        assert 0 <= n < 16, f"INT4 encode({x}) is not a nibble: {n}"
        got = n - 16 if n >= 8 else n
        assert got == want, f"INT4 encode({x}) = {got}, expected {want}"
    assert oracle.int4_encode(float("nan")) == 0
    rng = np.random.default_rng(24)
    x = rng.uniform(-7.4, 7.4, 3000).astype(np.float32)
    got = np.array([oracle.int4_encode(v) for v in x])
    got = np.where(got >= 8, got - 16, got)
    assert np.all(np.abs(got - x.astype(np.float64)) <= 0.5), "INT4 encode is not the nearest integer"


def check_quantize_int4():
    rng = np.random.default_rng(25)
    for dt, tdt in ((oracle.F16, torch.float16), (oracle.BF16, torch.bfloat16)):
        x = torch.from_numpy(rng.standard_normal((64, 128)).astype(np.float32))
        x[3, 17] = 40.0                        # an outlier channel in group 0 of row 3
        x[5, 64:96] = 0.0                      # an all-zero group
        x[9, 40] = float("nan")                # a NaN element (group 1 of row 9)
        xq = x.to(tdt)
        codes, scales = oracle.quantize_int4(to_words(xq), dt)
        assert codes.shape == (64, 64) and scales.shape == (64, 4)
        rows32 = xq.to(torch.float32).numpy().astype(np.float64)
        q = _unpack4(codes)
        deq = (q.reshape(64, 4, 32) * scales[..., None]).reshape(64, 128)
        fin = np.isfinite(rows32)
        step = scales.repeat(32, axis=1).astype(np.float64)
        bound = step * (0.5 + 8 * 2.0 ** -24)
        assert np.all(np.abs(deq - rows32)[fin] <= bound[fin]), "INT4 round trip exceeds half a step"
        assert np.all(np.abs(q) <= 7), "an INT4 code outside [-7, 7]"
        # the largest magnitude of each group is the extreme code, with its sign
        g = np.where(fin, rows32, 0).reshape(64, 4, 32)
        i = np.abs(g).argmax(axis=2)
        ext = np.take_along_axis(q.reshape(64, 4, 32), i[..., None], 2)[..., 0]
        sgn = np.sign(np.take_along_axis(g, i[..., None], 2)[..., 0])
        nz = scales > 0
        assert np.array_equal(ext[nz], 7 * sgn[nz]), "a group's extreme is not +-7"
        assert scales[5, 2] == 0 and np.all(q[5, 64:96] == 0)
        assert q[9, 40] == 0 and np.isfinite(scales[9, 1]) and scales[9, 1] > 0
        assert scales[3, 0] > 10 * np.median(scales[:, 0]) and scales[3, 1] < 3 * np.median(scales[:, 1])
    # packing: a row whose codes are known (x = code, max 7 -> s = 1): channel
    # 2i in the low nibble of byte i, 2i+1 in the high one
    want = np.array([(i % 15) - 7 for i in range(64)], dtype=np.float32)
    want[0] = 7.0
    codes, scales = oracle.quantize_int4(to_words(torch.from_numpy(want).to(torch.float16)), oracle.F16)
    assert np.array_equal(scales, np.ones(2, dtype=np.float32))
    lo = np.where(want[0::2] < 0, want[0::2] + 16, want[0::2]).astype(np.uint8)
    hi = np.where(want[1::2] < 0, want[1::2] + 16, want[1::2]).astype(np.uint8)
    assert np.array_equal(codes, lo | (hi << 4)), "INT4 nibble order"


def check_attend_int4_against_sdpa():
    for (B, H_q, H_kv, d, dt, lens, seed) in [(2, 8, 2, 128, "bf16", [40, 77], 43),
                                              (1, 4, 4, 64, "f16", [33], 44)]:
        c = case(B, H_q, H_kv, d, dt, lens, seed)
        k4, ks = oracle.quantize_int4(c["kc"], c["dt"])
        v4, vs = oracle.quantize_int4(c["vc"], c["dt"])
        out, lse = oracle.attend_int4(c["q"], k4, v4, ks, vs, c["bt"], c["sl"], c["scale"], c["dt"])
        G = H_q // H_kv
        for b in range(B):
            n = int(c["sl"][b])
            j = np.arange(n)
            pages, rows = c["bt"][b, j // 16], j % 16
            Kd = _unpack4(k4[pages, :, rows, :]) * np.repeat(ks[pages, :, rows, :], 32, axis=-1)
            Vd = _unpack4(v4[pages, :, rows, :]) * np.repeat(vs[pages, :, rows, :], 32, axis=-1)
            K = torch.from_numpy(Kd.transpose(1, 0, 2)).repeat_interleave(G, dim=0)[None]
            V = torch.from_numpy(Vd.transpose(1, 0, 2)).repeat_interleave(G, dim=0)[None]
            q = torch.from_numpy(f64(c["q"][b], c["dt"]))[None, :, None, :]
            ref = F.scaled_dot_product_attention(q, K, V, scale=c["scale"])[0, :, 0, :].numpy()
            close(out[b], ref, 1e-12, 1e-12, "int4 attention vs SDPA on dequantised K/V")
        full, _ = run(c)
        assert np.max(np.abs(out - full)) < 0.5, "int4 attention far from fp16/bf16 attention"


def check_append_int4():
    w = build_workload("pin4i", 4, 4, 2, 128, "bf16", [1, 16, 17, 40], seed=85)
    si = step_inputs(w, 0)
    kc, vc = to_words(w.k_cache), to_words(w.v_cache)
    k4, ks = oracle.quantize_int4(kc, oracle.BF16)
    v4, vs = oracle.quantize_int4(vc, oracle.BF16)
    k4_0, v4_0 = k4.copy(), v4.copy()
    oracle.append_int4(k4, v4, ks, vs, w.block_table.numpy(), si["slot"].numpy(),
                       to_words(si["k_new"]), to_words(si["v_new"]), oracle.BF16)
    kn4, kns = oracle.quantize_int4(to_words(si["k_new"]), oracle.BF16)
    vn4, vns = oracle.quantize_int4(to_words(si["v_new"]), oracle.BF16)
    bt = w.block_table.numpy()
    changed = np.any(k4 != k4_0, axis=(1, 3)) | np.any(v4 != v4_0, axis=(1, 3))
    for b, pos in enumerate(si["slot"].numpy()):
        p, r = bt[b, pos // 16], pos % 16
        assert np.array_equal(k4[p, :, r, :], kn4[b]) and np.array_equal(ks[p, :, r, :], kns[b])
        assert np.array_equal(v4[p, :, r, :], vn4[b]) and np.array_equal(vs[p, :, r, :], vns[b])
        changed[p, r] = False
    assert not changed.any(), "int4 append touched other rows"


ALL_CHECKS = [
    check_f16_decoder,
    check_bf16_decoder,
    check_kv_bytes_golden,
    check_toy_decoder_golden,
    check_against_sdpa,
    check_bruteforce_sweep,
    check_closed_forms,
    check_gqa_equals_repeated_mha,
    check_tiled_equals_one_shot,
    check_merge,
    check_paging_invariance,
    check_shared_prefix_equals_private,
    check_append,
    check_e4m3_decoder,
    check_e4m3_encoder,
    check_quantize_fp8,
    check_attend_fp8_against_sdpa,
    check_append_fp8,
    check_int8_decoder,
    check_int8_encoder,
    check_quantize_int8,
    check_attend_int8_against_sdpa,
    check_append_int8,
    check_int4_decoder,
    check_int4_encoder,
    check_quantize_int4,
    check_attend_int4_against_sdpa,
    check_append_int4,
]

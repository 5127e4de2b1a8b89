"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an oracle object (``oracle.OracleLib``) and
raises AssertionError if the oracle disagrees with what the mathematics fixes:

* brute-force dense attention, written independently with numpy (gather the
  pages into a contiguous K, one matmul, a softmax);
* closed forms: a single visible token, identical value rows, a zero softmax
  scale, equal-lse partials;
* invariances: relabelling physical pages, splitting the key range and
  merging, and the reduction of a causal multi-token row to a one-token call;
* lse recomputed in extended precision from the scores.

The same functions run against mutated copies of the oracle in
``test_oracle_mutants.py`` to show each planted mistake fails at least one pin.
"""
from __future__ import annotations

import math

import numpy as np

import mla_workloads as W

TOL = 1e-12


def small_inputs(seqlens, s_q=1, h_q=4, h_kv=1, causal=False, seed=0, d=W.D_QK, dv=W.D_V,
                 scale=W.SCALE_192, extra_pages=2):
    """Tiny seeded paged inputs with given lengths (optionally a narrower d)."""
    w = W.Workload("pin", len(seqlens), s_q, h_q, h_kv, causal, "explicit", (tuple(seqlens),),
                   seed=seed, softmax_scale=scale)
    inp = W.make_inputs(w, seqlens=seqlens, extra_pages=extra_pages)
    if d != W.D_QK:
        inp["q"] = np.ascontiguousarray(inp["q"][..., :d])
        inp["kvcache"] = np.ascontiguousarray(inp["kvcache"][..., :d])
        inp["d"] = d
    inp["dv"] = dv
    return inp


def dense_reference(inp):
    """Independent dense formulation: gather each sequence's rows, matmul, softmax."""
    q = W.bf16_bits_to_f32(inp["q"]).astype(np.float64)            # [b][s_q][h_q][d]
    kv = W.bf16_bits_to_f32(inp["kvcache"]).astype(np.float64)     # [P][64][h_kv][d]
    b, s_q, h_q, d = q.shape
    h_kv = kv.shape[2]
    dv = inp["dv"]
    o = np.zeros((b, s_q, h_q, dv))
    lse = np.full((b, h_q, s_q), -np.inf)
    for bi in range(b):
        L = int(inp["cache_seqlens"][bi])
        t = np.arange(L)
        pages = inp["block_table"][bi][t // W.PAGE]
        K = kv[pages, t % W.PAGE]                                   # [L][h_kv][d]
        for h in range(h_q):
            Kg = K[:, h // (h_q // h_kv), :]                        # [L][d]
            S = inp["softmax_scale"] * (q[bi, :, h, :] @ Kg.T)      # [s_q][L]
            if inp["causal"]:
                allowed = t[None, :] <= (L - s_q + np.arange(s_q))[:, None]
            else:
                allowed = np.ones((s_q, L), dtype=bool)
            for i in range(s_q):
                row = S[i][allowed[i]]
                if row.size == 0:
                    continue
                mx = row.max()
                wts = np.exp(row - mx)
                lse[bi, h, i] = mx + math.log(wts.sum())
                o[bi, i, h] = (wts / wts.sum()) @ Kg[allowed[i], :dv]
    return o, lse


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    same_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    diff = np.where(same_inf, 0.0, np.abs(a - b))
    assert not np.isnan(diff).any(), f"{what}: NaN"
    m = float(diff.max()) if diff.size else 0.0
    assert m <= tol, f"{what}: max diff {m:.3e} > {tol:.1e}"


def _run(ora, inp, **kw):
    return ora.decode_inputs(inp, **kw)


# --------------------------------------------------------------------------- pins
def pin_bruteforce(ora):
    cases = [
        dict(seqlens=[37, 130], h_q=16),
        dict(seqlens=[1, 63, 64, 65, 127], h_q=4),
        dict(seqlens=[5, 70], s_q=2, h_q=4, causal=True),
        dict(seqlens=[3, 66, 129], s_q=3, h_q=2, causal=True),
        dict(seqlens=[40, 90], h_q=4, h_kv=2),                       # grouped KV heads
        dict(seqlens=[70, 9], s_q=2, h_q=6, h_kv=3, causal=True, d=40, dv=24),
    ]
    for k, c in enumerate(cases):
        inp = small_inputs(seed=100 + k, **c)
        o, lse = _run(ora, inp)
        ro, rl = dense_reference(inp)
        _close(o, ro, what=f"o case {k}")
        _close(lse, rl, what=f"lse case {k}")


def pin_single_token(ora):
    inp = small_inputs([1, 1], h_q=8, seed=7)
    o, lse = _run(ora, inp)
    kv = W.bf16_bits_to_f32(inp["kvcache"]).astype(np.float64)
    q = W.bf16_bits_to_f32(inp["q"]).astype(np.float64)
    for b in range(2):
        row = kv[inp["block_table"][b][0], 0, 0]
        for h in range(8):
            assert np.array_equal(o[b, 0, h], row[:W.D_V]), "single token: o != its value row"
            _close(lse[b, h, 0], inp["softmax_scale"] * float(q[b, 0, h] @ row), what="single lse")


def pin_equal_values(ora):
    inp = small_inputs([50, 129], h_q=4, seed=8)
    kv = inp["kvcache"].copy()
    common = kv[0, 0, 0, :W.D_V].copy()
    kv[:, :, :, :W.D_V] = common                      # every value row identical
    inp["kvcache"] = kv
    o, _ = _run(ora, inp)
    want = W.bf16_bits_to_f32(common).astype(np.float64)
    _close(o, np.broadcast_to(want, o.shape), tol=1e-13, what="equal values")


def pin_page_permutation(ora):
    inp = small_inputs([100, 3, 190], h_q=4, seed=9, extra_pages=5)
    o1, l1 = _run(ora, inp)
    rng = np.random.default_rng(99)
    npages = inp["kvcache"].shape[0]
    perm = rng.permutation(npages)                    # new page id of old page p is perm[p]
    kv2 = np.empty_like(inp["kvcache"])
    kv2[perm] = inp["kvcache"]
    inp2 = dict(inp, kvcache=kv2, block_table=perm[inp["block_table"]].astype(np.int32))
    o2, l2 = _run(ora, inp2)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2), "page relabelling changed output"


def pin_lse_extended(ora):
    inp = small_inputs([77, 200], h_q=4, seed=10)
    _, lse = _run(ora, inp)
    q = W.bf16_bits_to_f32(inp["q"]).astype(np.longdouble)
    kv = W.bf16_bits_to_f32(inp["kvcache"]).astype(np.longdouble)
    sc = np.longdouble(inp["softmax_scale"])
    for b in range(2):
        L = int(inp["cache_seqlens"][b])
        t = np.arange(L)
        K = kv[inp["block_table"][b][t // W.PAGE], t % W.PAGE, 0]
        for h in range(4):
            s = sc * (K @ q[b, 0, h])
            m = s.max()
            want = m + np.log(np.sum(np.exp(s - m)))
            _close(lse[b, h, 0], float(want), what="lse extended")


def pin_zero_scale(ora):
    inp = small_inputs([33, 64, 65], s_q=2, h_q=4, causal=True, seed=11, scale=0.0)
    o, lse = _run(ora, inp)
    kv = W.bf16_bits_to_f32(inp["kvcache"]).astype(np.float64)
    for b, L in enumerate(inp["cache_seqlens"]):
        for i in range(2):
            n = int(L) - 2 + i + 1
            t = np.arange(n)
            V = kv[inp["block_table"][b][t // W.PAGE], t % W.PAGE, 0, :W.D_V]
            for h in range(4):
                _close(o[b, i, h], V.mean(axis=0), tol=1e-13, what="zero-scale mean")
                _close(lse[b, h, i], math.log(n), tol=1e-13, what="zero-scale lse")


def pin_causal_reduction(ora):
    s_q = 3
    inp = small_inputs([70, 129, 3], s_q=s_q, h_q=4, causal=True, seed=12)
    o, lse = _run(ora, inp)
    for i in range(s_q):
        lens = np.maximum(inp["cache_seqlens"] - (s_q - 1 - i), 0).astype(np.int32)
        one = dict(inp, q=np.ascontiguousarray(inp["q"][:, i:i + 1]), s_q=1, causal=False,
                   cache_seqlens=lens)
        o1, l1 = _run(ora, one)
        assert np.array_equal(o[:, i], o1[:, 0]), f"causal row {i} != shortened one-token call"
        assert np.array_equal(lse[:, :, i], l1[:, :, 0]), f"causal lse row {i}"


def pin_split_merge(ora):
    inp = small_inputs([300, 65, 2], h_q=4, seed=13)
    o, lse = _run(ora, inp)
    rng = np.random.default_rng(5)
    b = len(inp["cache_seqlens"])
    cuts = []
    for L in inp["cache_seqlens"]:
        inner = sorted(rng.choice(np.arange(1, max(int(L), 2)), size=min(3, max(int(L) - 1, 0)),
                              replace=False).tolist()) if L > 1 else []
        cuts.append([0] + inner + [int(L)])
    npieces = max(len(c) - 1 for c in cuts)
    parts = []
    for k in range(npieces):
        # piece k of each sequence; sequences with fewer pieces get an empty window
        lo = np.array([c[k] if k < len(c) - 1 else c[-1] for c in cuts], np.int32)
        hi = np.array([c[k + 1] if k < len(c) - 1 else c[-1] for c in cuts], np.int32)
        parts.append(_run(ora, inp, key_lo=lo, key_hi=hi))
    for bi in range(b):
        for h in range(4):
            po = np.stack([p[0][bi, 0, h] for p in parts])
            pl = np.array([p[1][bi, h, 0] for p in parts])
            mo, ml = ora.mla_combine(po, pl)
            _close(mo, o[bi, 0, h], what="split+merge o")
            _close(ml, lse[bi, h, 0], what="split+merge lse")


def pin_empty_rows(ora):
    inp = small_inputs([0, 1, 2], s_q=3, h_q=2, causal=True, seed=14)
    o, lse = _run(ora, inp)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0])), "L=0 must give o=0, lse=-inf"
    # L=1, s_q=3: query rows 0,1 see nothing; row 2 sees token 0
    assert np.all(o[1, :2] == 0) and np.all(np.isneginf(lse[1, :, :2]))
    assert np.all(np.isfinite(lse[1, :, 2]))
    assert np.all(np.isneginf(lse[2, :, 0])) and np.all(np.isfinite(lse[2, :, 1:]))


def pin_combine_closed_form(ora):
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal(16), rng.standard_normal(16)
    o, l = ora.mla_combine(np.stack([a, b]), np.array([0.25, 0.25]))
    _close(o, (a + b) / 2, what="combine equal weights")
    _close(l, 0.25 + math.log(2.0), what="combine lse")
    o, l = ora.mla_combine(np.stack([a, b]), np.array([1.5, -np.inf]))
    _close(o, a, what="combine with empty partial")
    _close(l, 1.5, what="combine lse with empty partial")
    o, l = ora.mla_combine(np.stack([a, b]), np.array([-np.inf, -np.inf]))
    assert np.all(o == 0) and l == -np.inf
    # weights exp(lse_k - lse) for lse = (0, log 3): 1/4 and 3/4
    o, l = ora.mla_combine(np.stack([a, b]), np.array([0.0, math.log(3.0)]))
    _close(o, 0.25 * a + 0.75 * b, what="combine 1:3")
    _close(l, math.log(4.0), what="combine lse 1:3")


def _gather_rows(kvcache, block_table, b, lo, hi):
    """Rows [lo, hi) of sequence b, gathered through the block table with numpy."""
    page = kvcache.shape[1]
    t = np.arange(lo, hi)
    return kvcache[block_table[b][t // page], t % page]


def pin_append_readback(ora):
    # new rows read back through the block table; every other byte unchanged;
    # a page boundary is crossed (62 + 5) and one sequence starts empty
    rng = np.random.default_rng(21)
    lens = np.array([62, 0, 130], dtype=np.int32)
    s_new, h_kv, page = 5, 2, 64
    need = (lens + s_new + page - 1) // page          # pages per sequence after the append
    pool = int(need.sum()) + 3
    perm = rng.permutation(pool).astype(np.int32)
    bt = np.zeros((3, int(need.max()) + 1), dtype=np.int32)
    k = 0
    for b in range(3):
        bt[b, :need[b]] = perm[k:k + need[b]]
        k += int(need[b])
    kv = rng.integers(0, 1 << 16, size=(pool, page, h_kv, W.D_QK), dtype=np.uint16)
    new = rng.integers(0, 1 << 16, size=(3, s_new, h_kv, W.D_QK), dtype=np.uint16)
    out, ok = ora.append_kvcache(new, bt, lens, kv)
    assert ok
    touched = np.zeros(kv.shape[:2], dtype=bool)
    for b in range(3):
        L = int(lens[b])
        assert np.array_equal(_gather_rows(out, bt, b, L, L + s_new), new[b]), f"sequence {b}"
        t = np.arange(L, L + s_new)
        touched[bt[b][t // page], t % page] = True
    assert np.array_equal(out[~touched], kv[~touched]), "rows outside the append changed"


def pin_append_then_decode(ora):
    # truncate a sequence by s_new tokens (garbage in their rows), append the true
    # rows back: the cache is restored bit for bit and so is the decode
    inp = small_inputs([200, 77], h_q=4, seed=22)
    s_new = 3
    L_full = inp["cache_seqlens"].copy()
    L_prev = L_full - s_new
    new = np.stack([_gather_rows(inp["kvcache"], inp["block_table"], b, int(L_prev[b]), int(L_full[b]))
                    for b in range(2)])
    damaged = inp["kvcache"].copy()
    rng = np.random.default_rng(22)
    for b in range(2):
        t = np.arange(int(L_prev[b]), int(L_full[b]))
        damaged[inp["block_table"][b][t // 64], t % 64] = rng.integers(0, 1 << 16, size=(s_new, 1, W.D_QK))
    out, ok = ora.append_kvcache(new, inp["block_table"], L_prev, damaged)
    assert ok and np.array_equal(out, inp["kvcache"]), "append did not restore the cache"
    o1, l1 = _run(ora, inp)
    o2, l2 = _run(ora, dict(inp, kvcache=out))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_append_overflow(ora):
    # a position past the block table is rejected and writes nothing
    inp = small_inputs([120], h_q=2, seed=23)
    bt = inp["block_table"][:, :2].copy()  # room for 128 tokens
    new = np.full((1, 10, 1, W.D_QK), 7, dtype=np.uint16)
    out, ok = ora.append_kvcache(new, bt, inp["cache_seqlens"], inp["kvcache"])
    assert not ok
    got = _gather_rows(out, bt, 0, 120, 128)
    assert np.all(got == 7), "rows that fit must still be written"


def _mla_weights(h, seed):
    rng = np.random.default_rng(seed)
    w_uk = rng.standard_normal((h, 128, 512)) / math.sqrt(512)
    w_uv = rng.standard_normal((h, 128, 512)) / math.sqrt(512)
    return w_uk, w_uv


def pin_unabsorbed_bruteforce(ora):
    # per-head up-projected keys and values, written densely with numpy
    inp = small_inputs([70, 5], h_q=3, seed=31, s_q=2, causal=True)
    rng = np.random.default_rng(31)
    b, s_q, h = 2, 2, 3
    qn = rng.standard_normal((b, s_q, h, 128))
    qr = rng.standard_normal((b, s_q, h, 64))
    w_uk, w_uv = _mla_weights(h, 31)
    o, lse = ora.mla_decode_unabsorbed(qn, qr, w_uk, w_uv, inp["kvcache"], inp["block_table"],
                                       inp["cache_seqlens"], True, inp["softmax_scale"])
    for bb in range(b):
        L = int(inp["cache_seqlens"][bb])
        rows = W.bf16_bits_to_f32(_gather_rows(inp["kvcache"], inp["block_table"], bb, 0, L)[:, 0]).astype(np.float64)
        C, KR = rows[:, :512], rows[:, 512:]
        for i in range(s_q):
            last = L - s_q + i
            for hh in range(h):
                kC = C[:last + 1] @ w_uk[hh].T
                v = C[:last + 1] @ w_uv[hh].T
                sc = inp["softmax_scale"] * (kC @ qn[bb, i, hh] + KR[:last + 1] @ qr[bb, i, hh])
                m = sc.max()
                p = np.exp(sc - m)
                assert np.allclose(o[bb, i, hh], (p / p.sum()) @ v, rtol=0, atol=1e-10)
                assert abs(lse[bb, hh, i] - (m + math.log(p.sum()))) < 1e-10


def pin_unabsorbed_equals_absorbed_route(ora):
    # W^UK = [I | 0] makes the absorbed query [q^C, 0, ..] exact in bf16, so the latent
    # decode oracle applies; W^UV times its output must equal the unabsorbed result
    inp = small_inputs([130, 40], h_q=2, seed=32)
    b, h = 2, 2
    q = inp["q"].copy()
    q[..., 128:512] = 0                    # latent query beyond the first 128 dims
    qn = W.bf16_bits_to_f32(q[..., :128]).astype(np.float64)
    qr = W.bf16_bits_to_f32(q[..., 512:]).astype(np.float64)
    w_uk = np.zeros((h, 128, 512))
    w_uk[:, np.arange(128), np.arange(128)] = 1.0
    _, w_uv = _mla_weights(h, 32)
    o_lat, lse_lat = _run(ora, dict(inp, q=q))
    o, lse = ora.mla_decode_unabsorbed(qn, qr, w_uk, w_uv, inp["kvcache"], inp["block_table"],
                                       inp["cache_seqlens"], False, inp["softmax_scale"])
    assert np.allclose(o, np.einsum("bshk,hrk->bshr", o_lat, w_uv), rtol=0, atol=1e-10)
    assert np.allclose(lse, lse_lat, rtol=0, atol=1e-10)


def pin_closed_form_golden(ora):
    # the worked examples of golden/closed_form_cases.txt (answers in closed form,
    # derivation in the file) to 1e-12
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_form_cases.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 4
    kv = np.zeros((1, 64, 1, W.D_QK), dtype=np.float32)
    kv[0, 0, 0, :512] = 1.0
    kv[0, 1, 0, :512] = 2.0
    kv[0, 1, 0, 512] = 1.0
    kv_bits = W.f32_to_bf16_bits(kv)
    for name, s_q, causal, scale, qi, lse_ref, o_ref in rows:
        s_q, causal, qi = int(s_q), bool(int(causal)), int(qi)
        q = np.zeros((1, s_q, 1, W.D_QK), dtype=np.float32)
        q[..., 512] = 1.0
        o, lse = ora.mla_decode(W.f32_to_bf16_bits(q), kv_bits, np.zeros((1, 1), np.int32),
                                np.array([2], np.int32), W.D_V, causal, float(scale))
        assert abs(lse[0, 0, qi] - float(lse_ref)) < 1e-12, name
        assert np.all(np.abs(o[0, qi, 0] - float(o_ref)) < 1e-12), name


ALL_PINS = [pin_bruteforce, pin_single_token, pin_equal_values, pin_page_permutation,
            pin_lse_extended, pin_zero_scale, pin_causal_reduction, pin_split_merge,
            pin_empty_rows, pin_combine_closed_form, pin_append_readback, pin_append_then_decode,
            pin_append_overflow, pin_unabsorbed_bruteforce, pin_unabsorbed_equals_absorbed_route,
            pin_closed_form_golden]

"""Helpers for the GPU parity tests: upload seeded inputs, run the library
through its Python binding (which calls the C ABI), compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import mla_workloads as W

# Parity bar for floating-point outputs (bf16 inputs, fp32 accumulation, bf16 o).
O_ATOL = 1e-2          # max |o_gpu - o_oracle|
COS_MIN = 0.99999      # cosine similarity of o over the whole tensor
LSE_ATOL = 1e-3        # max |lse_gpu - lse_oracle|


def to_device(inp: dict, device="cuda") -> dict:
    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return dict(q=bf(inp["q"]), kvcache=bf(inp["kvcache"]),
                block_table=torch.from_numpy(inp["block_table"]).to(device),
                cache_seqlens=torch.from_numpy(inp["cache_seqlens"]).to(device))


def run_gpu(inp: dict, device="cuda", dev_inputs: dict | None = None):
    import paged_mla_attention_b200 as pm
    d = dev_inputs if dev_inputs is not None else to_device(inp, device)
    meta, splits = pm.get_mla_metadata(d["cache_seqlens"], inp["s_q"] * inp["h_q"] // inp["h_kv"],
                                       inp["h_kv"])
    o, lse = pm.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"],
                                       W.D_V, meta, splits, softmax_scale=inp["softmax_scale"],
                                       causal=inp["causal"])
    torch.cuda.synchronize()
    err = pm.device_error()
    assert err == 0, f"device error word {err}"
    return (o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
            meta.cpu().numpy(), splits.cpu().numpy())


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    assert o_gpu.shape == o_ref.shape and lse_gpu.shape == lse_ref.shape
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite o"
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ninf_ref), f"{what}: -inf lse pattern differs"
    assert not np.isnan(lse_gpu).any(), f"{what}: NaN lse"
    d_o = float(np.abs(o_gpu - o_ref).max()) if o_ref.size else 0.0
    with np.errstate(invalid="ignore"):
        d_l = float(np.abs(np.where(ninf_ref, 0, lse_gpu - lse_ref)).max()) if lse_ref.size else 0.0
    a, b = o_gpu.ravel(), o_ref.ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    cos = 1.0 if (na == 0 and nb == 0) else float(a @ b / (na * nb))
    stats = dict(max_do=d_o, max_dlse=d_l, cos=cos, max_o=float(np.abs(o_ref).max()) if o_ref.size else 0.0)
    assert d_o <= O_ATOL, f"{what}: max|do| {d_o:.3e} > {O_ATOL} ({stats})"
    assert cos >= COS_MIN, f"{what}: cosine {cos:.7f} < {COS_MIN} ({stats})"
    assert d_l <= LSE_ATOL, f"{what}: max|dlse| {d_l:.3e} > {LSE_ATOL} ({stats})"
    return stats


def subset(inp: dict, seqs, heads=None) -> dict:
    """The same problem restricted to some sequences (and query heads, h_kv == 1)."""
    seqs = np.asarray(seqs)
    out = dict(inp)
    q = inp["q"][seqs]
    if heads is not None:
        assert inp["h_kv"] == 1
        q = q[:, :, np.asarray(heads)]
        out["h_q"] = len(heads)
    out["q"] = np.ascontiguousarray(q)
    out["block_table"] = np.ascontiguousarray(inp["block_table"][seqs])
    out["cache_seqlens"] = np.ascontiguousarray(inp["cache_seqlens"][seqs])
    out["batch"] = len(seqs)
    return out


def check_schedule(meta, splits, seqlens, num_parts):
    """Invariants of the scheduler output (no numeric oracle exists for it):
    every page of every sequence is covered by exactly one part, in order;
    num_splits is the exclusive prefix sum of pieces; piece ordinals match;
    and no part costs more than the scheduler's stated bound."""
    seqlens = np.asarray(seqlens, dtype=np.int64)
    n = (np.maximum(seqlens, 0) + 63) // 64
    batch = len(n)
    assert meta.shape == (num_parts, 8) and splits.shape == (batch + 1,)
    assert splits[0] == 0
    pieces = np.zeros(batch, dtype=np.int64)
    covered = [np.zeros(int(x), dtype=np.int64) for x in n]
    loads = []
    prev_end = (0, 0)
    for p in range(num_parts):
        b0, pg0, b1, pg1, ord0 = [int(x) for x in meta[p, :5]]
        assert (b0, pg0) == prev_end or (b0 >= batch), f"part {p} does not start where {p-1} ended"
        assert (b0, pg0) <= (b1, pg1)
        load = 0
        for b in range(b0, min(b1, batch - 1) + 1):
            s = pg0 if b == b0 else 0
            e = pg1 if b == b1 else int(n[b])
            if s >= e:
                continue
            if b == b0:
                assert ord0 == pieces[b], f"part {p}: ordinal {ord0} != {pieces[b]}"
            covered[b][s:e] += 1
            pieces[b] += 1
            load += (e - s) + 3
        loads.append(load)
        prev_end = (b1, pg1) if b1 < batch else (batch, 0)
    for b in range(batch):
        assert np.all(covered[b] == 1), f"sequence {b}: pages not covered exactly once"
    assert np.array_equal(np.diff(splits), pieces), "num_splits is not the prefix sum of pieces"
    # balance: the scheduler's guarantee -- no part costs more than its weight's
    # share of the total plus one overhead per possible cut, plus one piece's
    # overhead and two pages of snapping.  Weights (column 5) are 128, or one
    # smaller weight for the trailing parts that run on the SMs left free by
    # 4-CTA clusters.
    w = [int(x) for x in meta[:, 5]]
    assert len(set(w) - {128}) <= 1 and all(0 < x <= 128 for x in w), f"part weights {sorted(set(w))}"
    assert w == sorted(w, reverse=True), "the lighter parts must come last"
    assert np.all(meta[:, 6:] == 0)
    total = int(sum(int(x) + 3 for x in n if x > 0))
    A, W = total + (num_parts - 1) * 3, sum(w)
    for p, load in enumerate(loads):
        bound = -(-(w[p] * A) // W) + 3 + 2
        assert load <= bound, f"unbalanced part {p}: {load} > {bound} (weight {w[p]}, mean {sum(loads) / num_parts:.1f})"
    return loads

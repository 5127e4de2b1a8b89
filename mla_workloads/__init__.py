"""Seeded synthetic inputs for paged MLA decoding.

This module only draws inputs: it holds none of the attention arithmetic, so
both the fp64 oracle and the CUDA path can take their inputs from here without
sharing any of the method's code.

Shapes follow the decode interface of FlashMLA as the DeepSeek FlashMLA pages
state it (usage, steps 2-4: ``cache_seqlens``, ``q``, ``kvcache``,
``block_table``; 64-token pages):

* ``q``           bf16 ``[batch][s_q][h_q][576]``   (512 latent + 64 RoPE dims)
* ``kvcache``     bf16 ``[num_pages][64][h_kv][576]``
* ``block_table`` int32 ``[batch][max_pages]`` (logical page -> physical page)
* ``cache_seqlens`` int32 ``[batch]``

bf16 values are carried as ``uint16`` bit patterns (numpy has no bf16), made by
round-to-nearest-even from float32 draws of N(0, 1).

Draw order for a seed: sequence lengths, then the physical-page permutation,
then q, then the kv cache.  Pages are handed to sequences in order from the
permutation; block-table entries past a sequence's last page are 0.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

PAGE = 64          # tokens per KV page
D_QK = 576         # 512 latent (c^KV) + 64 RoPE (k^R)
D_V = 512          # value width: the latent part of the same cached row
SCALE_192 = 1.0 / math.sqrt(192.0)


@dataclasses.dataclass
class Workload:
    """A named decode configuration (sizes and the length recipe)."""

    name: str
    batch: int
    s_q: int
    h_q: int
    h_kv: int
    causal: bool
    seqlen_kind: str            # "fixed", "uniform", "lognormal", "skew", "explicit"
    seqlen_args: tuple
    pool_pages: Optional[int] = None   # None: exactly the pages the lengths need
    seed: int = 0
    softmax_scale: float = SCALE_192

    def describe(self) -> str:
        return (f"{self.name}: batch={self.batch} s_q={self.s_q} h_q={self.h_q} h_kv={self.h_kv} "
                f"causal={self.causal} lengths={self.seqlen_kind}{self.seqlen_args}")


# The five decode configurations, in order.  The seed of each is its 1-based index.
WORKLOADS = {
    "tiny": Workload("tiny", 2, 1, 16, 1, False, "explicit", ((37, 130),), pool_pages=8, seed=1),
    "uniform": Workload("uniform", 64, 1, 128, 1, False, "fixed", (4096,), seed=2),
    "varlen": Workload("varlen", 128, 1, 128, 1, False, "lognormal", (2048.0, 1.0, 1, 32768), seed=3),
    "causal2": Workload("causal2", 128, 2, 128, 1, True, "uniform", (1024, 8192), seed=4),
    "skew": Workload("skew", 16, 1, 128, 1, False, "skew", (131072, 64, 4096), seed=5),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def draw_seqlens(w: Workload, rng: np.random.Generator) -> np.ndarray:
    k, a = w.seqlen_kind, w.seqlen_args
    if k == "explicit":
        lens = np.asarray(a[0], dtype=np.int64)
    elif k == "fixed":
        lens = np.full(w.batch, a[0], dtype=np.int64)
    elif k == "uniform":
        lens = rng.integers(a[0], a[1], size=w.batch, endpoint=True)
    elif k == "lognormal":
        median, sigma, lo, hi = a
        lens = np.clip(np.rint(np.exp(rng.normal(math.log(median), sigma, size=w.batch))), lo, hi)
    elif k == "skew":
        longest, lo, hi = a
        lens = np.concatenate([[longest], rng.integers(lo, hi, size=w.batch - 1, endpoint=True)])
    else:
        raise ValueError(k)
    assert lens.shape == (w.batch,)
    return lens.astype(np.int32)


def _normal_bf16(rng: np.random.Generator, n: int, chunk: int = 1 << 24) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        out[s:e] = f32_to_bf16_bits(rng.standard_normal(e - s, dtype=np.float32))
    return out


def make_inputs(w: Workload, seed: Optional[int] = None, seqlens: Optional[Sequence[int]] = None,
                extra_pages: int = 0, pool_pages: Optional[int] = None) -> dict:
    """Draw one seeded input set for workload ``w``.

    ``seqlens`` overrides the length recipe (used by edge-case tests);
    ``extra_pages`` adds unused noise pages to the pool.
    Returns a dict of numpy arrays plus the scalar arguments.
    """
    rng = np.random.default_rng(w.seed if seed is None else seed)
    lens = draw_seqlens(w, rng) if seqlens is None else np.asarray(seqlens, dtype=np.int32)
    batch = int(lens.shape[0])
    n_pages = (lens.astype(np.int64) + PAGE - 1) // PAGE
    need = int(n_pages.sum())
    pool = pool_pages if pool_pages is not None else (w.pool_pages if (w.pool_pages and seqlens is None) else need)
    pool = max(pool, need, 1) + extra_pages
    perm = rng.permutation(pool).astype(np.int32)
    max_pages = max(int(n_pages.max()) if batch else 1, 1)
    block_table = np.zeros((batch, max_pages), dtype=np.int32)
    cursor = 0
    for b in range(batch):
        n = int(n_pages[b])
        block_table[b, :n] = perm[cursor:cursor + n]
        cursor += n
    q = _normal_bf16(rng, batch * w.s_q * w.h_q * D_QK).reshape(batch, w.s_q, w.h_q, D_QK)
    kv = _normal_bf16(rng, pool * PAGE * w.h_kv * D_QK).reshape(pool, PAGE, w.h_kv, D_QK)
    return dict(q=q, kvcache=kv, block_table=block_table, cache_seqlens=lens,
                batch=batch, s_q=w.s_q, h_q=w.h_q, h_kv=w.h_kv, d=D_QK, dv=D_V,
                causal=bool(w.causal), softmax_scale=float(w.softmax_scale),
                num_pages=pool, max_pages=max_pages)

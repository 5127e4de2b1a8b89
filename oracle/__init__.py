"""fp64 CPU oracle for paged MLA decoding (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference arms may import this package.  The product path never does: it has
no CPU fallback, and this oracle shares no code with it.

The arithmetic lives in ``mla_oracle.c`` (plain loops in double precision,
OpenMP over query rows); this module compiles it with gcc on first use and
marshals numpy arrays through ctypes.  See the C file for the definition it
follows and the readings it takes where the pages leave a step open.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute-force dense attention, closed forms, invariances, split invariance),
and ``tests/test_oracle_mutants.py`` checks that planted mistakes fail a pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "mla_oracle.c")
LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Compile the oracle shared library (gcc -O2, OpenMP, strict IEEE double)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleLib:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.oracle_mla_decode.argtypes = [P] * 6 + [I] * 9 + [ctypes.c_double, P, P, I]
        lib.oracle_mla_decode.restype = I
        lib.oracle_mla_combine.argtypes = [P, P, I, I, P, P]
        lib.oracle_mla_combine.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        lib.oracle_append_kvcache.argtypes = [P, P, P] + [I] * 7 + [P]
        lib.oracle_append_kvcache.restype = I
        lib.oracle_mla_decode_unabsorbed.argtypes = [P] * 7 + [I] * 6 + [ctypes.c_double, P, P, I]
        lib.oracle_mla_decode_unabsorbed.restype = I
        self.lib = lib
        self.path = path

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def mla_decode(self, q: np.ndarray, kvcache: np.ndarray, block_table: np.ndarray,
                   cache_seqlens: np.ndarray, dv: int, causal: bool, softmax_scale: float,
                   key_lo: Optional[np.ndarray] = None, key_hi: Optional[np.ndarray] = None,
                   nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
        """Reference decode.

        q: uint16 bf16 bits [b][s_q][h_q][d]; kvcache: uint16 [pages][page][h_kv][d];
        block_table: int32 [b][max_pages]; cache_seqlens: int32 [b].
        Returns (o float64 [b][s_q][h_q][dv], lse float64 [b][h_q][s_q]).
        key_lo / key_hi restrict each sequence's keys to [lo, hi) (partial results).
        """
        q = np.ascontiguousarray(q, dtype=np.uint16)
        kvcache = np.ascontiguousarray(kvcache, dtype=np.uint16)
        block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        cache_seqlens = np.ascontiguousarray(cache_seqlens, dtype=np.int32)
        b, s_q, h_q, d = q.shape
        _, page, h_kv, d2 = kvcache.shape
        assert d2 == d and block_table.shape[0] == b and cache_seqlens.shape == (b,)
        lo = None if key_lo is None else np.ascontiguousarray(key_lo, dtype=np.int32)
        hi = None if key_hi is None else np.ascontiguousarray(key_hi, dtype=np.int32)
        o = np.zeros((b, s_q, h_q, dv), dtype=np.float64)
        lse = np.zeros((b, h_q, s_q), dtype=np.float64)
        rc = self.lib.oracle_mla_decode(
            _ptr(q), _ptr(kvcache), _ptr(block_table), _ptr(cache_seqlens), _ptr(lo), _ptr(hi),
            b, s_q, h_q, h_kv, d, dv, page, block_table.shape[1], int(bool(causal)),
            float(softmax_scale), _ptr(o), _ptr(lse), int(nthreads))
        if rc != 0:
            raise ValueError("oracle_mla_decode rejected its arguments")
        return o, lse

    def mla_combine(self, part_o: np.ndarray, part_lse: np.ndarray) -> Tuple[np.ndarray, float]:
        """Merge partial results of one query row: part_o [n][dv], part_lse [n]."""
        part_o = np.ascontiguousarray(part_o, dtype=np.float64)
        part_lse = np.ascontiguousarray(part_lse, dtype=np.float64)
        n, dv = part_o.shape
        o = np.zeros(dv, dtype=np.float64)
        lse = np.zeros(1, dtype=np.float64)
        self.lib.oracle_mla_combine(_ptr(part_o), _ptr(part_lse), n, dv, _ptr(o), _ptr(lse))
        return o, float(lse[0])

    def append_kvcache(self, new_kv: np.ndarray, block_table: np.ndarray, cache_seqlens: np.ndarray,
                       kvcache: np.ndarray) -> Tuple[np.ndarray, bool]:
        """Reference append: returns (a new cache with the tokens written, all rows written?).

        new_kv: uint16 bf16 bits [b][s_new][h_kv][d]; kvcache: uint16 [pages][page][h_kv][d]
        (not modified); cache_seqlens: lengths before the append.
        """
        new_kv = np.ascontiguousarray(new_kv, dtype=np.uint16)
        out = np.array(kvcache, dtype=np.uint16, copy=True, order="C")
        block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        cache_seqlens = np.ascontiguousarray(cache_seqlens, dtype=np.int32)
        b, s_new, h_kv, d = new_kv.shape
        pages, page, h_kv2, d2 = out.shape
        assert h_kv2 == h_kv and d2 == d and block_table.shape[0] == b
        rc = self.lib.oracle_append_kvcache(_ptr(new_kv), _ptr(block_table), _ptr(cache_seqlens), b,
                                            s_new, h_kv, d, page, block_table.shape[1], pages, _ptr(out))
        return out, rc == 0

    def mla_decode_unabsorbed(self, q_nope: np.ndarray, q_rope: np.ndarray, w_uk: np.ndarray,
                              w_uv: np.ndarray, kvcache: np.ndarray, block_table: np.ndarray,
                              cache_seqlens: np.ndarray, causal: bool,
                              softmax_scale: float) -> Tuple[np.ndarray, np.ndarray]:
        """Per-head up-projected attention (h_kv = 1): q_nope [b][s_q][h][128], q_rope
        [b][s_q][h][64], w_uk and w_uv [h][128][512] (float64); kvcache uint16 bf16 bits.
        Returns (o float64 [b][s_q][h][128], lse float64 [b][h][s_q])."""
        q_nope = np.ascontiguousarray(q_nope, dtype=np.float64)
        q_rope = np.ascontiguousarray(q_rope, dtype=np.float64)
        w_uk = np.ascontiguousarray(w_uk, dtype=np.float64)
        w_uv = np.ascontiguousarray(w_uv, dtype=np.float64)
        kvcache = np.ascontiguousarray(kvcache, dtype=np.uint16)
        block_table = np.ascontiguousarray(block_table, dtype=np.int32)
        cache_seqlens = np.ascontiguousarray(cache_seqlens, dtype=np.int32)
        b, s_q, h, _ = q_nope.shape
        assert kvcache.shape[2] == 1 and kvcache.shape[3] == 576
        o = np.zeros((b, s_q, h, 128), dtype=np.float64)
        lse = np.zeros((b, h, s_q), dtype=np.float64)
        rc = self.lib.oracle_mla_decode_unabsorbed(
            _ptr(q_nope), _ptr(q_rope), _ptr(w_uk), _ptr(w_uv), _ptr(kvcache), _ptr(block_table),
            _ptr(cache_seqlens), b, s_q, h, kvcache.shape[1], block_table.shape[1], int(bool(causal)),
            float(softmax_scale), _ptr(o), _ptr(lse), 0)
        if rc != 0:
            raise ValueError("oracle_mla_decode_unabsorbed rejected its arguments")
        return o, lse

    def decode_inputs(self, inp: dict, nthreads: int = 0, **kw) -> Tuple[np.ndarray, np.ndarray]:
        """Run on an input dict from ``mla_workloads.make_inputs``."""
        return self.mla_decode(inp["q"], inp["kvcache"], inp["block_table"],
                               inp["cache_seqlens"], inp["dv"], inp["causal"],
                               inp["softmax_scale"], nthreads=nthreads, **kw)


_default: Optional[OracleLib] = None


def default() -> OracleLib:
    global _default
    if _default is None:
        _default = OracleLib(build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def mla_decode(*a, **kw):
    return default().mla_decode(*a, **kw)


def mla_combine(*a, **kw):
    return default().mla_combine(*a, **kw)


def append_kvcache(*a, **kw):
    return default().append_kvcache(*a, **kw)


def decode_inputs(inp: dict, nthreads: int = 0, **kw):
    return default().decode_inputs(inp, nthreads=nthreads, **kw)

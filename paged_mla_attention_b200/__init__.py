"""B200-native paged MLA decode: Python binding of libpagedmla.so.

The two calls mirror the FlashMLA usage the DeepSeek pages show (usage steps
3-4):

    tile_scheduler_metadata, num_splits = get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv)
    o, lse = flash_mla_with_kvcache(q, kvcache, block_table, cache_seqlens, dv,
                                    tile_scheduler_metadata, num_splits, causal=True)

Around them: ``append_kvcache`` (new tokens into their pages), ``PagePool`` (host
page allocator), ``absorb_query`` / ``project_output`` (the absorbed W^UK / W^UV
projections), ``metadata_sizes`` / ``workspace_bytes`` and ``device_error``.

This module only marshals arguments: it checks tensor dtypes/devices, allocates
the outputs and the split workspace with torch, and passes raw device pointers
and the current CUDA stream to the C ABI (``include/pagedmla.h``).  Every step
of the computation runs in the library's sm_100a kernels; there is no CPU or
PyTorch fallback, and importing this module fails loudly if the library has not
been built.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import numpy as np
import torch

__all__ = ["get_mla_metadata", "flash_mla_with_kvcache", "metadata_sizes", "workspace_bytes",
           "append_kvcache", "PagePool", "absorb_query", "project_output", "device_error", "library",
           "LIB_PATH", "PmlaError", "DEFAULT_SOFTMAX_SCALE"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedmla.so")
PAGE_SIZE = 64
HEAD_DIM = 576
HEAD_DIM_V = 512
METADATA_INTS = 8
# 1 / sqrt(d_h + d_h^R) with d_h = 128, d_h^R = 64: the scale in the MLA
# attention equation of the FlashMLA overview, section 2.2.
DEFAULT_SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)

ERRORS = {-1: "invalid argument", -2: "unsupported", -3: "alignment", -4: "CUDA error",
          -5: "workspace", -6: "device error", -7: "page pool exhausted"}


class PmlaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"pagedmla error {code} ({ERRORS.get(code, '?')}): {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m paged_mla_attention_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.mla_get_metadata_sizes.argtypes = [I, I, I, ctypes.POINTER(I), ctypes.POINTER(SZ)]
    lib.mla_get_metadata_sizes.restype = I
    lib.mla_get_metadata.argtypes = [P, I, I, I, P, I, P, P]
    lib.mla_get_metadata.restype = I
    for name in ("mla_decode_with_kvcache", "mla_decode_splits", "mla_merge_splits"):
        fn = getattr(lib, name)
        fn.argtypes = [P, P, P, P] + [I] * 8 + [P, I, P, I, ctypes.c_float, P, P, P, SZ, P]
        fn.restype = I
    lib.pmla_page_pool_create.argtypes = [I, ctypes.POINTER(P)]
    lib.pmla_page_pool_create.restype = I
    lib.pmla_page_pool_destroy.argtypes = [P]
    lib.pmla_page_pool_destroy.restype = None
    lib.pmla_page_pool_num_free.argtypes = [P]
    lib.pmla_page_pool_num_free.restype = I
    lib.pmla_page_pool_alloc.argtypes = [P, I, P]
    lib.pmla_page_pool_alloc.restype = I
    lib.pmla_page_pool_free.argtypes = [P, I, P]
    lib.pmla_page_pool_free.restype = I
    lib.pmla_page_pool_grow_sequence.argtypes = [P, P, I, I, I]
    lib.pmla_page_pool_grow_sequence.restype = I
    lib.pmla_page_pool_release_sequence.argtypes = [P, P, I]
    lib.pmla_page_pool_release_sequence.restype = I
    lib.mla_absorb_query.argtypes = [P, P, P, I, I, P, P]
    lib.mla_absorb_query.restype = I
    lib.mla_project_output.argtypes = [P, P, I, I, P, P]
    lib.mla_project_output.restype = I
    lib.mla_append_kvcache.argtypes = [P, P, P, I, I, I, I, P, I, I, P, P]
    lib.mla_append_kvcache.restype = I
    lib.pmla_device_error.argtypes = []
    lib.pmla_device_error.restype = I
    lib.pmla_last_error.argtypes = []
    lib.pmla_last_error.restype = ctypes.c_char_p
    lib.mla_get_last_error.argtypes = []
    lib.mla_get_last_error.restype = ctypes.c_char_p
    lib.pmla_version.argtypes = []
    lib.pmla_version.restype = ctypes.c_char_p
    return lib


class _Library:
    """The C library, loaded on first use (so that the build module, which lives
    in this package, can run before the library exists).  Any use raises
    ImportError when the library is missing: there is no fallback path."""

    _lib = None

    def __getattr__(self, name):
        if _Library._lib is None:
            _Library._lib = _load()
        return getattr(_Library._lib, name)


library = _Library()


def _check(rc: int) -> None:
    if rc != 0:
        raise PmlaError(rc, library.pmla_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def metadata_sizes(batch: int, num_heads_per_head_k: int, num_heads_k: int) -> Tuple[int, int]:
    """(num_parts, workspace_bytes) for this shape on the current device."""
    parts = ctypes.c_int(0)
    ws = ctypes.c_size_t(0)
    _check(library.mla_get_metadata_sizes(batch, num_heads_per_head_k, num_heads_k,
                                          ctypes.byref(parts), ctypes.byref(ws)))
    return parts.value, ws.value


def get_mla_metadata(cache_seqlens: torch.Tensor, num_heads_per_head_k: int,
                     num_heads_k: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Length-balanced split-KV schedule for one decode step.

    cache_seqlens: int32 [batch] on the GPU.  num_heads_per_head_k is
    s_q * h_q // h_kv and num_heads_k is h_kv.  Returns
    (tile_scheduler_metadata int32 [num_parts, 8], num_splits int32 [batch + 1]),
    both on the GPU, computed on the current stream without a host sync.
    """
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    batch = cache_seqlens.shape[0]
    with torch.cuda.device(cache_seqlens.device):
        parts, _ = metadata_sizes(batch, num_heads_per_head_k, num_heads_k)
        meta = torch.empty((parts, METADATA_INTS), dtype=torch.int32, device=cache_seqlens.device)
        splits = torch.empty((batch + 1,), dtype=torch.int32, device=cache_seqlens.device)
        _check(library.mla_get_metadata(_ptr(cache_seqlens), batch, num_heads_per_head_k,
                                        num_heads_k, _ptr(meta), parts, _ptr(splits),
                                        _stream_ptr(cache_seqlens.device)))
    return meta, splits


def flash_mla_with_kvcache(q: torch.Tensor, kvcache: torch.Tensor, block_table: torch.Tensor,
                           cache_seqlens: torch.Tensor, head_dim_v: int,
                           tile_scheduler_metadata: torch.Tensor, num_splits: torch.Tensor,
                           causal: bool = False, softmax_scale: Optional[float] = None, *,
                           out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                           workspace: Optional[torch.Tensor] = None, stage: str = "all"
                           ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Paged MLA decode.

    The positional order is the one of the FlashMLA usage call (usage step 4):
    q, kvcache, block_table, cache_seqlens, dv, tile_scheduler_metadata,
    num_splits, causal; softmax_scale follows it.

    q           bf16 [batch, s_q, h_q, 576]
    kvcache     bf16 [num_pages, 64, h_kv, 576]
    block_table int32 [batch, max_pages]
    cache_seqlens int32 [batch]
    head_dim_v  512
    causal      mask query token i of s_q to cached tokens j <= seqlen - s_q + i
    Returns o bf16 [batch, s_q, h_q, 512] and lse fp32 [batch, h_q, s_q] (natural log).
    softmax_scale defaults to 1/sqrt(192).  ``out`` and ``workspace`` (keyword
    only) may be passed to avoid per-call allocation.  ``stage`` selects the C entry point:
    "all" (mla_decode_with_kvcache), "decode" (mla_decode_splits, the decode
    kernel alone) or "merge" (mla_merge_splits, the merge kernel alone; pass the
    same ``out`` and ``workspace`` as the "decode" call).
    """
    fn = {"all": library.mla_decode_with_kvcache, "decode": library.mla_decode_splits,
          "merge": library.mla_merge_splits}.get(stage)
    if fn is None:
        raise ValueError(f"stage must be 'all', 'decode' or 'merge', got {stage!r}")
    _need(q, "q", torch.bfloat16, 4)
    _need(kvcache, "kvcache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    _need(tile_scheduler_metadata, "tile_scheduler_metadata", torch.int32, 2)
    _need(num_splits, "num_splits", torch.int32, 1)
    batch, s_q, h_q, d = q.shape
    num_pages, page, h_kv, d2 = kvcache.shape
    if page != PAGE_SIZE or d2 != d:
        raise ValueError(f"kvcache must be [num_pages, {PAGE_SIZE}, h_kv, {d}], got {tuple(kvcache.shape)}")
    if block_table.shape[0] != batch or cache_seqlens.shape[0] != batch or num_splits.shape[0] != batch + 1:
        raise ValueError("batch size mismatch between q, block_table, cache_seqlens, num_splits")
    if h_kv < 1 or h_q % h_kv:
        raise ValueError("h_q must be a multiple of h_kv")
    dev = q.device
    for name, t in (("kvcache", kvcache), ("block_table", block_table), ("cache_seqlens", cache_seqlens),
                    ("tile_scheduler_metadata", tile_scheduler_metadata), ("num_splits", num_splits)):
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, q on {dev}")
    scale = DEFAULT_SOFTMAX_SCALE if softmax_scale is None else float(softmax_scale)
    num_parts = tile_scheduler_metadata.shape[0]
    with torch.cuda.device(dev):
        _, ws_bytes = metadata_sizes(batch, s_q * (h_q // h_kv), h_kv)
        if out is None:
            o = torch.empty((batch, s_q, h_q, head_dim_v), dtype=torch.bfloat16, device=dev)
            lse = torch.empty((batch, h_q, s_q), dtype=torch.float32, device=dev)
        else:
            o, lse = out
        if workspace is None or workspace.numel() < ws_bytes:
            workspace = torch.empty((max(ws_bytes, 16),), dtype=torch.uint8, device=dev)
        _check(fn(
            _ptr(q), _ptr(kvcache), _ptr(block_table), _ptr(cache_seqlens), batch, s_q, h_q, h_kv,
            d, head_dim_v, num_pages, block_table.shape[1], _ptr(tile_scheduler_metadata), num_parts,
            _ptr(num_splits), int(bool(causal)), scale, _ptr(o), _ptr(lse), _ptr(workspace),
            workspace.numel(), _stream_ptr(dev)))
    return o, lse


def append_kvcache(new_kv: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
                   kvcache: torch.Tensor, new_seqlens: Optional[torch.Tensor] = None) -> Optional[torch.Tensor]:
    """Write new tokens into the paged cache in place (mla_append_kvcache).

    new_kv      bf16 [batch, s_new, h_kv, 576]
    block_table int32 [batch, max_pages] (pages already assigned for the new positions)
    cache_seqlens int32 [batch], lengths before the append
    kvcache     bf16 [num_pages, 64, h_kv, 576], modified in place
    new_seqlens optional int32 [batch] out: cache_seqlens + s_new (returned).
    """
    _need(new_kv, "new_kv", torch.bfloat16, 4)
    _need(kvcache, "kvcache", torch.bfloat16, 4)
    _need(block_table, "block_table", torch.int32, 2)
    _need(cache_seqlens, "cache_seqlens", torch.int32, 1)
    batch, s_new, h_kv, d = new_kv.shape
    num_pages, page, h_kv2, d2 = kvcache.shape
    if page != PAGE_SIZE or h_kv2 != h_kv or d2 != d:
        raise ValueError(f"kvcache {tuple(kvcache.shape)} does not match new_kv {tuple(new_kv.shape)}")
    if block_table.shape[0] != batch or cache_seqlens.shape[0] != batch:
        raise ValueError("batch size mismatch between new_kv, block_table and cache_seqlens")
    dev = new_kv.device
    for name, t in (("kvcache", kvcache), ("block_table", block_table), ("cache_seqlens", cache_seqlens)):
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, new_kv on {dev}")
    if new_seqlens is not None:
        _need(new_seqlens, "new_seqlens", torch.int32, 1)
    with torch.cuda.device(dev):
        _check(library.mla_append_kvcache(_ptr(new_kv), _ptr(block_table), _ptr(cache_seqlens), batch, s_new,
                                          h_kv, d, _ptr(kvcache), num_pages, block_table.shape[1],
                                          _ptr(new_seqlens) if new_seqlens is not None else None,
                                          _stream_ptr(dev)))
    return new_seqlens


def absorb_query(q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk: torch.Tensor,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Absorbed 576-wide query: [W^UK_h^T q_nope (512) ; q_rope (64)] per token and head.

    q_nope bf16 [T, H, 128], q_rope bf16 [T, H, 64], w_uk bf16 [H, 128, 512] -> bf16 [T, H, 576].
    """
    _need(q_nope, "q_nope", torch.bfloat16, 3)
    _need(q_rope, "q_rope", torch.bfloat16, 3)
    _need(w_uk, "w_uk", torch.bfloat16, 3)
    T, H, dn = q_nope.shape
    if dn != 128 or tuple(q_rope.shape) != (T, H, 64) or tuple(w_uk.shape) != (H, 128, 512):
        raise ValueError("shapes must be q_nope [T,H,128], q_rope [T,H,64], w_uk [H,128,512]")
    dev = q_nope.device
    if out is None:
        out = torch.empty((T, H, 576), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, 3)
    with torch.cuda.device(dev):
        _check(library.mla_absorb_query(_ptr(q_nope), _ptr(q_rope), _ptr(w_uk), T, H, _ptr(out),
                                        _stream_ptr(dev)))
    return out


def project_output(o_latent: torch.Tensor, w_uv: torch.Tensor,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per-head output W^UV_h o_latent: o_latent bf16 [T, H, 512], w_uv bf16 [H, 128, 512]
    -> bf16 [T, H, 128]."""
    _need(o_latent, "o_latent", torch.bfloat16, 3)
    _need(w_uv, "w_uv", torch.bfloat16, 3)
    T, H, dc = o_latent.shape
    if dc != 512 or tuple(w_uv.shape) != (H, 128, 512):
        raise ValueError("shapes must be o_latent [T,H,512], w_uv [H,128,512]")
    dev = o_latent.device
    if out is None:
        out = torch.empty((T, H, 128), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, 3)
    with torch.cuda.device(dev):
        _check(library.mla_project_output(_ptr(o_latent), _ptr(w_uv), T, H, _ptr(out), _stream_ptr(dev)))
    return out


class PagePool:
    """Host-side pool of 64-token cache pages (the pmla_page_pool_* C calls).

    Page ids index the kvcache's first dimension.  ``grow`` / ``release`` keep a
    sequence's block-table row (a host int32 numpy array) in step with its
    length; copy the table to the device for the decode call.
    """

    def __init__(self, num_pages: int):
        h = ctypes.c_void_p()
        _check(library.pmla_page_pool_create(int(num_pages), ctypes.byref(h)))
        self._h = h
        self.num_pages = int(num_pages)

    def close(self) -> None:
        if self._h:
            library.pmla_page_pool_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def num_free(self) -> int:
        n = library.pmla_page_pool_num_free(self._h)
        if n < 0:
            raise PmlaError(n, "pmla_page_pool_num_free failed")
        return int(n)

    def alloc(self, n: int) -> "np.ndarray":
        out = np.empty(int(n), dtype=np.int32)
        _check(library.pmla_page_pool_alloc(self._h, int(n), out.ctypes.data_as(ctypes.c_void_p)))
        return out

    def free(self, pages) -> None:
        a = np.ascontiguousarray(pages, dtype=np.int32)
        _check(library.pmla_page_pool_free(self._h, a.size, a.ctypes.data_as(ctypes.c_void_p)))

    def grow(self, row: "np.ndarray", cur_len: int, new_len: int) -> None:
        if row.dtype != np.int32 or not row.flags["C_CONTIGUOUS"]:
            raise ValueError("block-table row must be a contiguous int32 numpy array")
        _check(library.pmla_page_pool_grow_sequence(self._h, row.ctypes.data_as(ctypes.c_void_p), row.size,
                                                    int(cur_len), int(new_len)))

    def release(self, row: "np.ndarray", length: int) -> None:
        a = np.ascontiguousarray(row, dtype=np.int32)
        _check(library.pmla_page_pool_release_sequence(self._h, a.ctypes.data_as(ctypes.c_void_p), int(length)))


def workspace_bytes(batch: int, s_q: int, h_q: int, h_kv: int) -> int:
    return metadata_sizes(batch, s_q * (h_q // h_kv), h_kv)[1]


def device_error() -> int:
    """Read and clear the device error word (synchronises the current device)."""
    return int(library.pmla_device_error())

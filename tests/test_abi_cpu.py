"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments with error codes before touching a GPU (CPU only: no compute)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedmla.h")
LIB = os.path.join(ROOT, "paged_mla_attention_b200", "libpagedmla.so")


@pytest.fixture(scope="module")
def lib():
    from paged_mla_attention_b200 import build
    build.build()
    return ctypes.CDLL(LIB)


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"PMLA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ["mla_get_metadata", "mla_get_metadata_sizes", "mla_decode_with_kvcache",
              "pmla_device_error", "pmla_last_error", "pmla_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in pagedmla.h but not exported"


def test_version(lib):
    lib.pmla_version.restype = ctypes.c_char_p
    assert b"sm_100a" in lib.pmla_version()


def _decode(lib, **kw):
    P, I = ctypes.c_void_p, ctypes.c_int
    f = lib.mla_decode_with_kvcache
    f.argtypes = [P, P, P, P] + [I] * 8 + [P, I, P, I, ctypes.c_float, P, P, P, ctypes.c_size_t, P]
    f.restype = I
    a = dict(q=0x10000, kv=0x20000, bt=0x30000, sl=0x40000, batch=2, s_q=1, h_q=16, h_kv=1,
             d=576, dv=512, num_pages=8, max_pages=3, meta=0x50000, parts=4, splits=0x60000,
             causal=0, scale=0.07, o=0x70000, lse=0x80000, ws=0x90000, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return f(a["q"], a["kv"], a["bt"], a["sl"], a["batch"], a["s_q"], a["h_q"], a["h_kv"], a["d"],
             a["dv"], a["num_pages"], a["max_pages"], a["meta"], a["parts"], a["splits"], a["causal"],
             a["scale"], a["o"], a["lse"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(d=575), -2), (dict(dv=256), -2), (dict(h_q=15, h_kv=2), -2),
    (dict(h_q=96), -2), (dict(h_q=12, h_kv=3), -2), (dict(h_q=320), -2),
    (dict(batch=-1), -1), (dict(s_q=0), -1), (dict(num_pages=0), -1), (dict(parts=0), -1),
    (dict(scale=float("nan")), -1), (dict(scale=-1.0), -1),
    (dict(q=None), -1), (dict(lse=None), -1), (dict(splits=None), -1),
    (dict(q=0x10001), -3), (dict(o=0x70008), -3), (dict(o=0x70010), -3), (dict(kv=0x20002), -3),
    (dict(ws_bytes=16), -5), (dict(ws=None), -5), (dict(ws=0x90004), -5), (dict(ws=0x90010), -5),
])
def test_decode_rejects_bad_arguments(lib, kw, code):
    assert _decode(lib, **kw) == code
    lib.pmla_last_error.restype = ctypes.c_char_p
    assert lib.pmla_last_error()  # a message was recorded


def test_metadata_rejects_bad_arguments(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    f = lib.mla_get_metadata
    f.argtypes = [P, I, I, I, P, I, P, P]
    f.restype = I
    assert f(0x1000, -1, 128, 1, 0x2000, 4, 0x3000, None) == -1
    assert f(0x1000, 4, 0, 1, 0x2000, 4, 0x3000, None) == -1
    assert f(0x1000, 4, 128, 1, None, 4, 0x3000, None) == -1
    assert f(0x1000, 4, 128, 1, 0x2000, 0, 0x3000, None) == -1


@pytest.mark.parametrize("kw,code", [
    (dict(d=512), -2),            # UNSUPPORTED: only d = 576 rows
    (dict(s_new=-1), -1),         # INVALID_ARG
    (dict(h_kv=0), -1),
    (dict(num_pages=0), -1),
    (dict(new_kv=0x1008), -3),    # ALIGNMENT: new_kv not 16-byte aligned
    (dict(kvcache=0), -1),        # null pointer
])
def test_append_rejects_bad_arguments(lib, kw, code):
    args = dict(new_kv=0x1000, block_table=0x2000, cache_seqlens=0x3000, batch=2, s_new=1, h_kv=1,
                d=576, kvcache=0x4000, num_pages=8, max_pages=2, new_seqlens=None)
    args.update(kw)
    f = lib.mla_append_kvcache
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, I, I, I, I, P, I, I, P, P]
    f.restype = I
    rc = f(args["new_kv"], args["block_table"], args["cache_seqlens"], args["batch"], args["s_new"],
           args["h_kv"], args["d"], args["kvcache"], args["num_pages"], args["max_pages"],
           args["new_seqlens"], None)
    assert rc == code


def test_append_with_nothing_to_write_is_a_no_op(lib):
    f = lib.mla_append_kvcache
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, I, I, I, I, P, I, I, P, P]
    f.restype = I
    assert f(None, None, None, 0, 1, 1, 576, None, 8, 2, None, None) == 0   # empty batch
    assert f(None, None, None, 4, 0, 1, 576, None, 8, 2, None, None) == 0   # no new tokens


@pytest.mark.parametrize("kw,code", [
    (dict(tokens=-1), -1), (dict(heads=0), -1), (dict(heads=70000), -1),
    (dict(a=None), -1), (dict(w=None), -1), (dict(out=None), -1), (dict(rope=None), -1),
    (dict(a=0x1008), -3), (dict(w=0x2004), -3), (dict(rope=0x3002), -3),
    (dict(out=0x4010), -3),       # outputs need 32-byte alignment (256-bit stores)
])
def test_absorb_query_rejects_bad_arguments(lib, kw, code):
    args = dict(a=0x1000, rope=0x3000, w=0x2000, tokens=4, heads=16, out=0x4000)
    args.update(kw)
    P, I = ctypes.c_void_p, ctypes.c_int
    f = lib.mla_absorb_query
    f.argtypes = [P, P, P, I, I, P, P]
    f.restype = I
    assert f(args["a"], args["rope"], args["w"], args["tokens"], args["heads"], args["out"], None) == code


def test_project_output_rejects_bad_arguments(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    f = lib.mla_project_output
    f.argtypes = [P, P, I, I, P, P]
    f.restype = I
    assert f(0x1000, 0x2000, -1, 16, 0x4000, None) == -1
    assert f(0x1000, 0x2000, 4, 0, 0x4000, None) == -1
    assert f(None, 0x2000, 4, 16, 0x4000, None) == -1
    assert f(0x1000, 0x2000, 4, 16, 0x4008, None) == -3
    assert f(0x1000, 0x2008, 4, 16, 0x4000, None) == -3
    assert f(None, None, 0, 16, None, None) == 0   # no tokens: nothing to do


def test_decode_with_empty_batch_is_a_no_op(lib):
    # nothing to read or write: every pointer may be null (empty tensors)
    assert _decode(lib, batch=0, q=None, kv=None, bt=None, sl=None, meta=None, splits=None, o=None,
                   lse=None, ws=None, ws_bytes=0) == 0
    assert _decode(lib, batch=0, d=575) == -2       # shapes are still checked


def test_oversized_shapes_are_rejected_before_any_size_overflows(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    f = lib.mla_get_metadata_sizes
    f.argtypes = [I, I, I, P, P]
    f.restype = I
    parts, ws = ctypes.c_int(0), ctypes.c_size_t(0)
    assert f(65535, 1 << 20, 65535, ctypes.byref(parts), ctypes.byref(ws)) == -2
    assert f(1, (1 << 20) + 1, 1, ctypes.byref(parts), ctypes.byref(ws)) == -2
    assert _decode(lib, s_q=8192, h_q=256) == -2       # R = 2^21 rows per KV head


def test_mla_get_last_error_is_the_same_message(lib):
    lib.pmla_last_error.restype = ctypes.c_char_p
    lib.mla_get_last_error.restype = ctypes.c_char_p
    assert _decode(lib, d=575) == -2
    assert lib.mla_get_last_error() == lib.pmla_last_error() and b"576" in lib.mla_get_last_error()


def test_binding_follows_the_usage_call_order():
    # FlashMLA usage step 4: (q, kvcache, block_table, cache_seqlens, dv,
    # tile_scheduler_metadata, num_splits, causal); softmax_scale after it and the
    # buffers/stage selector keyword-only, so a positional causal cannot land elsewhere
    import inspect
    from paged_mla_attention_b200 import flash_mla_with_kvcache
    ps = list(inspect.signature(flash_mla_with_kvcache).parameters.values())
    assert [p.name for p in ps[:9]] == ["q", "kvcache", "block_table", "cache_seqlens", "head_dim_v",
                                        "tile_scheduler_metadata", "num_splits", "causal", "softmax_scale"]
    assert all(p.kind == p.POSITIONAL_OR_KEYWORD for p in ps[:9])
    assert all(p.kind == p.KEYWORD_ONLY for p in ps[9:])

"""mla_decode_with_kvcache_noalloc: the decode for callers that cannot allocate.

Callers such as code inside a CUDA stream capture, runtimes that own all device
memory up front, or plugins whose host forbids other allocations cannot hand the
library a workspace.  This entry point takes the split scratch from a fixed
array inside the library instead.  The test calls it through the C ABI and
checks that its output equals the workspace entry point's output bit for bit
(same inputs, same metadata, same kernels: only the scratch's address
differs), on two calls in a row (the second call reuses the array the first
one left behind), and that it matches the oracle at the parity tolerances.  It
runs last (file name) so a failure here never hides another test's result.
"""
import ctypes

import numpy as np
import pytest

import mla_workloads as W
import oracle
from gpu_helpers import compare, to_device

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    import paged_mla_attention_b200 as pm
    f = pm.library.mla_decode_with_kvcache_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P] + [I] * 8 + [P, I, P, I, ctypes.c_float, P, P, P]
    f.restype = I
    return f


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    import paged_mla_attention_b200 as pm
    # long sequences next to short ones, so split pieces really use the scratch
    w = W.Workload("noalloc", 5, 1, 128, 1, False, "explicit", ((9000, 70, 3000, 1, 5000),), seed=77)
    inp = W.make_inputs(w, seqlens=[9000, 70, 3000, 1, 5000], extra_pages=3)
    d = to_device(inp)
    R = inp["s_q"] * inp["h_q"] // inp["h_kv"]
    meta, splits = pm.get_mla_metadata(d["cache_seqlens"], R, inp["h_kv"])
    assert int(torch.diff(splits).max()) >= 2, "want split sequences so the scratch is used"
    o_ref, lse_ref = pm.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"],
                                               d["cache_seqlens"], W.D_V, meta, splits,
                                               softmax_scale=inp["softmax_scale"], causal=False)
    f = _noalloc_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        rc = f(d["q"].data_ptr(), d["kvcache"].data_ptr(), d["block_table"].data_ptr(),
               d["cache_seqlens"].data_ptr(), inp["batch"], inp["s_q"], inp["h_q"], inp["h_kv"],
               W.D_QK, W.D_V, inp["num_pages"], inp["max_pages"], meta.data_ptr(), meta.shape[0],
               splits.data_ptr(), 0, inp["softmax_scale"], o.data_ptr(), lse.data_ptr(), stream)
        assert rc == 0, pm.library.pmla_last_error().decode()
        torch.cuda.synchronize()
        assert pm.device_error() == 0
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16)), f"call {call}: o differs"
        assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32)), f"call {call}: lse differs"
    ro, rl = oracle.decode_inputs(inp)
    compare(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), ro, rl,
            what="noalloc vs oracle")


def test_noalloc_rejects_shapes_above_its_scratch():
    import torch
    import paged_mla_attention_b200 as pm
    f = _noalloc_fn()
    batch = 4096  # (4096 + parts) * 128 rows * 2 KB of partials is far above 32 MiB
    rc = f(16, 16, 16, 16, batch, 1, 128, 1, W.D_QK, W.D_V, 64, 4, 16, 74, 16, 0, 0.07, 16, 16,
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -5
    assert b"maximum" in pm.library.pmla_last_error()

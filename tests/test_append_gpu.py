"""GPU parity of the cache append (mla_append_kvcache) against the C oracle:
the whole cache must match byte for byte, and decoding the appended cache must
match decoding a cache built with every token from the start."""
import numpy as np
import pytest

import mla_workloads as W
import oracle
from gpu_helpers import compare, run_gpu, to_device

pytestmark = pytest.mark.gpu


def _case(lens, s_new, h_kv, seed):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, dtype=np.int32)
    need = (lens + s_new + 63) // 64
    pool = int(need.sum()) + 5
    perm = rng.permutation(pool).astype(np.int32)
    bt = np.zeros((len(lens), int(need.max()) + 1), dtype=np.int32)
    k = 0
    for b in range(len(lens)):
        bt[b, :need[b]] = perm[k:k + need[b]]
        k += int(need[b])
    kv = W.f32_to_bf16_bits(rng.standard_normal((pool, 64, h_kv, W.D_QK)).astype(np.float32))
    new = W.f32_to_bf16_bits(rng.standard_normal((len(lens), s_new, h_kv, W.D_QK)).astype(np.float32))
    return lens, bt, kv, new


def _gpu_append(lens, bt, kv, new):
    import torch
    import paged_mla_attention_b200 as pm
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    kv_d, new_d = bf(kv), bf(new)
    bt_d, sl_d = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    out_len = torch.empty_like(sl_d)
    pm.append_kvcache(new_d, bt_d, sl_d, kv_d, new_seqlens=out_len)
    torch.cuda.synchronize()
    err = pm.device_error()
    return kv_d.view(torch.int16).cpu().numpy().view(np.uint16), out_len.cpu().numpy(), err


@pytest.mark.parametrize("lens,s_new,h_kv", [
    ([62, 0, 130, 64], 5, 1),       # page crossing, empty sequence, page-aligned start
    ([1, 200], 130, 2),             # several pages per sequence, two KV heads
    ([4095, 17, 63], 1, 1),         # one decode step
])
def test_append_matches_oracle_bytewise(lens, s_new, h_kv):
    lens, bt, kv, new = _case(lens, s_new, h_kv, seed=len(lens) * 7 + s_new)
    ref, ok = oracle.append_kvcache(new, bt, lens, kv)
    assert ok
    got, new_len, err = _gpu_append(lens, bt, kv, new)
    assert err == 0
    assert np.array_equal(got, ref)
    assert np.array_equal(new_len, lens + s_new)


def test_append_then_decode_matches_full_build():
    # decode of (truncated cache + appended tokens) == decode of the full cache
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w)
    s_new = 3
    L_full = inp["cache_seqlens"].copy()
    L_prev = (L_full - s_new).astype(np.int32)
    page = 64
    new = np.stack([inp["kvcache"][inp["block_table"][b][np.arange(L_prev[b], L_full[b]) // page],
                                   np.arange(L_prev[b], L_full[b]) % page] for b in range(inp["batch"])])
    damaged = inp["kvcache"].copy()
    for b in range(inp["batch"]):
        t = np.arange(L_prev[b], L_full[b])
        damaged[inp["block_table"][b][t // page], t % page] = 0x7f7f
    got, new_len, err = _gpu_append(L_prev, inp["block_table"], damaged, new)
    assert err == 0 and np.array_equal(got, inp["kvcache"]) and np.array_equal(new_len, L_full)
    o, lse, _, _ = run_gpu(dict(inp, kvcache=got))
    ro, rl = oracle.decode_inputs(inp)
    compare(o, lse, ro, rl, what="append then decode")


def test_append_out_of_range_page_is_reported_not_written():
    lens, bt, kv, new = _case([10], 2, 1, seed=3)
    bt[0, 0] = kv.shape[0] + 5          # page id outside the pool
    got, _, err = _gpu_append(lens, bt, kv, new)
    assert err == 2                     # bad page
    assert np.array_equal(got, kv)      # nothing written

"""GPU parity of the absorbed MLA projections (mla_absorb_query, mla_project_output)
and of the whole absorbed pipeline against the fp64 oracles.

Both sides round where the pipeline stores bf16: the absorbed query and the
latent decode output are rounded to bf16 (round to nearest even) in the oracle
route too, so the remaining differences are accumulation order and the final
bf16 o: max|o - o_ref| <= 1e-2 and cosine >= 0.99999 as for the decode.  Against
the unabsorbed fp64 math (no intermediate rounding) the bar is cosine >= 0.9995,
the drift a bf16 query of 512 terms allows."""
import math

import numpy as np
import pytest

import mla_workloads as W
import oracle

pytestmark = pytest.mark.gpu


def _bf(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(W.f32_to_bf16_bits(np.asarray(a, np.float32))).view(np.int16)).cuda().view(torch.bfloat16)


def _np(t):
    import torch
    return W.bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def _rt(a):  # round to bf16 and back (RNE)
    return W.bf16_bits_to_f32(W.f32_to_bf16_bits(np.asarray(a, np.float32))).astype(np.float64)


def _weights(h, seed):
    rng = np.random.default_rng(seed)
    return (_rt(rng.standard_normal((h, 128, 512)) / math.sqrt(128)),
            _rt(rng.standard_normal((h, 128, 512)) / math.sqrt(512)))


@pytest.mark.parametrize("tokens,heads", [(1, 16), (6, 128), (33, 4), (64, 128), (96, 2), (130, 8), (257, 3)])
def test_projection_kernels_match_fp64(tokens, heads):
    import torch
    import paged_mla_attention_b200 as pm
    rng = np.random.default_rng(tokens + heads)
    qn = _rt(rng.standard_normal((tokens, heads, 128)))
    qr = _rt(rng.standard_normal((tokens, heads, 64)))
    ol = _rt(rng.standard_normal((tokens, heads, 512)))
    w_uk, w_uv = _weights(heads, 5)
    q_out = torch.empty((tokens, heads, 576), dtype=torch.bfloat16, device="cuda")
    o_out = torch.empty((tokens, heads, 128), dtype=torch.bfloat16, device="cuda")
    pm.absorb_query(_bf(qn), _bf(qr), _bf(w_uk), out=q_out)
    pm.project_output(_bf(ol), _bf(w_uv), out=o_out)
    torch.cuda.synchronize()
    assert pm.device_error() == 0
    q_ref = np.einsum("thk,hkn->thn", qn, w_uk)
    o_ref = np.einsum("thk,hnk->thn", ol, w_uv)
    q_gpu, o_gpu = _np(q_out), _np(o_out)
    # bf16 results of an fp32 accumulation: within one bf16 half-ulp of the exact value
    # plus the fp32 accumulation error (absolute, well under 1e-4 at these magnitudes)
    assert np.all(np.abs(q_gpu[..., :512] - q_ref) <= np.abs(q_ref) * 2.0 ** -8 + 1e-4)
    assert np.array_equal(q_gpu[..., 512:], qr)  # the RoPE part passes through
    assert np.all(np.abs(o_gpu - o_ref) <= np.abs(o_ref) * 2.0 ** -8 + 1e-4)


def test_rows_past_the_last_token_are_not_written():
    """The output views end at `tokens`; the rows after them in the same buffer keep
    their contents (boxes past the end are clipped, not written)."""
    import torch
    import paged_mla_attention_b200 as pm
    T, H = 70, 6
    rng = np.random.default_rng(3)
    w_uk, w_uv = _weights(H, 7)
    q_big = torch.full((T + 60, H, 576), 7.0, dtype=torch.bfloat16, device="cuda")
    o_big = torch.full((T + 60, H, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    pm.absorb_query(_bf(_rt(rng.standard_normal((T, H, 128)))), _bf(_rt(rng.standard_normal((T, H, 64)))),
                    _bf(w_uk), out=q_big[:T])
    pm.project_output(_bf(_rt(rng.standard_normal((T, H, 512)))), _bf(w_uv), out=o_big[:T])
    torch.cuda.synchronize()
    assert pm.device_error() == 0
    assert bool((q_big[T:] == 7.0).all()) and bool((o_big[T:] == 7.0).all())
    assert not bool((q_big[:T] == 7.0).all())


def test_weights_written_by_the_preceding_kernel():
    """The kernels start before the preceding kernel on the stream has completed
    (programmatic dependent launch) and prefetch their weights into L2 meanwhile:
    weights that this preceding kernel writes must still be read as written."""
    import torch
    import paged_mla_attention_b200 as pm
    T, H = 64, 128
    rng = np.random.default_rng(11)
    qn = _rt(rng.standard_normal((T, H, 128)))
    qr = _rt(rng.standard_normal((T, H, 64)))
    ol = _rt(rng.standard_normal((T, H, 512)))
    ws = [_weights(H, 20 + i) for i in range(3)]
    src_uk = [_bf(w[0]) for w in ws]
    src_uv = [_bf(w[1]) for w in ws]
    qn_d, qr_d, ol_d = _bf(qn), _bf(qr), _bf(ol)
    w_uk = torch.empty_like(src_uk[0])
    w_uv = torch.empty_like(src_uv[0])
    q = torch.empty((T, H, 576), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((T, H, 128), dtype=torch.bfloat16, device="cuda")
    for it in range(6):
        i = it % 3
        torch.mul(src_uk[i], 1, out=w_uk)  # a kernel writing the weights, directly before the call
        pm.absorb_query(qn_d, qr_d, w_uk, out=q)
        torch.mul(src_uv[i], 1, out=w_uv)
        pm.project_output(ol_d, w_uv, out=o)
        q_ref = np.einsum("thk,hkn->thn", qn, ws[i][0])
        o_ref = np.einsum("thk,hnk->thn", ol, ws[i][1])
        q_gpu, o_gpu = _np(q), _np(o)
        assert np.all(np.abs(q_gpu[..., :512] - q_ref) <= np.abs(q_ref) * 2.0 ** -8 + 1e-4), it
        assert np.all(np.abs(o_gpu - o_ref) <= np.abs(o_ref) * 2.0 ** -8 + 1e-4), it
    assert pm.device_error() == 0


def test_absorbed_pipeline_matches_oracles():
    import torch
    import paged_mla_attention_b200 as pm
    from gpu_helpers import to_device
    w = W.Workload("proj", 3, 2, 16, 1, True, "explicit", ((70, 300, 2),), seed=41)
    inp = W.make_inputs(w, seqlens=[70, 300, 2], extra_pages=2)
    b, s_q, h = 3, 2, 16
    rng = np.random.default_rng(41)
    qn = _rt(rng.standard_normal((b, s_q, h, 128)))
    qr = _rt(rng.standard_normal((b, s_q, h, 64)))
    w_uk, w_uv = _weights(h, 41)
    d = to_device(inp)
    T = b * s_q
    q = torch.empty((T, h, 576), dtype=torch.bfloat16, device="cuda")
    pm.absorb_query(_bf(qn.reshape(T, h, 128)), _bf(qr.reshape(T, h, 64)), _bf(w_uk), out=q)
    meta, splits = pm.get_mla_metadata(d["cache_seqlens"], s_q * h, 1)
    o_lat, lse = pm.flash_mla_with_kvcache(q.view(b, s_q, h, 576), d["kvcache"], d["block_table"],
                                           d["cache_seqlens"], 512, meta, splits,
                                           softmax_scale=inp["softmax_scale"], causal=True)
    o = torch.empty((T, h, 128), dtype=torch.bfloat16, device="cuda")
    pm.project_output(o_lat.reshape(T, h, 512), _bf(w_uv), out=o)
    torch.cuda.synchronize()
    assert pm.device_error() == 0
    o_gpu = _np(o).reshape(b, s_q, h, 128)
    # oracle route with the same bf16 roundings: absorb (fp64) -> bf16 -> latent decode
    # oracle -> bf16 -> project (fp64)
    q_abs = np.concatenate([np.einsum("bshk,hkn->bshn", qn, w_uk), qr], axis=-1)
    q_bits = W.f32_to_bf16_bits(q_abs.astype(np.float32))
    ol_ref, _ = oracle.mla_decode(q_bits, inp["kvcache"], inp["block_table"], inp["cache_seqlens"], 512,
                                  True, inp["softmax_scale"])
    o_ref = np.einsum("bshk,hnk->bshn", _rt(ol_ref), w_uv)
    err = float(np.abs(o_gpu - o_ref).max())
    cos = float(o_gpu.ravel() @ o_ref.ravel() / (np.linalg.norm(o_gpu) * np.linalg.norm(o_ref)))
    assert err <= 1e-2 and cos >= 0.99999, (err, cos)
    # against the unabsorbed fp64 math (up-projected keys and values per head)
    o_un, _ = oracle.default().mla_decode_unabsorbed(qn, qr, w_uk, w_uv, inp["kvcache"], inp["block_table"],
                                           inp["cache_seqlens"], True, inp["softmax_scale"])
    cos_un = float(o_gpu.ravel() @ o_un.ravel() / (np.linalg.norm(o_gpu) * np.linalg.norm(o_un)))
    assert cos_un >= 0.9995, cos_un

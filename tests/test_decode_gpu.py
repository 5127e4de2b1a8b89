"""GPU parity: the sm_100a decode path (through the C ABI) against the fp64 oracle.

Parity bar (bf16 inputs, fp32 accumulation, bf16 o):
max|o - o_ref| <= 1e-2, cosine(o, o_ref) >= 0.99999, max|lse - lse_ref| <= 1e-3.
"""
import numpy as np
import pytest

import mla_workloads as W
import oracle
from gpu_helpers import check_schedule, compare, run_gpu, subset, to_device

pytestmark = pytest.mark.gpu


def _small(seqlens, s_q=1, h_q=128, h_kv=1, causal=False, seed=0, extra_pages=3, scale=W.SCALE_192):
    w = W.Workload("case", len(seqlens), s_q, h_q, h_kv, causal, "explicit", (tuple(seqlens),),
                   seed=seed, softmax_scale=scale)
    return W.make_inputs(w, seqlens=seqlens, extra_pages=extra_pages)


def _check(inp, what):
    o, lse, meta, splits = run_gpu(inp)
    ro, rl = oracle.decode_inputs(inp)
    return compare(o, lse, ro, rl, what=what), meta, splits


def test_tiny_config():
    inp = W.make_inputs(W.WORKLOADS["tiny"])
    stats, _, _ = _check(inp, "tiny")
    assert stats["max_o"] < 4.0  # bf16 half-ulp of |o| stays under the o tolerance


@pytest.mark.parametrize("h_q", [16, 64, 128])
def test_page_boundary_lengths(h_q):
    _check(_small([1, 63, 64, 65, 127, 128, 129, 200], h_q=h_q, seed=h_q), f"edges h_q={h_q}")


def test_empty_and_single_token_sequences():
    stats, _, splits = _check(_small([0, 1, 0, 70, 1], h_q=32, seed=5), "empty/single")
    assert list(np.diff(splits)[[0, 2]]) == [0, 0]


@pytest.mark.parametrize("s_q,h_q", [(2, 128), (2, 64), (3, 32), (4, 16)])
def test_causal_multi_token(s_q, h_q):
    # includes sequences shorter than s_q, whose first rows see nothing
    _check(_small([1, 2, 3, 66, 130, 700], s_q=s_q, h_q=h_q, causal=True, seed=10 + s_q),
           f"causal s_q={s_q} h_q={h_q}")


def test_non_causal_multi_token():
    _check(_small([5, 90, 300], s_q=2, h_q=64, causal=False, seed=21), "s_q=2 non-causal")


def test_two_stage_calls_equal_the_single_call():
    # mla_decode_splits then mla_merge_splits == mla_decode_with_kvcache, bit for bit
    import torch
    import paged_mla_attention_b200 as pm
    inp = _small([9000, 100, 3000, 0, 64, 1], h_q=128, seed=23)
    d = to_device(inp)
    meta, splits = pm.get_mla_metadata(d["cache_seqlens"], 128, 1)
    assert int((splits[1:] - splits[:-1]).max()) >= 2
    args = (d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"], W.D_V, meta, splits)
    o1, l1 = pm.flash_mla_with_kvcache(*args, softmax_scale=inp["softmax_scale"])
    ws = torch.empty((pm.workspace_bytes(inp["batch"], 1, 128, 1),), dtype=torch.uint8, device="cuda")
    o2 = torch.full_like(o1, float("nan"))
    l2 = torch.full_like(l1, float("nan"))
    pm.flash_mla_with_kvcache(*args, softmax_scale=inp["softmax_scale"], out=(o2, l2), workspace=ws,
                              stage="decode")
    pm.flash_mla_with_kvcache(*args, softmax_scale=inp["softmax_scale"], out=(o2, l2), workspace=ws,
                              stage="merge")
    torch.cuda.synchronize()
    assert pm.device_error() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))


def test_split_sequences_merge():
    # long sequences next to short ones: pieces of the long ones go through the merge kernel
    stats, meta, splits = _check(_small([9000, 100, 3000, 64, 1], h_q=128, seed=22), "splits")
    assert np.diff(splits).max() >= 2, "expected at least one split sequence"


@pytest.mark.parametrize("lens,s_q,h_q,h_kv,causal", [
    ([5000, 64], 2, 128, 1, True),        # two row groups per KV head (4-CTA clusters)
    ([12000, 200, 5], 1, 64, 2, False),   # two KV heads
    ([2200, 2200, 1], 1, 128, 1, False),  # two long sequences sharing the parts
])
def test_merge_of_many_pieces(lens, s_q, h_q, h_kv, causal):
    # few sequences, one or two of them long: more than 16 pieces each, merged by the
    # many-piece variant (8 column slices, two groups of warps taking pieces in turns)
    stats, meta, splits = _check(_small(lens, s_q=s_q, h_q=h_q, h_kv=h_kv, causal=causal, seed=sum(lens) % 97),
                                 f"many pieces {lens}")
    assert np.diff(splits).max() > 16, f"expected a sequence in more than 16 pieces, got {np.diff(splits)}"


def test_grouped_kv_heads():
    _check(_small([70, 300, 5], s_q=1, h_q=32, h_kv=2, seed=23), "h_kv=2")
    _check(_small([129, 40], s_q=2, h_q=64, h_kv=4, causal=True, seed=24), "h_kv=4 causal")


def test_row_groups_beyond_128():
    # s_q * h_q / h_kv = 256 and 192: two row groups per KV head
    _check(_small([200, 1000], s_q=2, h_q=128, causal=True, seed=25), "R=256")
    _check(_small([77, 513], s_q=3, h_q=64, causal=True, seed=26), "R=192")


def test_zero_scale_gives_mean_of_values():
    _check(_small([10, 150], h_q=16, seed=27, scale=0.0), "scale=0")


def test_page_relabelling_is_bitwise_invariant():
    inp = _small([300, 64, 1000], h_q=128, seed=28, extra_pages=9)
    o1, l1, _, _ = run_gpu(inp)
    perm = np.random.default_rng(7).permutation(inp["kvcache"].shape[0])
    kv2 = np.empty_like(inp["kvcache"])
    kv2[perm] = inp["kvcache"]
    inp2 = dict(inp, kvcache=kv2, block_table=perm[inp["block_table"]].astype(np.int32))
    o2, l2, _, _ = run_gpu(inp2)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_deterministic():
    inp = _small([4000, 33, 1500], h_q=128, seed=29)
    d = to_device(inp)
    a = run_gpu(inp, dev_inputs=d)
    b = run_gpu(inp, dev_inputs=d)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_lazy_rescale_path():
    # q aligned with later keys so the running max climbs page after page:
    # forces the O-row rescale command many times
    inp = _small([64 * 12], h_q=128, seed=30)
    kv = W.bf16_bits_to_f32(inp["kvcache"]).copy()
    L = 64 * 12
    t = np.arange(L)
    pages = inp["block_table"][0][t // 64]
    ramp = np.linspace(0.0, 6.0, L).astype(np.float32)  # scores grow along the sequence
    kv[pages, t % 64, 0, :] *= 0.25
    kv[pages, t % 64, 0, 570] = ramp * 40.0       # a RoPE column: not part of the values
    q = W.bf16_bits_to_f32(inp["q"]).copy()
    q[..., 570] = np.abs(q[..., 570]) + 1.0
    inp["kvcache"] = W.f32_to_bf16_bits(kv)
    inp["q"] = W.f32_to_bf16_bits(q)
    _check(inp, "rescale")


def test_pair_clusters_rescale_one_row_group():
    # s_q = 2, causal, 128 heads: both row groups (query token 0, query token 1)
    # share one 4-CTA cluster.  The last cached token scores far above all others
    # and only query token 1 sees it, so only the second row group moves its
    # reference max there: the O pair must rescale on the other CTA's flag too.
    L = 64 * 12 + 7
    inp = _small([L, 300], s_q=2, h_q=128, causal=True, seed=35)
    kv = W.bf16_bits_to_f32(inp["kvcache"]).copy()
    q = W.bf16_bits_to_f32(inp["q"]).copy()
    last = inp["block_table"][0][(L - 1) // 64]
    kv[last, (L - 1) % 64, 0, 570] = 200.0     # a RoPE column: not part of the values
    q[..., 570] = np.abs(q[..., 570]) + 0.5
    t = np.arange(L - 1)
    pages = inp["block_table"][0][t // 64]
    kv[pages, t % 64, 0, 570] = np.linspace(-4.0, 4.0, L - 1)   # a climbing max for both groups
    inp["kvcache"] = W.f32_to_bf16_bits(kv)
    inp["q"] = W.f32_to_bf16_bits(q)
    _check(inp, "pair rescale")


def test_pair_clusters_two_kv_heads_and_non_causal():
    # two row groups per KV head with two KV heads (h_q 256, h_kv 2, s_q 2), and
    # the non-causal two-token case at 128 heads: both run the 4-CTA variant
    _check(_small([130, 2000, 64, 1], s_q=2, h_q=256, h_kv=2, causal=True, seed=37), "pair h_kv=2")
    _check(_small([700, 5, 3100], s_q=2, h_q=128, causal=False, seed=38), "pair non-causal")


def test_pair_clusters_odd_row_groups():
    # s_q = 3 x 128 heads: three row groups, so the second 4-CTA cluster's upper
    # half has no rows at all
    _check(_small([5, 200, 1300, 64], s_q=3, h_q=128, causal=True, seed=36), "R=384")


@pytest.mark.parametrize("seed", range(6))
def test_scheduler_invariants(seed):
    import torch
    import paged_mla_attention_b200 as pm
    rng = np.random.default_rng(1000 + seed)
    for trial in range(20):
        batch = int(rng.integers(1, 200))
        kind = trial % 4
        if kind == 0:
            lens = rng.integers(0, 300, size=batch)
        elif kind == 1:
            lens = rng.integers(0, 40000, size=batch)
        elif kind == 2:
            lens = np.where(rng.random(batch) < 0.1, rng.integers(10000, 200000, size=batch),
                            rng.integers(0, 100, size=batch))
        else:
            lens = np.full(batch, int(rng.integers(0, 5000)))
        for heads in (16, 128, 256):
            sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
            meta, splits = pm.get_mla_metadata(sl, heads, 1)
            torch.cuda.synchronize()
            m = meta.cpu().numpy()
            check_schedule(m, splits.cpu().numpy(), lens, meta.shape[0])
            # two row groups: 4-CTA clusters leave SMs free on B200 (148 = 4 x 33 + 16),
            # whose parts weigh less (107); one row group: every part weighs 128
            if heads == 256:
                assert (m[:, 5] == 107).sum() >= 1
            else:
                assert np.all(m[:, 5] == 128)


def test_scheduler_exhaustive_small():
    """Every length vector with batch <= 4 over lengths {0, 1, 64, 65, 129, 256}, for
    1, 2, 5 and 74 parts, through the C entry point: coverage, ordinals, prefix sums
    and the stated balance bound all hold."""
    import ctypes
    import itertools
    import torch
    import paged_mla_attention_b200 as pm
    vals = [0, 1, 64, 65, 129, 256]
    lib = pm.library
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for batch in range(1, 5):
        for lens in itertools.product(vals, repeat=batch):
            sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
            for parts in (1, 2, 5, 74):
                meta = torch.empty((parts, 8), dtype=torch.int32, device="cuda")
                splits = torch.empty((batch + 1,), dtype=torch.int32, device="cuda")
                rc = lib.mla_get_metadata(ctypes.c_void_p(sl.data_ptr()), batch, 128, 1,
                                          ctypes.c_void_p(meta.data_ptr()), parts,
                                          ctypes.c_void_p(splits.data_ptr()), stream)
                assert rc == 0
                check_schedule(meta.cpu().numpy(), splits.cpu().numpy(), np.array(lens), parts)


FULL = ["uniform", "varlen", "causal2", "skew"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_configs_in_full(name):
    """Full-size workloads in the benchmark's launch configuration: every row of
    o and lse against the oracle, element by element (the cosine over the whole
    o tensor), plus the schedule invariants and properties that hold at any
    size."""
    inp = W.make_inputs(W.WORKLOADS[name])
    o, lse, meta, splits = run_gpu(inp)
    lens = inp["cache_seqlens"]
    check_schedule(meta, splits, lens, meta.shape[0])
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    vmax = float(np.abs(W.bf16_bits_to_f32(inp["kvcache"][..., :512])).max())
    assert np.abs(o).max() <= vmax + 1e-2
    ro, rl = oracle.decode_inputs(inp)
    stats = compare(o, lse, ro, rl, what=name)
    print(f"full-size parity {name}: rows={o.shape[0] * o.shape[1] * o.shape[2]} "
          f"max|do|={stats['max_do']:.3e} cos={stats['cos']:.8f} max|dlse|={stats['max_dlse']:.3e} "
          f"max|o_ref|={stats['max_o']:.3f} split sequences={int((np.diff(splits) >= 2).sum())}")


def test_causal_is_the_eighth_positional_argument():
    # the FlashMLA usage call passes causal right after num_splits
    import torch
    import paged_mla_attention_b200 as pm
    inp = _small([70, 300, 5], s_q=2, h_q=64, causal=True, seed=33)
    d = to_device(inp)
    meta, splits = pm.get_mla_metadata(d["cache_seqlens"], 2 * 64, 1)
    o, lse = pm.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"],
                                       W.D_V, meta, splits, True, inp["softmax_scale"])
    torch.cuda.synchronize()
    assert pm.device_error() == 0
    ro, rl = oracle.decode_inputs(inp)
    compare(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), ro, rl,
            what="positional causal")


def test_sequence_longer_than_its_block_table_is_reported():
    # cache_seqlens[1] claims more tokens than its block-table row holds: that
    # sequence is not read, its rows come back empty (o = 0, lse = -inf), the
    # device error word says why, and the other sequences are unaffected
    import torch
    import paged_mla_attention_b200 as pm
    for lens in ([300, 9000, 4000], [300, 130, 20]):  # a split neighbour, and a short batch
        inp = _small(lens, h_q=128, seed=34)
        d = to_device(inp)
        cap = 64 * inp["max_pages"]
        bad = d["cache_seqlens"].clone()
        bad[1] = cap + 1
        meta, splits = pm.get_mla_metadata(bad, 128, 1)
        o, lse = pm.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], bad, W.D_V,
                                           meta, splits, False, inp["softmax_scale"])
        torch.cuda.synchronize()
        assert pm.device_error() == 4  # PMLA_DEVERR_BAD_SEQLEN
        og = o.float().cpu().numpy().astype(np.float64)
        lg = lse.cpu().numpy().astype(np.float64)
        assert np.all(og[1] == 0) and np.all(np.isneginf(lg[1]))
        keep = [0, 2]
        ro, rl = oracle.decode_inputs(subset(inp, keep))
        compare(og[keep], lg[keep], ro, rl, what="neighbours of an over-long sequence")


def test_empty_batch():
    import torch
    import paged_mla_attention_b200 as pm
    sl = torch.empty((0,), dtype=torch.int32, device="cuda")
    meta, splits = pm.get_mla_metadata(sl, 128, 1)
    q = torch.empty((0, 1, 128, W.D_QK), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((1, 64, 1, W.D_QK), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((0, 1), dtype=torch.int32, device="cuda")
    o, lse = pm.flash_mla_with_kvcache(q, kv, bt, sl, W.D_V, meta, splits)
    torch.cuda.synchronize()
    assert pm.device_error() == 0
    assert tuple(o.shape) == (0, 1, 128, W.D_V) and tuple(lse.shape) == (0, 128, 1)
    assert splits.cpu().tolist() == [0]


def test_all_sequences_empty():
    # every row sees nothing: o = 0, lse = -inf (no merge work, no NaN)
    stats, _, splits = _check(_small([0, 0, 0], h_q=64, seed=31), "all empty")
    assert list(splits) == [0, 0, 0, 0]


def test_four_query_tokens_128_heads():
    # s_q = 4 x h_q = 128: four 128-row groups per KV head, causal
    _check(_small([3, 64, 200, 1000], s_q=4, h_q=128, causal=True, seed=32), "s_q=4 h_q=128")


def test_back_to_back_calls_share_a_workspace():
    # two decode calls queued on one stream with no host sync in between, on the same
    # workspace: the second call's counter clear must wait for the first decode
    # (programmatic launch chain) and both results must match the oracle
    import torch
    import paged_mla_attention_b200 as pm
    a = _small([9000, 100, 3000, 64], h_q=128, seed=41)
    b = _small([300, 7000, 1, 2500], h_q=128, seed=42)
    da, db = to_device(a), to_device(b)
    ws = torch.empty((pm.workspace_bytes(4, 1, 128, 1),), dtype=torch.uint8, device="cuda")
    outs = []
    for inp, d in ((a, da), (b, db)):
        meta, splits = pm.get_mla_metadata(d["cache_seqlens"], 128, 1)
        outs.append(pm.flash_mla_with_kvcache(d["q"], d["kvcache"], d["block_table"], d["cache_seqlens"],
                                              W.D_V, meta, splits, softmax_scale=inp["softmax_scale"],
                                              workspace=ws))
    torch.cuda.synchronize()
    assert pm.device_error() == 0
    for inp, (o, lse) in zip((a, b), outs):
        ro, rl = oracle.decode_inputs(inp)
        compare(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), ro, rl,
                what="back to back")


@pytest.mark.parametrize("batch", [1500, 5000])
def test_large_batch_schedule_and_sampled_parity(batch):
    # more sequences than scheduler threads: each thread owns a chunk of several
    # sequences; the merge grid spans thousands of sequences
    rng = np.random.default_rng(batch)
    lens = rng.integers(0, 400, size=batch)
    lens[rng.choice(batch, size=batch // 50, replace=False)] = rng.integers(2000, 9000, size=batch // 50)
    inp = _small(lens.tolist(), h_q=16, seed=batch, extra_pages=2)
    o, lse, meta, splits = run_gpu(inp)
    check_schedule(meta, splits, inp["cache_seqlens"], meta.shape[0])
    assert np.isfinite(o).all()
    pick = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 0, batch - 1,
                   *[int(x) for x in rng.choice(batch, size=6, replace=False)]})
    sub = subset(inp, pick)
    ro, rl = oracle.decode_inputs(sub)
    compare(o[pick], lse[pick], ro, rl, what=f"batch {batch}")

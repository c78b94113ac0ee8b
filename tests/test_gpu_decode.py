"""paged_attention_decode on the GPU against the fp64 oracle, small shapes.

Sizes are chosen so that the oracle finishes in seconds while the kernels
still run several tiles, several blocks per tile (block_size below the tile)
and several tiles per block, ragged tails, and split-K on and off.
"""

import copy

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import check_workload, compare, device_pools, fill_history, run_gpu, to_device
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu


def cfg(**kw):
    base = dict(name="dec", num_seqs=5, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16, ctx_lo=1,
                ctx_hi=300)
    base.update(kw)
    return W.DecodeConfig(**base)


SHAPES = []
for d in (64, 128):
    for g in (1, 2, 4, 8):
        for bs in (16, 256):
            for fp8 in (False, True):
                SHAPES.append(cfg(head_dim=d, num_q_heads=2 * g, num_kv_heads=2, block_size=bs,
                                  cache_dtype=W.CACHE_FP8 if fp8 else W.CACHE_BF16))


@pytest.mark.parametrize("c", SHAPES, ids=lambda c: f"d{c.head_dim}-g{c.group}-bs{c.block_size}-{c.cache_dtype}")
@pytest.mark.parametrize("split", [-1, 64], ids=["nosplit", "split64"])
def test_decode_shapes(c, split):
    check_workload(W.generate(c, 11), partition_request=split)


@pytest.mark.parametrize("bs", [8, 16, 32, 256])
def test_lengths_at_block_and_tile_boundaries(bs):
    # lengths 1, bs-1, bs, bs+1, ... around block and tile edges
    lens = sorted({1, 2, bs - 1, bs, bs + 1, 2 * bs - 1, 2 * bs, 31, 32, 33, 63, 64, 65, 127, 128, 129} - {0})
    c = cfg(num_seqs=len(lens), block_size=bs, ctx_lo=1, ctx_hi=max(lens))
    wl = W.generate(c, 12)
    # replace the drawn lengths by the boundary lengths (re-deriving slots)
    wl = _with_lengths(c, wl, lens)
    for split in (-1, 32):
        check_workload(wl, partition_request=split)


@pytest.mark.parametrize("bs", [8, 16, 32, 256])
def test_fp8_lengths_at_group_and_tile_boundaries(bs):
    """E4M3 cache, head_dim 128 (the warp-MMA kernel): lengths around its
    16-token groups, 32-token warp slices and 128-token tiles, whole and
    split into 128-token partitions."""
    lens = sorted({1, 2, 15, 16, 17, 31, 32, 33, 47, 63, 64, 65, 95, 96, 97, 127, 128, 129, 255, 256, 257,
                   bs - 1, bs, bs + 1} - {0})
    c = cfg(num_seqs=len(lens), num_q_heads=8, num_kv_heads=2, block_size=bs, ctx_lo=1, ctx_hi=max(lens),
            cache_dtype=W.CACHE_FP8)
    wl = _with_lengths(c, W.generate(c, 12), lens)
    for split in (-1, 128):
        check_workload(wl, partition_request=split)


@pytest.mark.parametrize("d,dt", [(64, W.CACHE_BF16), (128, W.CACHE_BF16), (128, W.CACHE_FP8),
                                  (128, W.CACHE_FP8_TOKEN)])
def test_unsplit_partition_beyond_the_staged_block_ids(d, dt):
    """No split on contexts of up to 500 blocks of 8 tokens: the block ids
    past the 256 staged in shared memory come from the table row."""
    c = cfg(num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=d, block_size=8, ctx_lo=2100, ctx_hi=4000,
            cache_dtype=dt)
    wl = W.generate(c, 17)
    if dt == W.CACHE_FP8_TOKEN:
        from test_gpu_token_scales import run_decode

        out, _, st = run_decode(wl, partition=-1)
        ref, _, _, rst, _, _ = O.run_workload(wl, num_threads=8)
        assert st == K.PKV_OK and rst == O.ORC_OK
        compare(out, ref, True, "unsplit, per-token scales")
    else:
        check_workload(wl, partition_request=-1)


def _with_lengths(c, wl, lens):
    """A workload of the same pool with given lengths (rows re-drawn)."""
    g = torch.Generator().manual_seed(99)
    S = len(lens)
    bs = c.block_size
    nblk = sum(-(-n // bs) for n in lens) + 5
    perm = torch.randperm(nblk, generator=g)
    tables = torch.full((S, c.max_blocks_per_seq), -1, dtype=torch.int32)
    nxt = 0
    rows_k, rows_v, slots, hist_rows = [], [], [], []
    k_new = torch.randn(S, c.num_kv_heads, c.head_dim, generator=g).to(torch.bfloat16)
    v_new = torch.randn(S, c.num_kv_heads, c.head_dim, generator=g).to(torch.bfloat16)
    slot_new = torch.empty(S, dtype=torch.int32)
    n_rows = 0
    for i, n in enumerate(lens):
        nb = -(-n // bs)
        tables[i, :nb] = perm[nxt:nxt + nb].to(torch.int32)
        nxt += nb
        pos = torch.arange(n)
        sl = tables[i, pos // bs].long() * bs + pos % bs
        rows_k.append(torch.randn(n - 1, c.num_kv_heads, c.head_dim, generator=g).to(torch.bfloat16))
        rows_v.append(torch.randn(n - 1, c.num_kv_heads, c.head_dim, generator=g).to(torch.bfloat16))
        slots.append(sl[:-1].to(torch.int32))
        slot_new[i] = int(sl[-1])
        hist_rows.append(torch.arange(n_rows, n_rows + n - 1))
        n_rows += n - 1
    w2 = copy.copy(wl)
    w2.num_blocks = nblk
    w2.q = torch.randn(S, c.num_q_heads, c.head_dim, generator=g).to(torch.bfloat16)
    w2.k_hist, w2.v_hist, w2.slot_hist = torch.cat(rows_k), torch.cat(rows_v), torch.cat(slots)
    w2.k_new, w2.v_new, w2.slot_new = k_new, v_new, slot_new
    w2.block_tables, w2.context_lens = tables, torch.tensor(lens, dtype=torch.int32)
    w2.hist_rows = hist_rows
    return w2


def test_block_relabelling_is_bit_identical_on_gpu():
    import oracle_pins as P

    c = cfg(num_seqs=6, ctx_lo=50, ctx_hi=400)
    wl = W.generate(c, 13)
    out1, _, _, st1 = run_gpu(to_device(wl))
    perm = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(5))
    out2, _, _, st2 = run_gpu(to_device(P._relabel(wl, perm)))
    assert st1 == st2 == K.PKV_OK
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_prefix_shared_equals_private_copies_on_gpu():
    c = cfg(num_seqs=6, block_size=16, prefix_tokens=64, ctx_lo=0, ctx_hi=70)
    wl = W.generate(c, 14)
    out1, _, _, _ = run_gpu(to_device(wl))
    # private copies of the 4 shared blocks for every sequence
    P, bs, S = c.prefix_tokens, c.block_size, c.num_seqs
    ns = P // bs
    w2 = copy.copy(wl)
    w2.num_blocks = wl.num_blocks + S * ns
    bt = wl.block_tables.clone()
    ks, vs, ss = [wl.k_hist], [wl.v_hist], [wl.slot_hist]
    for i in range(S):
        first = wl.num_blocks + i * ns
        bt[i, :ns] = torch.arange(first, first + ns, dtype=torch.int32)
        ks.append(wl.k_hist[:P])
        vs.append(wl.v_hist[:P])
        ss.append(torch.arange(first * bs, first * bs + P, dtype=torch.int32))
    w2.block_tables, w2.k_hist, w2.v_hist, w2.slot_hist = bt, torch.cat(ks), torch.cat(vs), torch.cat(ss)
    out2, _, _, _ = run_gpu(to_device(w2))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_single_token_returns_v_bits():
    c = cfg(num_seqs=7, ctx_lo=1, ctx_hi=1)
    wl = to_device(W.generate(c, 15))
    out, _, _, st = run_gpu(wl)
    assert st == K.PKV_OK
    expect = wl.v_new.repeat_interleave(c.group, dim=1)
    assert torch.equal(out.view(torch.int16), expect.view(torch.int16))


def test_deterministic_and_split_consistent():
    c = cfg(num_seqs=8, ctx_lo=200, ctx_hi=900, block_size=16)
    wl = to_device(W.generate(c, 16))
    kp, vp = device_pools(wl)
    fill_history(wl, kp, vp)
    a, _, _, _ = run_gpu(wl, partition_request=-1, pools=(kp, vp))
    b, _, _, _ = run_gpu(wl, partition_request=-1, pools=(kp, vp))
    assert torch.equal(a.view(torch.int16), b.view(torch.int16)), "same call, different bits"
    for pt in (32, 64, 128, 320):
        s, _, _, _ = run_gpu(wl, partition_request=pt, pools=(kp, vp))
        s2, _, _, _ = run_gpu(wl, partition_request=pt, pools=(kp, vp))
        assert torch.equal(s.view(torch.int16), s2.view(torch.int16))
        # split-K reassociates fp32 sums, so the two bf16 results may round to
        # neighbouring values: allow two ulps of the larger plus a small floor
        # for outputs near zero (each is checked against the oracle elsewhere)
        diff = (s.float() - a.float()).abs()
        ulp = torch.maximum(a.float().abs(), s.float().abs()) * 2.0**-6 + 2.0**-12
        assert bool((diff <= ulp).all()), f"split {pt}: {float(diff.max())}"


def test_device_bounds_errors_zero_rows():
    c = cfg(num_seqs=4, ctx_lo=40, ctx_hi=200, num_q_heads=4, num_kv_heads=2)
    wl = to_device(W.generate(c, 17))
    kp, vp = device_pools(wl)
    fill_history(wl, kp, vp)
    for split in (-1, 32):
        good, _, _, st = run_gpu(wl, partition_request=split, pools=(kp, vp))
        assert st == K.PKV_OK
        for case in ("block", "len0", "len_big"):
            w2 = copy.copy(wl)
            w2.block_tables = wl.block_tables.clone()
            w2.context_lens = wl.context_lens.clone()
            if case == "block":
                w2.block_tables[1, 0] = wl.num_blocks
            elif case == "len0":
                w2.context_lens[1] = 0
            else:
                w2.context_lens[1] = c.max_context + 1
            err = torch.zeros(1, dtype=torch.int32, device="cuda")
            out = K.paged_attention_decode(w2.q, kp, vp, w2.block_tables, w2.context_lens, c.softmax_scale,
                                           max_context_len=c.max_context, partition_request=split, dev_err=err)
            assert K.read_device_error(err) == K.PKV_ERR_DEVICE_BOUNDS, case
            assert bool((out[1] == 0).all()), case
            for i in (0, 2, 3):
                assert torch.equal(out[i].view(torch.int16), good[i].view(torch.int16)), case


def test_workspace_too_small_is_refused():
    c = cfg(num_seqs=3, ctx_lo=100, ctx_hi=300)
    wl = to_device(W.generate(c, 18))
    kp, vp = device_pools(wl)
    plan = K.plan_decode(3, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.max_context, False, 64)
    assert plan["workspace_bytes"] > 0
    ws = torch.empty(plan["workspace_bytes"] - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(K.PagedKVError) as e:
        K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                 max_context_len=c.max_context, partition_request=64, workspace=ws)
    assert e.value.status == K.PKV_ERR_WORKSPACE


def test_canary_never_reaches_output():
    """Pools full of NaN outside the written slots: any stray read would show."""
    c = cfg(num_seqs=9, ctx_lo=1, ctx_hi=500, block_size=32)
    wl = to_device(W.generate(c, 19))
    out, _, _, st = run_gpu(wl, partition_request=0)
    assert st == K.PKV_OK and bool(torch.isfinite(out.float()).all())


def test_sequence_order_does_not_change_results():
    """seq_order only changes the schedule: outputs are bit-identical."""
    c = cfg(num_seqs=9, ctx_lo=1, ctx_hi=600, block_size=16)
    wl = to_device(W.generate(c, 20))
    kp, vp = device_pools(wl)
    fill_history(wl, kp, vp)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new)
    orders = [K.longest_first(wl.context_lens.cpu()).cuda(),
              torch.randperm(c.num_seqs, generator=torch.Generator().manual_seed(3)).to(torch.int32).cuda()]
    for split in (0, 64):
        base = K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                        max_context_len=c.max_context, partition_request=split)
        for o in orders:
            err = torch.zeros(1, dtype=torch.int32, device="cuda")
            out = K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                           max_context_len=c.max_context, partition_request=split, seq_order=o,
                                           dev_err=err)
            assert K.read_device_error(err) == K.PKV_OK
            assert torch.equal(out.view(torch.int16), base.view(torch.int16))
    # an entry outside the sequences is reported and skipped: the sequence it
    # displaced keeps its old out rows (split or not, after a call that left
    # that sequence's partials in the workspace), every other row is exact
    bad = orders[0].clone()
    skipped = int(bad[0])
    bad[0] = c.num_seqs
    for split in (0, 64):
        base = K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                        max_context_len=c.max_context, partition_request=split)
        plan = K.plan_decode(c.num_seqs, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.max_context,
                             False, split)
        ws = torch.empty(max(plan["workspace_bytes"], 256), dtype=torch.uint8, device="cuda")
        K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                 max_context_len=c.max_context, partition_request=split, workspace=ws)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = torch.full_like(wl.q, 7.0)
        K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale, out=out,
                                 max_context_len=c.max_context, partition_request=split, workspace=ws,
                                 seq_order=bad, dev_err=err)
        assert K.read_device_error(err) == K.PKV_ERR_DEVICE_BOUNDS
        assert bool((out[skipped].float() == 7.0).all())
        keep = [i for i in range(c.num_seqs) if i != skipped]
        assert torch.equal(out[keep].view(torch.int16), base[keep].view(torch.int16))

"""The seeded input generator: reproducible, and the bookkeeping is consistent."""

import pytest
import torch

from paged_kv_cache_482_b200 import workloads as W


def small(**kw):
    base = dict(name="t", num_seqs=5, num_q_heads=4, num_kv_heads=2, head_dim=16, block_size=4, ctx_lo=1, ctx_hi=19)
    base.update(kw)
    return W.DecodeConfig(**base)


@pytest.mark.parametrize("c", [small(), small(prefix_tokens=8, ctx_lo=0, ctx_hi=6), small(cache_dtype=W.CACHE_FP8)])
def test_same_seed_same_inputs(c):
    a, b = W.generate(c, 3), W.generate(c, 3)
    for f in ("q", "k_new", "v_new", "slot_new", "k_hist", "v_hist", "slot_hist", "block_tables", "context_lens"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    other = W.generate(c, 4)
    assert not torch.equal(a.q, other.q)


@pytest.mark.parametrize("c", [small(), small(prefix_tokens=8, ctx_lo=0, ctx_hi=6), small(block_size=16, ctx_lo=1, ctx_hi=70)])
def test_tables_slots_and_lengths(c):
    wl = W.generate(c, 5)
    bs, P = c.block_size, c.prefix_tokens
    ctx = wl.context_lens.long()
    assert int(ctx.min()) >= P + c.ctx_lo and int(ctx.max()) <= P + c.ctx_hi
    used = []
    for i in range(c.num_seqs):
        nb = -(-int(ctx[i]) // bs)
        row = wl.block_tables[i].tolist()
        assert all(b >= 0 for b in row[:nb]) and all(b == -1 for b in row[nb:])
        used += row[P // bs : nb]
    shared = wl.block_tables[:, : P // bs]
    assert (shared == shared[0]).all()
    assert len(set(used)) == len(used), "private blocks must be distinct"
    assert not set(used) & set(shared[0].tolist())
    in_use = len(used) + P // bs
    assert wl.num_blocks == in_use + -(-in_use // 10)
    # every written slot is distinct and sits at the right logical position
    written = torch.cat([wl.slot_hist, wl.slot_new[wl.slot_new >= 0]]).tolist()
    assert len(set(written)) == len(written)
    for i in range(c.num_seqs):
        last = int(ctx[i]) - 1
        s = int(wl.slot_new[i])
        if last < P:
            assert s == -1
        else:
            assert s == int(wl.block_tables[i, last // bs]) * bs + last % bs
        for p, r in enumerate(wl.hist_rows[i].tolist()):
            sl = int(wl.slot_hist[r])
            assert sl == int(wl.block_tables[i, p // bs]) * bs + p % bs


def test_fp8_scales_are_head_amax_over_448():
    c = small(cache_dtype=W.CACHE_FP8)
    wl = W.generate(c, 6)
    allk = torch.cat([wl.k_hist, wl.k_new])
    want = allk.abs().amax(dim=(0, 2)).float() / 448.0
    assert torch.equal(wl.k_scale, want)
    assert wl.k_scale.dtype == torch.float32 and wl.k_scale.shape == (c.num_kv_heads,)


def test_full_size_structure_matches_the_workloads():
    """Pool sizes of the full-size workloads (no K/V drawn)."""
    ctx, tables, nblk = W._structure(W.CONFIGS["qwen3_8b"], 0)
    assert ctx.numel() == 1024 and 100 <= int(ctx.min()) and int(ctx.max()) <= 2048
    assert tables.shape == (1024, 8) and 5000 < nblk < 6000
    ctx, tables, nblk = W._structure(W.CONFIGS["long_fp8"], 0)
    assert tables.shape == (64, 2048) and 16384 <= int(ctx.min()) and int(ctx.max()) <= 32768
    ctx, tables, nblk = W._structure(W.CONFIGS["prefix_shared"], 0)
    assert (tables[:, :4] == tables[0, :4]).all() and int(ctx.min()) >= 1024


def test_logical_kv_orders_rows():
    c = small(prefix_tokens=8, ctx_lo=0, ctx_hi=6)
    wl = W.generate(c, 7)
    for i in range(c.num_seqs):
        k, v = W.logical_kv(wl, i)
        n = int(wl.context_lens[i])
        assert k.shape == (n, c.num_kv_heads, c.head_dim)
        assert torch.equal(k[:8], wl.k_hist[:8])
        if n > 8:
            assert torch.equal(k[-1], wl.k_new[i])


@pytest.mark.parametrize("name", ["prefill_tiny", "prefill_qwen3_8b", "prefill_mixed"])
def test_prefill_bookkeeping(name):
    c = W.PREFILL_CONFIGS[name]
    wl = W.generate_prefill(c, 8) if name == "prefill_tiny" else None
    if wl is None:  # full size: structure only, no K/V drawn on the CPU
        wl = W.generate_prefill(c.with_(head_dim=8, num_q_heads=2, num_kv_heads=1), 8)
    S, bs = c.total_seqs, c.block_size
    cu, ctx = wl.cu_q_lens.long(), wl.context_lens.long()
    n = cu[1:] - cu[:-1]
    assert int(cu[0]) == 0 and int(cu[-1]) == wl.total_q and (n >= 1).all()
    assert (n[: c.num_seqs] >= c.chunk_lo).all() and (n[: c.num_seqs] <= c.chunk_hi).all()
    assert (n[c.num_seqs :] == 1).all()
    written = torch.cat([wl.slot_hist, wl.slot_new]).tolist()
    assert len(set(written)) == len(written) and min(written) >= 0 and max(written) < wl.num_blocks * bs
    for i in range(S):
        nb = -(-int(ctx[i]) // bs)
        row = wl.block_tables[i].tolist()
        assert all(b >= 0 for b in row[:nb]) and all(b == -1 for b in row[nb:])
        h = int(ctx[i] - n[i])
        assert len(wl.hist_rows[i]) == h
        for p in range(int(ctx[i])):  # every logical position's slot follows the table
            sl = int(wl.slot_hist[wl.hist_rows[i][p]]) if p < h else int(wl.slot_new[int(cu[i]) + p - h])
            assert sl == row[p // bs] * bs + p % bs

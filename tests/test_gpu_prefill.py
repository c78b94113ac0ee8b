"""Chunked-prefill paged attention on the GPU against the fp64 oracle.

Pools are filled with store_kvcache (history, then the chunk tokens) and the
tcgen05 prefill kernel attends; the oracle does the same on the host. Small
cases compare every row; the full-size Qwen3-8B-shaped steps (bf16 and E4M3 caches) compare sampled
rows, each recomputed by the oracle as a one-token chunk at its position
(a query's result depends only on the tokens up to it).
"""

import copy

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import compare, device_pools, pool_bytes
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu


def to_device(wl):
    w2 = copy.copy(wl)
    for f in ("q", "k_new", "v_new", "slot_new", "k_hist", "v_hist", "slot_hist", "block_tables", "cu_q_lens",
              "context_lens", "k_scale", "v_scale"):
        t = getattr(wl, f)
        if t is not None:
            setattr(w2, f, t.cuda().contiguous())
    return w2


def max_q_len(wl):
    cu = wl.cu_q_lens.cpu().long()
    return max(1, int((cu[1:] - cu[:-1]).max()))


def run_gpu(wl, pools=None, mq=None):
    kp, vp = pools if pools is not None else device_pools(wl)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if pools is None:
        K.store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist, wl.k_scale, wl.v_scale, err)
        K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale, err)
    out = K.paged_attention_prefill(wl.q, kp, vp, wl.block_tables, wl.cu_q_lens, wl.context_lens,
                                    wl.cfg.softmax_scale, mq or max_q_len(wl), k_scale=wl.k_scale,
                                    v_scale=wl.v_scale, dev_err=err)
    return out, kp, vp, K.read_device_error(err)


def check(cfg, seed=0):
    wl_cpu = W.generate_prefill(cfg, seed)
    wl = to_device(wl_cpu)
    out, kp, vp, st = run_gpu(wl)
    assert st == K.PKV_OK, f"device status {st}"
    ref, rkp, rvp, rst = O.run_prefill_workload(wl_cpu, num_threads=8)
    assert rst == O.ORC_OK
    assert np.array_equal(pool_bytes(kp), rkp) and np.array_equal(pool_bytes(vp), rvp)
    return compare(out, ref, wl.is_fp8, cfg.name), out, wl


SMALL = [
    W.PREFILL_CONFIGS["prefill_tiny"],                                           # d 64, G 2, bs 16
    W.PrefillConfig("g4_d128_bs16", 3, 8, 2, 128, 16, 100, 300, 1, 160),          # chunks across 128-token tiles
    W.PrefillConfig("g8_d64_bs256", 2, 8, 1, 64, 256, 0, 200, 20, 60),
    W.PrefillConfig("g1_d128", 2, 4, 4, 128, 16, 0, 150, 100, 300),                # 128 tokens per CTA
    W.PrefillConfig("g4_no_history", 3, 8, 2, 128, 256, 0, 0, 129, 257),          # the whole prompt is the chunk
    W.PrefillConfig("mixed", 2, 32, 8, 128, 256, 0, 700, 60, 200, decode_seqs=6, decode_hist_lo=1,
                    decode_hist_hi=900),
    W.PrefillConfig("fp8_bs16", 2, 8, 2, 128, 16, 50, 400, 30, 200, cache_dtype=W.CACHE_FP8),
    W.PrefillConfig("fp8_g8_d64", 2, 8, 1, 64, 256, 0, 300, 1, 90, cache_dtype=W.CACHE_FP8),
    # the smallest and largest block sizes the API accepts: 8-row copies, and
    # one block spanning sixteen 64-token tiles
    W.PrefillConfig("bs8_g4", 3, 32, 8, 128, 8, 0, 200, 40, 300),
    W.PrefillConfig("bs1024_g2_d64", 2, 8, 4, 64, 1024, 500, 1500, 70, 400),
    # E4M3 chunks longer than one query tile take the converter warps of the
    # warp-specialised kernel: every group size, both head sizes, the block
    # size extremes, and tails that end inside a 128-token tile
    W.PrefillConfig("fp8_g1_bs8", 2, 4, 4, 128, 8, 0, 300, 100, 300, cache_dtype=W.CACHE_FP8),
    W.PrefillConfig("fp8_g2_d64_bs1024", 2, 8, 4, 64, 1024, 500, 1500, 70, 400, cache_dtype=W.CACHE_FP8),
    W.PrefillConfig("fp8_g4_d128_bs256", 3, 32, 8, 128, 256, 0, 600, 33, 520, cache_dtype=W.CACHE_FP8),
    W.PrefillConfig("fp8_mixed", 2, 32, 8, 128, 16, 0, 700, 60, 200, decode_seqs=6, decode_hist_lo=1,
                    decode_hist_hi=900, cache_dtype=W.CACHE_FP8),
]


@pytest.mark.parametrize("cfg", SMALL, ids=[c.name for c in SMALL])
def test_prefill_matches_oracle(cfg):
    check(cfg, seed=1)


def test_exact_tile_boundaries():
    """Chunk and context lengths on multiples of the 128-token KV tile and of
    the 32-token query tile (G = 4)."""
    for hist, chunk in ((0, 128), (128, 128), (96, 32), (127, 1), (255, 129)):
        cfg = W.PrefillConfig(f"edge_{hist}_{chunk}", 1, 8, 2, 128, 16, hist, hist, chunk, chunk)
        check(cfg, seed=2)


def test_chunking_is_bit_invariant():
    """A prompt prefilled in one chunk or in two gives the same bits for every
    token: a row's arithmetic depends only on its own scores and the same
    128-token KV tiling."""
    cfg = W.PrefillConfig("split", 3, 32, 8, 128, 256, 0, 300, 300, 500)
    wl = to_device(W.generate_prefill(cfg, 3))
    out, kp, vp, st = run_gpu(wl)
    assert st == K.PKV_OK
    cu, cl = wl.cu_q_lens.long().cpu(), wl.context_lens.long().cpu()
    n = cu[1:] - cu[:-1]
    first = (n // 3 // 16) * 16 + 5  # not aligned to any tile
    rows1 = torch.cat([torch.arange(int(cu[i]), int(cu[i] + first[i])) for i in range(3)]).cuda()
    rows2 = torch.cat([torch.arange(int(cu[i] + first[i]), int(cu[i + 1])) for i in range(3)]).cuda()
    cu1 = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(first, 0)]).int().cuda()
    cu2 = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(n - first, 0)]).int().cuda()
    o1 = K.paged_attention_prefill(wl.q[rows1].contiguous(), kp, vp, wl.block_tables, cu1,
                                   (cl - (n - first)).int().cuda(), cfg.softmax_scale, int(first.max()))
    o2 = K.paged_attention_prefill(wl.q[rows2].contiguous(), kp, vp, wl.block_tables, cu2, wl.context_lens,
                                   cfg.softmax_scale, int((n - first).max()))
    assert torch.equal(o1, out[rows1]) and torch.equal(o2, out[rows2])


def test_one_token_chunks_agree_with_decode():
    cfg = W.PrefillConfig("decode_only", 0, 32, 8, 128, 256, 0, 0, 1, 1, decode_seqs=64, decode_hist_lo=1,
                          decode_hist_hi=3000)
    _, out, wl = check(cfg, seed=4)
    dec = K.paged_attention_decode(wl.q, *device_pools_filled(wl), wl.block_tables, wl.context_lens,
                                   cfg.softmax_scale)
    assert (out.float() - dec.float()).abs().max().item() <= 2e-2


def device_pools_filled(wl):
    kp, vp = device_pools(wl)
    K.store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist, wl.k_scale, wl.v_scale)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale)
    return kp, vp


def test_empty_chunks_and_loose_bound():
    """Sequences with no rows in the batch, and max_q_len above every chunk."""
    cfg = W.PrefillConfig("gaps", 4, 8, 2, 128, 16, 10, 200, 1, 70)
    wl_cpu = W.generate_prefill(cfg, 5)
    ref, _, _, _ = O.run_prefill_workload(wl_cpu, num_threads=8)
    wl = to_device(wl_cpu)
    kp, vp = device_pools_filled(wl)
    # drop sequence 1's rows: it stays in the batch with c = 0
    cu = wl_cpu.cu_q_lens.long()
    keep = torch.cat([torch.arange(int(cu[0]), int(cu[1])), torch.arange(int(cu[2]), int(cu[4]))])
    n = cu[1:] - cu[:-1]
    n[1] = 0
    cu2 = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(n, 0)]).int().cuda()
    cl = wl_cpu.context_lens.clone()
    out = K.paged_attention_prefill(wl.q[keep.cuda()].contiguous(), kp, vp, wl.block_tables, cu2, cl.cuda(),
                                    cfg.softmax_scale, 1000)
    compare(out, ref[keep.numpy()], False, "gaps")


@pytest.mark.parametrize("name", ["prefill_qwen3_8b", "prefill_fp8"])
def test_full_size_sampled(name):
    cfg = W.PREFILL_CONFIGS[name]
    wl = W.generate_prefill(cfg, 0, device="cuda")
    out, kp, vp, st = run_gpu(wl)
    assert st == K.PKV_OK
    assert bool(torch.isfinite(out.float()).all())
    g = torch.Generator().manual_seed(0)
    cu, cl = wl.cu_q_lens.cpu().long(), wl.context_lens.cpu().long()
    rows = []
    for s in range(cfg.total_seqs):
        n = int(cu[s + 1] - cu[s])
        for j in {0, n - 1, 31, 32, int(torch.randint(n, (1,), generator=g))}:
            if 0 <= j < n:
                rows.append((s, j))
    # each sampled row as a one-token chunk at its own position, over a host copy of its blocks
    kp_h, vp_h = pool_bytes(kp), pool_bytes(vp)
    q_rows = torch.stack([wl.q[int(cu[s]) + j] for s, j in rows]).cpu()
    bt = torch.stack([wl.block_tables[s] for s, _ in rows]).cpu()
    ctx = torch.tensor([int(cl[s] - (cu[s + 1] - cu[s]) + j + 1) for s, j in rows], dtype=torch.int32)
    cu1 = torch.arange(len(rows) + 1, dtype=torch.int32)
    ks = wl.k_scale.cpu() if wl.is_fp8 else None
    vs = wl.v_scale.cpu() if wl.is_fp8 else None
    ref, rst = O.paged_attention_prefill(q_rows, kp_h, vp_h, bt, cu1, ctx, cfg.num_kv_heads, cfg.block_size,
                                         cfg.softmax_scale, k_scale=ks, v_scale=vs, num_threads=8)
    assert rst == O.ORC_OK
    got = torch.stack([out[int(cu[s]) + j] for s, j in rows])
    compare(got, ref, wl.is_fp8, f"{name} sampled")


def test_device_bounds():
    cfg = W.PrefillConfig("bounds", 3, 8, 2, 128, 16, 20, 100, 5, 40)
    wl_cpu = W.generate_prefill(cfg, 6)
    ref, _, _, _ = O.run_prefill_workload(wl_cpu, num_threads=8)
    wl = to_device(wl_cpu)
    kp, vp = device_pools_filled(wl)
    cu = wl_cpu.cu_q_lens.long()
    r1 = slice(int(cu[1]), int(cu[2]))
    others = np.r_[0:int(cu[1]), int(cu[2]):wl.total_q]
    for what in ("block", "short_ctx", "long_chunk"):
        bt, cl, mq = wl.block_tables.clone(), wl.context_lens.clone(), max_q_len(wl)
        if what == "block":
            bt[1, 0] = wl.num_blocks
        elif what == "short_ctx":
            cl[1] = int(cu[2] - cu[1]) - 1
        else:
            mq -= 1  # the longest chunk is now longer than the stated bound
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = K.paged_attention_prefill(wl.q, kp, vp, bt, wl.cu_q_lens, cl, cfg.softmax_scale, mq, dev_err=err)
        assert K.read_device_error(err) == K.PKV_ERR_DEVICE_BOUNDS, what
        if what != "long_chunk":
            assert bool((out[r1] == 0).all()), what
            compare(out[torch.from_numpy(others).cuda()], ref[others], False, what)
    bad_cu = wl.cu_q_lens.clone()
    bad_cu[1] = wl.total_q + 5
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.paged_attention_prefill(wl.q, kp, vp, wl.block_tables, bad_cu, wl.context_lens, cfg.softmax_scale,
                              max_q_len(wl), dev_err=err)
    assert K.read_device_error(err) == K.PKV_ERR_DEVICE_BOUNDS


@pytest.mark.parametrize("dt", [W.CACHE_BF16, W.CACHE_FP8_TOKEN])
def test_mixed_batch_is_ordered_on_the_callers_stream(dt):
    """A mixed batch runs its one-token chunks on the library's side stream.
    Work queued on the caller's (non-default) stream right after the call,
    with no synchronisation in between, must see every output row: a copy
    taken that way equals the oracle's result, and a second call that
    overwrites the output on the same stream is not overtaken either."""
    cfg = W.PrefillConfig("ordered", 3, 32, 8, 128, 16, 100, 1500, 200, 400, cache_dtype=dt, decode_seqs=64,
                          decode_hist_lo=500, decode_hist_hi=3000)
    wl_cpu = W.generate_prefill(cfg, 3)
    wl = to_device(wl_cpu)
    kp, vp = device_pools(wl)
    if wl.token_scales:
        wl.k_scale, wl.v_scale = W.scale_pools(wl.num_blocks, cfg.num_kv_heads, cfg.block_size, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist, wl.k_scale, wl.v_scale, err)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale, err)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = torch.full_like(wl.q, float("nan"))
        K.paged_attention_prefill(wl.q, kp, vp, wl.block_tables, wl.cu_q_lens, wl.context_lens, cfg.softmax_scale,
                                  max_q_len(wl), k_scale=wl.k_scale, v_scale=wl.v_scale, out=out, dev_err=err)
        first = out.clone()  # queued right behind the call on s
        out.fill_(float("nan"))
        K.paged_attention_prefill(wl.q, kp, vp, wl.block_tables, wl.cu_q_lens, wl.context_lens, cfg.softmax_scale,
                                  max_q_len(wl), k_scale=wl.k_scale, v_scale=wl.v_scale, out=out, dev_err=err)
        second = out.clone()
    s.synchronize()
    assert K.read_device_error(err) == K.PKV_OK
    assert bool(torch.isfinite(first.float()).all()) and torch.equal(first.view(torch.int16), second.view(torch.int16))
    if dt == W.CACHE_BF16:
        ref, _, _, rst = O.run_prefill_workload(wl_cpu, num_threads=8)
        assert rst == O.ORC_OK
        compare(first, ref, False, "mixed batch on a side stream")

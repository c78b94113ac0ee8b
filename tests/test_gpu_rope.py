"""Fused rotary embedding + store_kvcache on the GPU against the oracle.

The rotated q, both pools and (per-token E4M3) both scale pools must equal
the oracle's bit for bit: the rotation's binary32 steps are part of the
contract, so the bf16 bits, the codes and the scales are decided the same way
on both sides. Then a decode over a cache filled this way must match the
oracle's attention over its own rotated cache.
"""

import os

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import compare, pool_bytes
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, len(os.sched_getaffinity(0))))


def _pools(wl, device):
    c = wl.cfg
    shape = (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)
    if c.is_fp8:
        kp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device=device)
        vp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device=device)
    else:
        kp = torch.full(shape, W.CANARY_BF16, dtype=torch.int16, device=device).view(torch.bfloat16)
        vp = torch.full(shape, W.CANARY_BF16, dtype=torch.int16, device=device).view(torch.bfloat16)
    return kp, vp


def _host_pools(wl):
    c = wl.cfg
    fill = W.CANARY_FP8 if c.is_fp8 else W.CANARY_BF16
    return (O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, c.is_fp8, fill),
            O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, c.is_fp8, fill))


def run_both(wl, positions=None, slots=None, with_q=True, in_place=False):
    """(gpu q_out, gpu pools, gpu scales, gpu status), (oracle ...)."""
    c = wl.cfg
    pos = wl.positions if positions is None else positions
    sl = wl.slot_mapping if slots is None else slots
    kp, vp = _pools(wl, "cuda")
    if c.token_scales:
        ks, vs = W.scale_pools(wl.num_blocks, c.num_kv_heads, c.block_size, device="cuda")
    else:
        ks = wl.k_scale.cuda() if wl.k_scale is not None else None
        vs = wl.v_scale.cuda() if wl.v_scale is not None else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = wl.q.cuda().contiguous() if with_q else None
    q_out = q if in_place else None
    q_out = K.store_kvcache_rope(wl.k.cuda(), wl.v.cuda(), kp, vp, sl.cuda(), pos.cuda(), wl.cos_sin.cuda(), q=q,
                                 q_out=q_out, style=c.style, k_scale=ks, v_scale=vs, dev_err=err)
    st = K.read_device_error(err)
    hk, hv = _host_pools(wl)
    if c.token_scales:
        hks, hvs = O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size), \
            O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size)
    else:
        hks, hvs = wl.k_scale, wl.v_scale
    rq, rst = O.store_kvcache_rope(wl.q if with_q else None, wl.k, wl.v, hk, hv, sl, pos, wl.cos_sin, wl.num_blocks,
                                   c.block_size, hks, hvs, style=c.style)
    return (q_out, kp, vp, ks, vs, st), (rq, hk, hv, hks, hvs, rst)


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _check_equal(g, r, wl, rows_written=None):
    q_out, kp, vp, ks, vs, st = g
    rq, hk, hv, hks, hvs, rst = r
    if q_out is not None:
        got = _bits(q_out)
        if rows_written is not None:
            got, rq = got[rows_written], rq[rows_written]
        assert np.array_equal(got, rq), "rotated q differs"
    assert np.array_equal(pool_bytes(kp), hk), "K pool differs"
    assert np.array_equal(pool_bytes(vp), hv), "V pool differs"
    if wl.cfg.token_scales:
        assert np.array_equal(ks.cpu().numpy().view(np.uint32), hks.view(np.uint32)), "K scale pool differs"
        assert np.array_equal(vs.cpu().numpy().view(np.uint32), hvs.view(np.uint32)), "V scale pool differs"


CASES = []
for dt in (W.CACHE_BF16, W.CACHE_FP8, W.CACHE_FP8_TOKEN):
    for style in (W.ROPE_HALF, W.ROPE_INTERLEAVED):
        for d, nq, nkv, bs in ((64, 4, 2, 16), (128, 32, 8, 256), (128, 8, 8, 8)):
            CASES.append(W.RopeConfig(f"rope_{dt}_s{style}_d{d}_g{nq // nkv}", 37, nq, nkv, d, bs, 40000,
                                      style=style, cache_dtype=dt))


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_bit_exact_against_oracle(cfg):
    wl = W.generate_rope(cfg, 41)
    g, r = run_both(wl)
    assert g[5] == K.PKV_OK and r[5] == O.ORC_OK
    _check_equal(g, r, wl)


@pytest.mark.parametrize("dt", [W.CACHE_BF16, W.CACHE_FP8_TOKEN])
def test_skipped_slots_bad_positions_keys_only_in_place(dt):
    cfg = W.RopeConfig("rope_edges", 12, 8, 2, 128, 16, 500, cache_dtype=dt)
    wl = W.generate_rope(cfg, 42)
    pos = wl.positions.clone()
    pos[3] = 500  # out of range: nothing of token 3 is written
    pos[7] = -2
    slots = wl.slot_mapping.clone()
    slots[5] = -1  # q rotated, nothing stored
    g, r = run_both(wl, positions=pos, slots=slots, in_place=True)
    assert g[5] == K.PKV_ERR_DEVICE_BOUNDS and r[5] == O.ORC_ERR_BOUNDS
    good = [i for i in range(cfg.num_tokens) if i not in (3, 7)]
    _check_equal(g, r, wl, rows_written=good)
    # keys only (no q)
    g, r = run_both(wl, with_q=False)
    assert g[0] is None and g[5] == K.PKV_OK and r[5] == O.ORC_OK
    _check_equal(g, r, wl)


@pytest.mark.parametrize("name", ["rope_qwen3_8b", "rope_prefill_qwen3_8b_fp8"])
def test_full_size_bit_exact(name):
    wl = W.generate_rope(W.ROPE_CONFIGS[name], 0)
    g, r = run_both(wl)
    assert g[5] == K.PKV_OK and r[5] == O.ORC_OK
    _check_equal(g, r, wl)


@pytest.mark.parametrize("dt", [W.CACHE_BF16, W.CACHE_FP8_TOKEN])
@pytest.mark.parametrize("style", [W.ROPE_HALF, W.ROPE_INTERLEAVED])
def test_decode_over_a_rotated_cache(dt, style):
    """Every cached token and each step token stored through the fused call at
    its own position, q rotated at the step position; decode against the
    oracle's decode over its own rotated cache."""
    c = W.DecodeConfig("rope_dec", 6, 16, 4, 128, 16, 1, 700, cache_dtype=dt)
    wl = W.generate(c, 43)
    mp = c.max_context
    cos_sin = W.rope_cache(mp, c.head_dim)
    hist_pos = torch.empty(wl.k_hist.shape[0], dtype=torch.int32)
    for rows in wl.hist_rows:
        hist_pos[rows] = torch.arange(len(rows), dtype=torch.int32)
    new_pos = (wl.context_lens - 1).to(torch.int32)
    shape = (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)
    if dt == W.CACHE_BF16:
        kp = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
        ks = vs = hks = hvs = None
    else:
        kp = torch.zeros(shape, dtype=torch.uint8, device="cuda")
        ks, vs = W.scale_pools(wl.num_blocks, c.num_kv_heads, c.block_size, device="cuda")
        hks = O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size)
        hvs = O.new_scale_pool(wl.num_blocks, c.num_kv_heads, c.block_size)
    vp = torch.zeros_like(kp)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cs = cos_sin.cuda()
    K.store_kvcache_rope(wl.k_hist.cuda(), wl.v_hist.cuda(), kp, vp, wl.slot_hist.cuda(), hist_pos.cuda(), cs,
                         style=style, k_scale=ks, v_scale=vs, dev_err=err)
    q_rot = K.store_kvcache_rope(wl.k_new.cuda(), wl.v_new.cuda(), kp, vp, wl.slot_new.cuda(), new_pos.cuda(), cs,
                                 q=wl.q.cuda(), style=style, k_scale=ks, v_scale=vs, dev_err=err)
    out = K.paged_attention_decode(q_rot, kp, vp, wl.block_tables.cuda(), wl.context_lens.cuda(), c.softmax_scale,
                                   k_scale=ks, v_scale=vs, max_context_len=c.max_context, dev_err=err)
    assert K.read_device_error(err) == K.PKV_OK
    fp8 = dt != W.CACHE_BF16
    hk = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, fp8, 0)
    hv = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, fp8, 0)
    _, st1 = O.store_kvcache_rope(None, wl.k_hist, wl.v_hist, hk, hv, wl.slot_hist, hist_pos, cos_sin,
                                  wl.num_blocks, c.block_size, hks, hvs, style=style)
    rq, st2 = O.store_kvcache_rope(wl.q, wl.k_new, wl.v_new, hk, hv, wl.slot_new, new_pos, cos_sin, wl.num_blocks,
                                   c.block_size, hks, hvs, style=style)
    assert st1 == st2 == O.ORC_OK
    assert np.array_equal(_bits(q_rot), rq)
    assert np.array_equal(pool_bytes(kp), hk) and np.array_equal(pool_bytes(vp), hv)
    ref, st = O.paged_attention_decode(torch.from_numpy(rq.view(np.int16)).view(torch.bfloat16), hk, hv,
                                       wl.block_tables, wl.context_lens, c.num_kv_heads, c.block_size,
                                       c.softmax_scale, hks, hvs, num_threads=THREADS)
    assert st == O.ORC_OK
    compare(out, ref, fp8, f"decode over rotated cache ({dt}, style {style})")

"""E4M3 chunked prefill through the widening workspace.

With a workspace, the codes of the long chunks' contexts are widened once
per call into dense 16-bit rows and the warp-specialised kernel copies its
tiles from there. The MMAs then see the same operand values as when every CTA
widens the codes itself, so the two paths must give the same bits; the staged
path is also compared with the fp64 oracle directly. The workspace is filled
with NaN bit patterns before each call, so a row the widening kernel did not
write and the attention kernel read would show.
"""

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import compare, device_pools
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W
from test_gpu_prefill import max_q_len, to_device

pytestmark = pytest.mark.gpu


def filled(wl):
    """Device pools (and per-token scale pools) holding the history and the chunk tokens."""
    kp, vp = device_pools(wl)
    ks, vs = wl.k_scale, wl.v_scale
    if wl.token_scales:
        ks, vs = W.scale_pools(wl.num_blocks, wl.cfg.num_kv_heads, wl.cfg.block_size, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist, ks, vs, err)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, ks, vs, err)
    assert K.read_device_error(err) == K.PKV_OK
    return kp, vp, ks, vs


def workspace_for(wl, block_tables=None):
    c = wl.cfg
    bt = wl.block_tables if block_tables is None else block_tables
    dt = K.PKV_CACHE_FP8_E4M3_TOKEN if wl.token_scales else K.PKV_CACHE_FP8_E4M3
    n = K.prefill_workspace_bytes(bt.shape[0], c.num_kv_heads, c.head_dim, bt.shape[1], c.block_size, dt)
    assert n > 0
    return torch.full((n,), 0xFF, dtype=torch.uint8, device="cuda")  # 0xFFFF: a NaN in f16 and bf16


def attend(wl, pools, ws=None, block_tables=None, context_lens=None, cu_q_lens=None, q=None, mq=None):
    kp, vp, ks, vs = pools
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.paged_attention_prefill(wl.q if q is None else q, kp, vp,
                                    wl.block_tables if block_tables is None else block_tables,
                                    wl.cu_q_lens if cu_q_lens is None else cu_q_lens,
                                    wl.context_lens if context_lens is None else context_lens,
                                    wl.cfg.softmax_scale, mq or max_q_len(wl), k_scale=ks, v_scale=vs, dev_err=err,
                                    workspace=ws)
    return out, K.read_device_error(err)


def same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


FP8 = W.CACHE_FP8
TOK = W.CACHE_FP8_TOKEN
CASES = [
    # every group size, both head sizes, block sizes 8 .. 1024, tails inside a 128-token tile
    W.PrefillConfig("st_g1_bs8", 2, 4, 4, 128, 8, 0, 300, 100, 300, cache_dtype=FP8),
    W.PrefillConfig("st_g2_d64_bs1024", 2, 8, 4, 64, 1024, 500, 1500, 70, 400, cache_dtype=FP8),
    W.PrefillConfig("st_g4_d128_bs16", 3, 32, 8, 128, 16, 0, 600, 33, 520, cache_dtype=FP8),
    W.PrefillConfig("st_g8_d64_bs256", 2, 8, 1, 64, 256, 0, 300, 17, 90, cache_dtype=FP8),
    W.PrefillConfig("st_g4_no_history", 3, 8, 2, 128, 256, 0, 0, 129, 257, cache_dtype=FP8),
    W.PrefillConfig("st_mixed", 2, 32, 8, 128, 16, 0, 700, 60, 200, decode_seqs=6, decode_hist_lo=1,
                    decode_hist_hi=900, cache_dtype=FP8),
    W.PrefillConfig("st_tok_g1_bs1024", 2, 4, 4, 128, 1024, 0, 1500, 130, 400, cache_dtype=TOK),
    W.PrefillConfig("st_tok_g2_d64_bs32", 2, 8, 4, 64, 32, 100, 600, 70, 300, cache_dtype=TOK),
    W.PrefillConfig("st_tok_g4_bs16", 3, 32, 8, 128, 16, 50, 400, 30, 300, cache_dtype=TOK),
    W.PrefillConfig("st_tok_g8_bs8", 2, 16, 2, 128, 8, 10, 150, 20, 90, cache_dtype=TOK),
    W.PrefillConfig("st_tok_mixed", 2, 32, 8, 128, 256, 0, 600, 60, 200, decode_seqs=4, decode_hist_lo=1,
                    decode_hist_hi=700, cache_dtype=TOK),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_staged_equals_in_kernel_widening_and_oracle(cfg):
    wl_cpu = W.generate_prefill(cfg, 7)
    wl = to_device(wl_cpu)
    pools = filled(wl)
    plain, st1 = attend(wl, pools)
    staged, st2 = attend(wl, pools, ws=workspace_for(wl))
    assert st1 == K.PKV_OK and st2 == K.PKV_OK
    assert same_bits(staged, plain), "staged and in-kernel widening differ"
    res = O.run_prefill_workload(wl_cpu, num_threads=8)
    assert res[3] == O.ORC_OK
    compare(staged, res[0], True, f"{cfg.name} staged")


@pytest.mark.parametrize("name", ["prefill_fp8", "prefill_fp8_token"])
def test_full_size_staged_equals_in_kernel(name):
    cfg = W.PREFILL_CONFIGS[name]
    wl = W.generate_prefill(cfg, 0, device="cuda")
    pools = filled(wl)
    plain, st1 = attend(wl, pools)
    staged, st2 = attend(wl, pools, ws=workspace_for(wl))
    assert st1 == K.PKV_OK and st2 == K.PKV_OK
    assert bool(torch.isfinite(staged.float()).all())
    assert same_bits(staged, plain)


def test_workspace_reused_by_a_shorter_batch():
    """A second call on the same workspace with shorter contexts and fewer
    sequences: the rows the first call left behind are never read."""
    big = W.PrefillConfig("reuse_big", 3, 32, 8, 128, 16, 800, 1200, 200, 300, cache_dtype=FP8)
    wl = to_device(W.generate_prefill(big, 8))
    pools = filled(wl)
    ws = workspace_for(wl)
    _, st = attend(wl, pools, ws=ws)
    assert st == K.PKV_OK
    small = W.PrefillConfig("reuse_small", 2, 32, 8, 128, 16, 0, 100, 130, 200, cache_dtype=FP8)
    wl2 = to_device(W.generate_prefill(small, 9))
    pools2 = filled(wl2)
    plain, _ = attend(wl2, pools2)
    staged, st = attend(wl2, pools2, ws=ws[:workspace_for(wl2).numel()])
    assert st == K.PKV_OK and same_bits(staged, plain)


def test_bad_block_id_with_staging():
    """A block id outside the pool in a long chunk's table: the widening
    kernel reads nothing through it, the attention kernel reports it and
    zeros that sequence's rows; the other sequences are unaffected."""
    cfg = W.PrefillConfig("st_bounds", 3, 8, 2, 128, 16, 20, 300, 100, 200, cache_dtype=FP8)
    wl_cpu = W.generate_prefill(cfg, 6)
    wl = to_device(wl_cpu)
    pools = filled(wl)
    bt = wl.block_tables.clone()
    bt[1, 2] = wl.num_blocks
    cu = wl_cpu.cu_q_lens.long()
    r1 = slice(int(cu[1]), int(cu[2]))
    others = torch.from_numpy(np.r_[0:int(cu[1]), int(cu[2]):wl.total_q]).cuda()
    plain, _ = attend(wl, pools)
    staged, st = attend(wl, pools, ws=workspace_for(wl), block_tables=bt)
    assert st == K.PKV_ERR_DEVICE_BOUNDS
    assert bool((staged[r1] == 0).all())
    assert same_bits(staged[others], plain[others])


def test_too_small_workspace_is_refused():
    cfg = W.PrefillConfig("st_small_ws", 2, 8, 2, 128, 16, 0, 100, 130, 200, cache_dtype=FP8)
    wl = to_device(W.generate_prefill(cfg, 10))
    pools = filled(wl)
    ws = workspace_for(wl)
    with pytest.raises(K.PagedKVError):
        attend(wl, pools, ws=ws[:-16])

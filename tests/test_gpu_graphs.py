"""The library's calls recorded in CUDA graphs: a replay gives the same bits
as the eager call. Covers the warp-MMA decode with split-K (tensor maps as
kernel parameters, the merge), the shared-prefix cascade, and a mixed
prefill batch (whose one-token chunks fork onto the library's side stream
and join back inside the capture)."""

import pytest
import torch

from gpu_harness import device_pools, fill_history, to_device
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _same(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("dt", [W.CACHE_BF16, W.CACHE_FP8])
def test_decode_replay_matches_eager(dt):
    c = W.DecodeConfig("graph_dec", 6, 32, 8, 128, 16, 100, 2500, cache_dtype=dt)
    wl = to_device(W.generate(c, 7))
    kp, vp = device_pools(wl)
    fill_history(wl, kp, vp)
    out = torch.empty_like(wl.q)
    plan = K.plan_decode(c.num_seqs, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.max_context,
                         wl.is_fp8, 256)
    ws = torch.empty(max(256, plan["workspace_bytes"]), dtype=torch.uint8, device="cuda")

    def step():
        K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale)
        K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale, out=out,
                                 k_scale=wl.k_scale, v_scale=wl.v_scale, max_context_len=c.max_context,
                                 partition_request=256, workspace=ws)

    step()
    torch.cuda.synchronize()
    eager = out.clone()
    replay = K.graphed(step)
    out.fill_(float("nan"))
    replay()
    torch.cuda.synchronize()
    assert _same(out, eager)


def test_shared_prefix_replay_matches_eager():
    parts = [W.generate(W.DecodeConfig("a", 9, 32, 8, 128, 16, 0, 200, prefix_tokens=256), 1),
             W.generate(W.DecodeConfig("b", 3, 32, 8, 128, 16, 1, 300), 2)]
    wl = to_device(W.merge(parts))
    kp, vp = device_pools(wl)
    fill_history(wl, kp, vp)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new)
    cu = torch.tensor(wl.group_bounds, dtype=torch.int32, device="cuda")
    pre = torch.tensor(wl.group_prefix, dtype=torch.int32, device="cuda")
    out = torch.empty_like(wl.q)
    plan = K.plan_decode_shared_prefix(wl.cfg.num_seqs, 32, 8, 128, 16, wl.cfg.max_context)
    ws = torch.empty(plan["workspace_bytes"], dtype=torch.uint8, device="cuda")

    def step():
        K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, wl.cfg.softmax_scale,
                                               cu, pre, 9, out=out, max_context_len=wl.cfg.max_context, workspace=ws)

    step()
    torch.cuda.synchronize()
    eager = out.clone()
    replay = K.graphed(step)
    out.fill_(float("nan"))
    replay()
    torch.cuda.synchronize()
    assert _same(out, eager)


def test_mixed_prefill_replay_matches_eager():
    from test_gpu_prefill import max_q_len
    from test_gpu_prefill import to_device as prefill_to_device

    cfg = W.PrefillConfig("graph_mixed", 2, 32, 8, 128, 16, 100, 900, 100, 300, decode_seqs=20, decode_hist_lo=50,
                          decode_hist_hi=1500)
    wl = prefill_to_device(W.generate_prefill(cfg, 4))
    kp, vp = device_pools(wl)
    K.store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new)
    out = torch.empty_like(wl.q)
    mq = max_q_len(wl)

    def step():
        K.paged_attention_prefill(wl.q, kp, vp, wl.block_tables, wl.cu_q_lens, wl.context_lens, cfg.softmax_scale, mq,
                                  out=out)

    step()
    torch.cuda.synchronize()
    eager = out.clone()
    replay = K.graphed(step)
    out.fill_(float("nan"))
    replay()
    torch.cuda.synchronize()
    assert _same(out, eager)

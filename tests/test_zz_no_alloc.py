"""The decode entry point for callers that cannot allocate device memory.

pkv_paged_attention_decode_static_scratch takes its split-K scratch from a
fixed array inside the library instead of a caller-provided workspace, for
callers with no device allocator at hand (an engine that reserves all device
memory for its KV pool at start-up, a plugin that cannot reach its host
framework's allocator through a C ABI). It must give the same result as the
workspace entry point, call after call, since every call reuses the same
array. This file is collected last so that a run stopping at the first
failure has already run every other test.
"""

import pytest
import torch

from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

def _setup(cfg, seed):
    wl = W.generate(cfg, seed)
    dev = {f: getattr(wl, f).cuda().contiguous() if getattr(wl, f) is not None else None
           for f in ("q", "k_new", "v_new", "slot_new", "k_hist", "v_hist", "slot_hist", "block_tables",
                     "context_lens", "k_scale", "v_scale")}
    shape = (wl.num_blocks, cfg.num_kv_heads, cfg.block_size, cfg.head_dim)
    if wl.is_fp8:
        kp = torch.zeros(shape, dtype=torch.uint8, device="cuda")
    else:
        kp = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    K.store_kvcache(dev["k_hist"], dev["v_hist"], kp, vp, dev["slot_hist"], dev["k_scale"], dev["v_scale"])
    K.store_kvcache(dev["k_new"], dev["v_new"], kp, vp, dev["slot_new"], dev["k_scale"], dev["v_scale"])
    return wl, dev, kp, vp


def _padded_tables(bt, width):
    """Block tables widened to `width` columns with -1 (unused entries)."""
    if bt.shape[1] >= width:
        return bt
    pad = torch.full((bt.shape[0], width - bt.shape[1]), -1, dtype=bt.dtype, device=bt.device)
    return torch.cat([bt, pad], dim=1).contiguous()


def _both(d, kp, vp, cfg, part, max_ctx, width, fp8):
    """(static-scratch result, workspace result) on the same inputs and plan."""
    bt = _padded_tables(d["block_tables"], width)
    ref = K.paged_attention_decode(d["q"], kp, vp, bt, d["context_lens"], cfg.softmax_scale, k_scale=d["k_scale"],
                                   v_scale=d["v_scale"], max_context_len=max_ctx, partition_request=part)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full_like(d["q"], float("nan"))
    K.paged_attention_decode_static_scratch(d["q"], kp, vp, bt, d["context_lens"], cfg.softmax_scale, out=out,
                                            k_scale=d["k_scale"], v_scale=d["v_scale"], max_context_len=max_ctx,
                                            partition_request=part, dev_err=err)
    assert K.read_device_error(err) == K.PKV_OK
    return out, ref


@pytest.mark.gpu
@pytest.mark.parametrize("cfg,part", [
    (W.DecodeConfig("na_bf16", 6, 16, 4, 128, 16, 200, 1500), 256),
    (W.DecodeConfig("na_fp8", 5, 32, 8, 128, 16, 600, 2500, cache_dtype=W.CACHE_FP8), 0),
    (W.DecodeConfig("na_bf16_d64", 4, 4, 2, 64, 32, 1, 900), 128),
])
def test_static_scratch_matches_workspace_entry_point_twice(cfg, part):
    """Two calls in a row on different batches: the second batch has shorter
    contexts, so it has fewer partitions per sequence than the first and the
    array still holds first-call partials that would be wrong if read. Both
    results must be bit-identical to the workspace entry point on the same
    inputs and plan (the same kernels run on the same data)."""
    wl_a, da, kpa, vpa = _setup(cfg, 5)
    short = cfg.with_(name=cfg.name + "_short", ctx_lo=1, ctx_hi=max(2, cfg.ctx_hi // 3))
    wl_b, db, kpb, vpb = _setup(short, 6)
    max_ctx = cfg.max_context
    width = da["block_tables"].shape[1]
    plan = K.plan_decode(cfg.num_seqs, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size, max_ctx,
                         wl_a.is_fp8, part)
    assert plan["workspace_bytes"] > 0, "the case must exercise the split-K scratch"
    pt = plan["partition_tokens"]
    parts_a = (-(-da["context_lens"].long() // pt)).max().item()
    parts_b = (-(-db["context_lens"].long() // pt)).max().item()
    assert parts_b < parts_a, "the second call must leave stale first-call partials behind"
    for d, kp, vp, wl in ((da, kpa, vpa, wl_a), (db, kpb, vpb, wl_b)):
        out, ref = _both(d, kp, vp, cfg, part, max_ctx, width, wl.is_fp8)
        assert bool(torch.isfinite(out.float()).all())
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_plan_beyond_the_array_is_refused_before_launch():
    """A split that needs more scratch than the array holds returns
    PKV_ERR_WORKSPACE on the host, without touching the device."""
    L = K.lib()
    S, nq, nkv, d, bs, max_ctx, part = 1024, 32, 8, 128, 16, 32768, 64
    p = K.plan_decode(S, nq, nkv, d, bs, max_ctx, False, part)
    assert p["workspace_bytes"] > K.STATIC_SCRATCH_BYTES
    st = L.pkv_paged_attention_decode_static_scratch(0x10000, 0x20000, 0x30000, 0x40000, max_ctx // bs, 0x50000, None, S,
                                                     nq, nkv, d, bs, 100000, 0.088, 0, None, None, max_ctx, part,
                                                     0x60000, None, None)
    assert st == K.PKV_ERR_WORKSPACE

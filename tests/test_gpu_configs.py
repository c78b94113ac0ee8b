"""The five workloads at full size, in the launch configuration the benchmark times."""

import os

import pytest

from gpu_harness import check_sampled, check_workload, sample_ids
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, len(os.sched_getaffinity(0))))


def test_tiny_full():
    check_workload(W.generate(W.CONFIGS["tiny"], 1), threads=THREADS)


def test_qwen3_0p6b_full():
    check_workload(W.generate(W.CONFIGS["qwen3_0.6b"], 1), threads=THREADS)


def test_qwen3_8b_sampled():
    wl = W.generate(W.CONFIGS["qwen3_8b"], 0, device="cuda")
    check_sampled(wl, sample_ids(wl, 48), threads=THREADS)


def test_prefix_shared_sampled():
    wl = W.generate(W.CONFIGS["prefix_shared"], 0, device="cuda")
    ids = sample_ids(wl, 48)
    # include sequences whose step token sits inside the shared prefix (slot -1)
    zero = (wl.slot_new < 0).nonzero().flatten().tolist()[:4]
    check_sampled(wl, sorted(set(ids) | set(zero)), threads=THREADS)


def edge_lengths(cfg, n_edges=8):
    """{sequence: length} putting n_edges sequences on split-K partition
    edges of the plan the launch uses: exact multiples of its partition
    length, one token past, and one token short."""
    p = K.plan_decode(cfg.num_seqs, cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size,
                      cfg.max_context, cfg.cache_dtype != W.CACHE_BF16)
    pt = p["partition_tokens"]
    assert pt > 0, "the workload must split"
    lens = []
    for k in range(1, cfg.max_context // pt + 1):
        for delta in (0, 1, -1):
            n = k * pt + delta
            if cfg.ctx_lo <= n <= cfg.ctx_hi:
                lens.append(n)
    lens = sorted(set(lens))[:n_edges]
    step = max(1, cfg.num_seqs // max(1, len(lens)))
    return {1 + i * step: n for i, n in enumerate(lens)}, pt


def _sampled_at_edges(name):
    cfg = W.CONFIGS[name]
    override, pt = edge_lengths(cfg)
    wl = W.generate(cfg, 0, device="cuda", ctx_override=override)
    ids = sorted(set(sample_ids(wl, 10)) | set(override))
    assert len(ids) >= 16
    cl = wl.context_lens.cpu()
    assert any(int(cl[i]) % pt == 0 for i in ids) and any(int(cl[i]) % pt == 1 for i in ids)
    check_sampled(wl, ids, threads=THREADS)


def test_long_fp8_sampled():
    """The full-size split-K step; 16+ sequences checked, among them lengths
    on partition edges (k * P, k * P + 1, k * P - 1)."""
    _sampled_at_edges("long_fp8")

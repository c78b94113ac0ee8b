"""The five workloads at full size, in the launch configuration the benchmark times."""

import os

import pytest

from gpu_harness import check_sampled, check_workload, sample_ids
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


def test_long_fp8_sampled():
    wl = W.generate(W.CONFIGS["long_fp8"], 0, device="cuda")
    check_sampled(wl, sample_ids(wl, 5), threads=THREADS)

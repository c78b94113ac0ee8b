"""Host-side helpers of bench.py that need no GPU: the sizing of the CPU
oracle's probe sample."""

import types

import torch

import bench


def _wl(lens):
    return types.SimpleNamespace(context_lens=torch.tensor(lens, dtype=torch.int32))


def test_probe_takes_at_least_one_sequence():
    # a single sequence longer than the token budget is still probed
    assert bench.probe_size(_wl([100_000, 5, 5]), [0, 1, 2], threads=8, max_tokens=32768) == 1


def test_probe_stops_at_the_token_budget():
    lens = [10_000] * 10
    # 10k + 10k + 10k = 30k fits, a fourth would pass 32768
    assert bench.probe_size(_wl(lens), list(range(10)), threads=16, max_tokens=32768) == 3


def test_probe_is_capped_by_threads_and_by_the_sample():
    lens = [10] * 100
    assert bench.probe_size(_wl(lens), list(range(100)), threads=8) == 8
    assert bench.probe_size(_wl(lens), list(range(100)), threads=1) == 4  # at least four when they fit
    assert bench.probe_size(_wl(lens[:2]), [0, 1], threads=8) == 2


def test_probe_follows_the_given_order():
    lens = [40_000, 10, 10, 10]
    # the order decides which sequences are probed: the long one first stops the probe at one
    assert bench.probe_size(_wl(lens), [0, 1, 2, 3], threads=8) == 1
    assert bench.probe_size(_wl(lens), [1, 2, 3, 0], threads=8) == 3

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


def _pwl(cu, ctx, fp8=False, token_scales=False, nq=8, nkv=2, d=128):
    cfg = types.SimpleNamespace(num_q_heads=nq, num_kv_heads=nkv, head_dim=d)
    return types.SimpleNamespace(cfg=cfg, cu_q_lens=torch.tensor(cu, dtype=torch.int32),
                                 context_lens=torch.tensor(ctx, dtype=torch.int32), is_fp8=fp8,
                                 token_scales=token_scales)


def test_prefill_split_separates_chunks_from_decode_rows():
    # chunk of 3 after a history of 2 (keys 3 + 4 + 5), two decode rows with contexts 10 and 7
    wl = _pwl([0, 3, 4, 5], [5, 10, 7])
    flops, kv = bench.prefill_split(wl)
    assert flops == (3 + 4 + 5) * 8 * 4 * 128
    assert kv == (10 + 7) * 2 * (2 * 128 * 2)  # bf16 K and V rows per KV head
    # the FLOPs of every row together are the chunk FLOPs plus the decode rows' own
    assert bench.prefill_flops(wl) == flops + (10 + 7) * 8 * 4 * 128
    # E4M3: one byte per element; per-token scales add a K and a V scale per row
    assert bench.prefill_split(_pwl([0, 1], [9], fp8=True))[1] == 9 * 2 * 2 * 128
    assert bench.prefill_split(_pwl([0, 1], [9], fp8=True, token_scales=True))[1] == 9 * 2 * (2 * 128 + 8)
    # no decode rows: nothing to stream
    assert bench.prefill_split(_pwl([0, 4], [4]))[1] == 0

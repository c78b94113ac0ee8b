"""Shared-prefix (cascade) decode on the GPU against the fp64 oracle.

Groups of consecutive sequences share their first P tokens (the same
physical blocks); the prefix kernel attends those once per group of members,
the decode kernel each sequence's own tokens, the split-K merge combines
them. The oracle knows nothing of groups: it attends every sequence over its
whole context through its own block table, so agreement pins the split, the
merge and the member-to-column mapping.
"""

import os

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import compare, device_pools, fill_history, sample_ids, to_device
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu
THREADS = max(1, min(32, len(os.sched_getaffinity(0))))


def groups_of(wl, device="cuda"):
    cu = torch.tensor(wl.group_bounds, dtype=torch.int32, device=device)
    pre = torch.tensor(wl.group_prefix, dtype=torch.int32, device=device)
    return cu, pre, max(b - a for a, b in zip(wl.group_bounds[:-1], wl.group_bounds[1:]))


def pools_for(wl):
    """Device pools (and per-token scale pools) filled with the workload's
    history and step tokens."""
    c = wl.cfg
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    if wl.token_scales:
        shape = (wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim)
        kp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device="cuda")
        vp = torch.full(shape, W.CANARY_FP8, dtype=torch.uint8, device="cuda")
        ks, vs = W.scale_pools(wl.num_blocks, c.num_kv_heads, c.block_size, device="cuda")
        wl.k_scale, wl.v_scale = ks, vs
    else:
        kp, vp = device_pools(wl)
    fill_history(wl, kp, vp, err)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale, err)
    assert K.read_device_error(err) == K.PKV_OK
    return kp, vp


def run_shared(wl, kp, vp, partition=0, cu=None, pre=None):
    c = wl.cfg
    cu0, pre0, mg = groups_of(wl)
    cu = cu0 if cu is None else cu
    pre = pre0 if pre is None else pre
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                                 cu, pre, mg, k_scale=wl.k_scale, v_scale=wl.v_scale,
                                                 max_context_len=c.max_context, partition_request=partition,
                                                 dev_err=err)
    return out, K.read_device_error(err)


def oracle_of(wl_cpu, seq_ids=None):
    res = O.run_workload(wl_cpu, num_threads=THREADS, seq_ids=seq_ids)
    assert res[3] == O.ORC_OK
    return res[0]


def mixed_groups(dt, g=4, bs=16, seed=0):
    """Three groups: five sequences sharing 64 tokens, one sequence alone,
    seven sharing 256 tokens with own suffixes of 0..100 tokens (some step
    tokens inside the prefix), and 40 sharing 32 tokens (more members than
    one block takes)."""
    nq, nkv = 2 * g, 2
    mk = lambda name, S, lo, hi, P: W.DecodeConfig(name, S, nq, nkv, 128, bs, lo, hi, cache_dtype=dt,  # noqa: E731
                                                   prefix_tokens=P)
    parts = [W.generate(mk("a", 5, 0, 80, 64), seed + 1), W.generate(mk("b", 1, 1, 120, 0), seed + 2),
             W.generate(mk("c", 7, 0, 100, 256), seed + 3), W.generate(mk("d", 40, 1, 60, 32), seed + 4)]
    return W.merge(parts)


CASES = [(dt, g) for dt in (W.CACHE_BF16, W.CACHE_FP8, W.CACHE_FP8_TOKEN) for g in (1, 4, 8)] + [(W.CACHE_BF16, 2)]


@pytest.mark.parametrize("dt,g", CASES, ids=[f"{dt}-g{g}" for dt, g in CASES])
@pytest.mark.parametrize("partition", [0, 32])
def test_groups_match_oracle_and_plain_decode(dt, g, partition):
    wl_cpu = mixed_groups(dt, g)
    wl = to_device(wl_cpu)
    kp, vp = pools_for(wl)
    out, st = run_shared(wl, kp, vp, partition)
    assert st == K.PKV_OK
    ref = oracle_of(wl_cpu)
    compare(out, ref, dt != W.CACHE_BF16, f"shared prefix {dt} g{g} p{partition}")
    plain = K.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, wl.cfg.softmax_scale,
                                     k_scale=wl.k_scale, v_scale=wl.v_scale, max_context_len=wl.cfg.max_context)
    tol = 5e-2 if dt != W.CACHE_BF16 else 2e-2
    assert float((out.float() - plain.float()).abs().max()) <= tol


def test_bs256_and_bs8():
    for bs in (8, 256):
        parts = [W.generate(W.DecodeConfig("a", 9, 32, 8, 128, bs, 0, 300, prefix_tokens=2 * max(bs, 256)), 5),
                 W.generate(W.DecodeConfig("b", 3, 32, 8, 128, bs, 1, 700), 6)]
        wl_cpu = W.merge(parts)
        wl = to_device(wl_cpu)
        kp, vp = pools_for(wl)
        out, st = run_shared(wl, kp, vp)
        assert st == K.PKV_OK
        compare(out, oracle_of(wl_cpu), False, f"shared prefix bs {bs}")


def test_bad_groups_zero_only_their_rows():
    """A member whose shared block ids differ from the first member's, and a
    group whose prefix is not a whole number of blocks: PKV_DEVERR_BOUNDS,
    zeros in exactly those sequences' rows, the others still correct."""
    wl_cpu = mixed_groups(W.CACHE_BF16)
    wl = to_device(wl_cpu)
    kp, vp = pools_for(wl)
    bt = wl.block_tables.clone()
    victim = wl.group_bounds[2] + 3  # a member of the 256-token group
    bt[victim, 1] = (bt[victim, 1] + 1) % wl.num_blocks  # a different block in its shared part
    wl.block_tables = bt
    cu, pre, mg = groups_of(wl)
    pre_bad = pre.clone()
    pre_bad[0] = 40  # not a multiple of 16 (the block size): the whole first group
    out, st = run_shared(wl, kp, vp, cu=cu, pre=pre_bad)
    assert st == K.PKV_ERR_DEVICE_BOUNDS
    zero = list(range(wl.group_bounds[0], wl.group_bounds[1])) + [victim]
    assert bool((out[zero].float() == 0).all())
    keep = [i for i in range(wl.cfg.num_seqs) if i not in zero]
    ref = oracle_of(wl_cpu)
    compare(out[keep], ref[keep], False, "rows outside the bad groups")


def test_prefix_shared_full_size_sampled():
    wl = W.generate(W.CONFIGS["prefix_shared"], 0, device="cuda")
    kp, vp = pools_for(wl)
    out, st = run_shared(wl, kp, vp)
    assert st == K.PKV_OK and bool(torch.isfinite(out.float()).all())
    ids = sorted(set(sample_ids(wl, 24)) | set((wl.slot_new < 0).nonzero().flatten().tolist()[:4]))
    ref = oracle_of(wl, seq_ids=ids)
    compare(out[torch.tensor(ids, device="cuda")], ref, False, "prefix_shared full size")


@pytest.mark.parametrize("dt", [W.CACHE_BF16, W.CACHE_FP8])
def test_cascade_is_ordered_on_the_callers_stream(dt):
    """The bf16 cascade runs its suffix decode on the library's side stream,
    beside the shared-prefix kernel on the caller's stream. Work queued on the
    caller's (non-default) stream right after the call, with no
    synchronisation in between, must see every output row, and a second call
    that overwrites the output on the same stream must not be overtaken."""
    wl_cpu = mixed_groups(dt, g=4, bs=16, seed=11)
    wl = to_device(wl_cpu)
    kp, vp = pools_for(wl)
    cu, pre, mg = groups_of(wl)
    c = wl.cfg
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = torch.full_like(wl.q, float("nan"))
        kw = dict(out=out, k_scale=wl.k_scale, v_scale=wl.v_scale, max_context_len=c.max_context, dev_err=err)
        K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale, cu,
                                               pre, mg, **kw)
        first = out.clone()  # queued right behind the call on s
        out.fill_(float("nan"))
        K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale, cu,
                                               pre, mg, **kw)
        second = out.clone()
    s.synchronize()
    assert K.read_device_error(err) == K.PKV_OK
    assert bool(torch.isfinite(first.float()).all())
    assert torch.equal(first.view(torch.int16), second.view(torch.int16))
    compare(first, oracle_of(wl_cpu), dt != W.CACHE_BF16, f"cascade on a side stream ({dt})")


@pytest.mark.parametrize("dt", [W.CACHE_BF16, W.CACHE_FP8_TOKEN])
def test_cascade_with_seq_order_is_bit_identical(dt):
    """A visiting order (longest first, and a reversed one) changes when each
    sequence's suffix runs, not what it computes: same bits as the natural
    order; an order entry outside the batch is reported and its row skipped."""
    wl_cpu = mixed_groups(dt, g=4, bs=16, seed=12)
    wl = to_device(wl_cpu)
    kp, vp = pools_for(wl)
    cu, pre, mg = groups_of(wl)
    c = wl.cfg
    kw = dict(k_scale=wl.k_scale, v_scale=wl.v_scale, max_context_len=c.max_context)
    base = K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                                  cu, pre, mg, **kw)
    S = c.num_seqs
    for order in (K.longest_first(wl_cpu.context_lens).cuda(), torch.arange(S - 1, -1, -1, dtype=torch.int32,
                                                                            device="cuda")):
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                                                     c.softmax_scale, cu, pre, mg, dev_err=err, seq_order=order, **kw)
        assert K.read_device_error(err) == K.PKV_OK
        assert torch.equal(out.view(torch.int16), base.view(torch.int16))
    bad = torch.arange(S, dtype=torch.int32, device="cuda")
    bad[5] = S + 3  # sequence 5 is named by no valid entry
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full_like(base, 7.0)
    K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale, cu, pre,
                                           mg, out=out, dev_err=err, seq_order=bad, **kw)
    assert K.read_device_error(err) == K.PKV_ERR_DEVICE_BOUNDS
    keep = [i for i in range(S) if i != 5]
    assert torch.equal(out[keep].view(torch.int16), base[keep].view(torch.int16))


def test_group_larger_than_the_stated_bound():
    """max_group_seqs below the largest group: the prefix kernels' grid does not
    cover that group's later members, so the whole group is reported
    (PKV_DEVERR_BOUNDS) and written as zeros; the other groups are exact."""
    wl_cpu = mixed_groups(W.CACHE_BF16, g=4, bs=16, seed=13)
    wl = to_device(wl_cpu)
    kp, vp = pools_for(wl)
    cu, pre, _ = groups_of(wl)
    sizes = [b - a for a, b in zip(wl.group_bounds[:-1], wl.group_bounds[1:])]
    bound = sorted(sizes)[-2]  # below the largest group (40 members), at least the others
    big = sizes.index(max(sizes))
    c = wl.cfg
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = K.paged_attention_decode_shared_prefix(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.softmax_scale,
                                                 cu, pre, bound, k_scale=wl.k_scale, v_scale=wl.v_scale,
                                                 max_context_len=c.max_context, dev_err=err)
    assert K.read_device_error(err) == K.PKV_ERR_DEVICE_BOUNDS
    zero = list(range(wl.group_bounds[big], wl.group_bounds[big + 1]))
    assert bool((out[zero].float() == 0).all())
    keep = [i for i in range(c.num_seqs) if i not in zero]
    compare(out[keep], oracle_of(wl_cpu)[keep], False, "groups within the bound")

"""DecodeStep.run_host: host inputs in, host output out, the copies of one
step overlapping the kernels of the next on copy streams with two buffer
sets. A sequence of steps with inputs that change every step must give, step
for step, the bits of the same steps run on device inputs."""

import pytest
import torch

from gpu_harness import device_pools, fill_history, to_device
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dt,shared", [(W.CACHE_BF16, False), (W.CACHE_FP8, False), (W.CACHE_BF16, True)])
def test_pipelined_host_steps_match_device_steps(dt, shared):
    c = W.DecodeConfig("e2e", 8, 32, 8, 128, 16, 0 if shared else 50, 600, cache_dtype=dt,
                       prefix_tokens=64 if shared else 0)
    wl = to_device(W.generate(c, 9))
    groups = (wl.group_bounds, wl.group_prefix, c.num_seqs) if shared else None
    pools = []
    for _ in range(2):
        kp, vp = device_pools(wl)
        fill_history(wl, kp, vp)
        pools.append((kp, vp))
    steps = [K.DecodeStep(kp, vp, c.num_seqs, c.num_q_heads, wl.block_tables.shape[1], c.softmax_scale,
                          wl.k_scale, wl.v_scale, max_context_len=c.max_context, groups=groups) for kp, vp in pools]
    g = torch.Generator(device="cuda").manual_seed(3)
    n = 6
    seq_inputs = []
    for i in range(n):  # every step brings new q and new K/V rows for the same slots
        q = torch.randn(wl.q.shape, generator=g, device="cuda").to(torch.bfloat16)
        kn = torch.randn(wl.k_new.shape, generator=g, device="cuda").to(torch.bfloat16)
        vn = torch.randn(wl.v_new.shape, generator=g, device="cuda").to(torch.bfloat16)
        seq_inputs.append((q, kn, vn, wl.slot_new, wl.block_tables, wl.context_lens))
    expected = []
    for inp in seq_inputs:  # device inputs, one step at a time
        expected.append(steps[0].run(*inp, seq_order=K.longest_first(wl.context_lens.cpu()).cuda()).clone())
    torch.cuda.synchronize()
    host_inputs = [[t.cpu().pin_memory() for t in inp] for inp in seq_inputs]
    outs = [torch.empty(wl.q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(n)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for inp, out in zip(host_inputs, outs):
            steps[1].run_host(*inp, out)
        steps[1].flush()
    s.synchronize()
    assert int(steps[1].dev_err.item()) == 0
    for i in range(n):
        assert torch.equal(outs[i].view(torch.int16), expected[i].cpu().view(torch.int16)), f"step {i}"

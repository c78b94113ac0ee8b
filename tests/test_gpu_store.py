"""store_kvcache on the GPU: bit-exact against the oracle's store."""

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import device_pools, pool_bytes, to_device
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu


def small(**kw):
    base = dict(name="store", num_seqs=6, num_q_heads=4, num_kv_heads=2, head_dim=128, block_size=16, ctx_lo=1,
                ctx_hi=70)
    base.update(kw)
    return W.DecodeConfig(**base)


@pytest.mark.parametrize("c", [small(), small(head_dim=64, num_kv_heads=3, num_q_heads=6),
                               small(cache_dtype=W.CACHE_FP8), small(cache_dtype=W.CACHE_FP8, head_dim=64),
                               small(prefix_tokens=32, ctx_lo=0, ctx_hi=40, block_size=16)],
                         ids=["bf16", "bf16-d64", "fp8", "fp8-d64", "prefix"])
def test_store_pools_bit_exact(c):
    wl_cpu = W.generate(c, 1)
    wl = to_device(wl_cpu)
    kp, vp = device_pools(wl)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist, wl.k_scale, wl.v_scale, err)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.k_scale, wl.v_scale, err)
    assert K.read_device_error(err) == K.PKV_OK
    fill = W.CANARY_FP8 if wl.is_fp8 else W.CANARY_BF16
    rk = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, wl.is_fp8, fill)
    rv = O.new_pool(wl.num_blocks, c.num_kv_heads, c.block_size, c.head_dim, wl.is_fp8, fill)
    assert O.store_kvcache(wl_cpu.k_hist, wl_cpu.v_hist, rk, rv, wl_cpu.slot_hist, wl.num_blocks, c.block_size,
                           wl_cpu.k_scale, wl_cpu.v_scale) == O.ORC_OK
    assert O.store_kvcache(wl_cpu.k_new, wl_cpu.v_new, rk, rv, wl_cpu.slot_new, wl.num_blocks, c.block_size,
                           wl_cpu.k_scale, wl_cpu.v_scale) == O.ORC_OK
    assert np.array_equal(pool_bytes(kp), rk)
    assert np.array_equal(pool_bytes(vp), rv)


@pytest.mark.parametrize("scale", [1.0, 0.0123, 3.7, 1.0 / 448.0, 2.0**-10])
def test_fp8_codes_for_every_bf16_value(scale):
    """Every finite bf16 input, through the GPU store, gets the oracle's E4M3 code."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    finite = bits[exp != 0xFF]
    n = finite.size // 128 * 128
    x = torch.from_numpy(finite[:n].view(np.int16)).view(torch.bfloat16).reshape(-1, 1, 128)
    N = x.shape[0]
    slots = torch.arange(N, dtype=torch.int32)
    sc = torch.tensor([scale], dtype=torch.float32)
    kp = torch.full((N, 1, 1, 128), W.CANARY_FP8, dtype=torch.uint8, device="cuda")
    vp = torch.full_like(kp, W.CANARY_FP8)
    xd = x.cuda()
    K.store_kvcache(xd, xd, kp, vp, slots.cuda(), sc.cuda(), sc.cuda())
    rk = O.new_pool(N, 1, 1, 128, True, W.CANARY_FP8)
    rv = O.new_pool(N, 1, 1, 128, True, W.CANARY_FP8)
    assert O.store_kvcache(x, x, rk, rv, slots, N, 1, sc, sc) == O.ORC_OK
    got = pool_bytes(kp)
    bad = np.nonzero(got.ravel() != rk.ravel())[0]
    assert bad.size == 0, f"{bad.size} codes differ; first input bits {finite[bad[0]]:#06x}"


def test_slot_minus_one_and_out_of_pool():
    c = small(num_seqs=4)
    wl = to_device(W.generate(c, 2))
    kp, vp = device_pools(wl)
    before = pool_bytes(kp).copy()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots = torch.full_like(wl.slot_new, -1)
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, slots, dev_err=err)
    assert K.read_device_error(err) == K.PKV_OK
    assert np.array_equal(pool_bytes(kp), before), "slot -1 must not write"
    slots[1] = wl.num_blocks * c.block_size  # one past the pool
    K.store_kvcache(wl.k_new, wl.v_new, kp, vp, slots, dev_err=err)
    assert K.read_device_error(err) == K.PKV_ERR_DEVICE_BOUNDS
    assert np.array_equal(pool_bytes(kp), before)


def test_host_checks_launch_nothing():
    c = small(num_seqs=2)
    wl = to_device(W.generate(c, 3))
    kp, vp = device_pools(wl)
    with pytest.raises(K.PagedKVError) as e:
        # FP8 pool without scales
        K.store_kvcache(wl.k_new, wl.v_new, kp.view(torch.uint8)[..., :128].contiguous(),
                        vp.view(torch.uint8)[..., :128].contiguous(), wl.slot_new)
    assert e.value.status == K.PKV_ERR_INVALID_ARG

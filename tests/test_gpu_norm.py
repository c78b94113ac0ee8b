"""Fused residual add + RMSNorm on the GPU against the fp64 oracle.

The updated residual is compared bit for bit: it is bf16(x + r) rounded to
nearest even, and the fp32 sum of two bf16 values rounds to the same bf16 as
the exact sum (it is exact unless the smaller operand lies below 2^-16 of the
larger, far from any bf16 tie). The normalised output is rounded to bf16 from
an fp32 computation, so it must lie within half a bf16 ulp (at most 2^-8 of
its magnitude) of the fp64 value, plus a small allowance for the fp32
arithmetic (1e-5 relative, 1e-6 absolute).
"""

import numpy as np
import pytest
import torch

import oracle as O
from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200 import workloads as W

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2.0 ** -8 + 1e-5, 1e-6


def bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check(wl, inplace=False):
    c = wl.cfg
    x = wl.x.cuda()
    r = wl.residual.cuda() if wl.residual is not None else None
    w = wl.weight.cuda()
    ref, rref, st = O.fused_add_rmsnorm(wl.x, wl.residual, wl.weight, c.eps, num_threads=8)
    assert st == O.ORC_OK
    out = K.fused_add_rmsnorm(x, r, w, c.eps, out=x if inplace else None)
    torch.cuda.synchronize()
    if r is not None:
        assert np.array_equal(bits(r), rref), "residual is not bf16(x + r)"
    g = out.float().cpu().double().numpy()
    assert np.all(np.isfinite(g) | ~np.isfinite(ref))
    err = np.abs(g - ref)
    bound = RTOL * np.abs(ref) + ATOL
    worst = float((err / bound).max())
    assert worst <= 1.0, f"{c.name}: error {worst:.2f} x the bound"
    if inplace:
        assert out.data_ptr() == x.data_ptr()
    return worst


@pytest.mark.parametrize("name", ["norm_tiny", "norm_qwen3_0.6b", "norm_qwen3_8b_decode", "norm_qwen3_8b"])
def test_workloads(name):
    check(W.generate_norm(W.NORM_CONFIGS[name], 1))


@pytest.mark.parametrize("T,H", [(1, 8), (3, 24), (7, 1000), (5, 5120), (2, 16384), (300, 64)])
def test_odd_shapes(T, H):
    check(W.generate_norm(W.NormConfig(f"shape_{T}_{H}", T, H), 2))


def test_without_residual_and_in_place():
    check(W.generate_norm(W.NormConfig("plain", 33, 4096, 1e-5, residual=False), 3))
    check(W.generate_norm(W.NormConfig("inplace", 33, 4096), 4), inplace=True)


def test_extremes():
    """eps 0, a zero row (eps > 0 gives zeros), huge and tiny magnitudes, and
    a residual sum that overflows bf16 (to infinity, like the oracle)."""
    wl = W.generate_norm(W.NormConfig("ext", 6, 256, 1e-6), 5)
    wl.x[0] = 0
    wl.residual[0] = 0
    wl.x[1] *= 1e15  # squares summed in fp32: |h| must stay well below 1e19
    wl.x[2] *= 1e-30
    wl.residual[2] = 0
    check(wl)
    wl0 = W.generate_norm(W.NormConfig("eps0", 4, 512, 0.0), 6)
    check(wl0)
    big = W.generate_norm(W.NormConfig("overflow", 1, 8, 1e-6), 7)
    big.x[0, 0] = 3.0e38
    big.residual[0, 0] = 3.0e38
    x, r = big.x.cuda(), big.residual.cuda()
    K.fused_add_rmsnorm(x, r, big.weight.cuda(), 1e-6)
    _, rref, _ = O.fused_add_rmsnorm(big.x, big.residual, big.weight, 1e-6)
    assert np.array_equal(bits(r), rref) and rref[0, 0] == 0x7F80

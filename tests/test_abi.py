"""The C-ABI library on the host (no GPU): it loads, exports every symbol the
header declares, and refuses bad arguments before launching anything."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def K():
    from paged_kv_cache_482_b200 import build as B

    B.build()
    from paged_kv_cache_482_b200 import pagedkv

    pagedkv.lib()
    return pagedkv


def declared_symbols():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(r"PKV_API\s+[\w\s\*]+?\b(pkv_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(K):
    names = declared_symbols()
    assert {"pkv_store_kvcache", "pkv_paged_attention_decode", "pkv_plan_decode"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", K.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT\s+(pkv_\w+)", out))
    assert names <= exported, f"missing: {names - exported}"
    assert exported <= names, f"exported but not declared: {exported - names}"
    for n in names:
        getattr(K.lib(), n)


def test_version_and_status_strings(K):
    assert K.version() == 0x000100
    for s in range(7):
        assert K.status_string(s) and K.status_string(s) != "unknown status"
    assert K.status_string(99) == "unknown status"


def _decode(L, **kw):
    a = dict(q=0x10000, kc=0x20000, vc=0x30000, bt=0x40000, maxb=8, cl=0x50000, S=4, nq=32, nkv=8, d=128, bs=256,
             nblk=100, scale=0.088, dt=0, ks=None, vs=None, maxctx=2048, part=0, ws=None, wsb=0, out=0x60000,
             err=None, stream=None)
    a.update(kw)
    return L.pkv_paged_attention_decode(a["q"], a["kc"], a["vc"], a["bt"], a["maxb"], a["cl"], None, a["S"], a["nq"],
                                        a["nkv"], a["d"], a["bs"], a["nblk"], a["scale"], a["dt"], a["ks"], a["vs"],
                                        a["maxctx"], a["part"], a["ws"], a["wsb"], a["out"], a["err"], a["stream"])


def test_decode_host_checks(K):
    L = K.lib()
    assert _decode(L, q=None) == K.PKV_ERR_INVALID_ARG
    assert _decode(L, q=0x10008) == K.PKV_ERR_INVALID_ARG  # misaligned
    assert _decode(L, d=96) == K.PKV_ERR_UNSUPPORTED
    assert _decode(L, nq=24, nkv=8) == K.PKV_ERR_UNSUPPORTED  # group 3
    assert _decode(L, nq=30, nkv=8) == K.PKV_ERR_INVALID_ARG
    assert _decode(L, bs=100) == K.PKV_ERR_INVALID_ARG
    assert _decode(L, bs=4) == K.PKV_ERR_INVALID_ARG
    assert _decode(L, maxctx=4096) == K.PKV_ERR_INVALID_ARG  # beyond the table
    assert _decode(L, dt=1) == K.PKV_ERR_INVALID_ARG  # FP8 without scales
    assert _decode(L, scale=float("nan")) == K.PKV_ERR_INVALID_ARG
    assert _decode(L, part=256) == K.PKV_ERR_WORKSPACE  # split needs a workspace
    assert _decode(L, part=256, ws=0x70000, wsb=16) == K.PKV_ERR_WORKSPACE
    assert _decode(L, S=0) == K.PKV_OK  # nothing to do, nothing launched


def test_store_host_checks(K):
    L = K.lib()
    ok = dict(k=0x10000, v=0x20000, kc=0x30000, vc=0x40000, sm=0x50000, N=4, nkv=8, d=128, bs=16, nblk=10, dt=0,
              ks=None, vs=None)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return L.pkv_store_kvcache(a["k"], a["v"], a["kc"], a["vc"], a["sm"], a["N"], a["nkv"], a["d"], a["bs"],
                                   a["nblk"], a["dt"], a["ks"], a["vs"], None, None)

    assert call(k=None) == K.PKV_ERR_INVALID_ARG
    assert call(kc=0x30004) == K.PKV_ERR_INVALID_ARG
    assert call(d=12) == K.PKV_ERR_INVALID_ARG
    assert call(dt=1) == K.PKV_ERR_INVALID_ARG
    assert call(dt=7) == K.PKV_ERR_INVALID_ARG
    assert call(N=0) == K.PKV_OK
    assert call(N=0, k=None, v=None, sm=None, kc=None, vc=None) == K.PKV_OK  # nothing to read or write


@pytest.mark.parametrize("name,split,ws", [
    ("tiny", False, False), ("qwen3_0.6b", False, False), ("qwen3_8b", False, False),
    ("prefix_shared", False, False), ("long_fp8", True, True)])
def test_plans_of_the_workloads(K, name, split, ws):
    from paged_kv_cache_482_b200 import workloads as W

    c = W.CONFIGS[name]
    p = K.plan_decode(c.num_seqs, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size, c.max_context,
                      c.cache_dtype == W.CACHE_FP8)
    if name == "tiny":
        return  # latency-bound; either plan is valid
    assert (p["partition_tokens"] > 0) == split, p
    assert (p["workspace_bytes"] > 0) == ws
    if split:
        assert p["max_partitions"] == -(-c.max_context // p["partition_tokens"])
        rows = c.num_seqs * c.num_q_heads * p["max_partitions"]
        assert p["workspace_bytes"] >= rows * (c.head_dim + 2) * 4


def test_plan_requests(K):
    p = K.plan_decode(4, 32, 8, 128, 16, 32768, True, 1000)
    assert p["partition_tokens"] % 64 == 0 and p["partition_tokens"] >= 1000
    p = K.plan_decode(4, 32, 8, 128, 256, 2048, False, -1)
    assert p["partition_tokens"] == 0 and p["workspace_bytes"] == 0
    # one partition may span any number of blocks (ids beyond the staged ones come from the table)
    p = K.plan_decode(4, 32, 8, 128, 16, 32768, True, -1)
    assert p["partition_tokens"] == 0 and p["workspace_bytes"] == 0
    p = K.plan_decode(4, 32, 8, 128, 16, 32768, True, 20000)
    assert p["partition_tokens"] >= 20000 and p["max_partitions"] == 2


@pytest.mark.parametrize("name", ["tiny", "qwen3_0.6b", "qwen3_8b", "prefix_shared", "long_fp8"])
def test_workspace_bound_covers_every_automatic_plan(K, name):
    """pkv_decode_workspace_bytes(num_seqs, nq, d, max_context_len) is enough
    for the automatic plan of every KV head count, block size and cache type
    those four sizes allow, and is 0 exactly when no such plan can split."""
    from paged_kv_cache_482_b200 import workloads as W

    c = W.CONFIGS[name]
    bound = K.decode_workspace_bytes(c.num_seqs, c.num_q_heads, c.head_dim, c.max_context)
    L = K.lib()
    worst = 0
    for g in (1, 2, 4, 8):
        if c.num_q_heads % g:
            continue
        for bs in (8, 16, 32, 64, 128, 256, 512, 1024):
            for dt in (K.PKV_CACHE_BF16, K.PKV_CACHE_FP8_E4M3, K.PKV_CACHE_FP8_E4M3_TOKEN):
                plan = K._Plan()
                st = L.pkv_plan_decode(c.num_seqs, c.num_q_heads, c.num_q_heads // g, c.head_dim, bs,
                                       c.max_context, dt, 0, ctypes.byref(plan))
                assert st == K.PKV_OK
                assert plan.workspace_bytes <= bound, (g, bs, dt)
                worst = max(worst, plan.workspace_bytes)
    assert (bound == 0) == (c.max_context <= 1024)
    if name == "long_fp8":
        assert worst > 0  # the bound is exercised by a real split


def test_workspace_bound_sweep(K):
    import random

    rng = random.Random(3)
    L = K.lib()
    for _ in range(400):
        S, nq, d, ctx = rng.randint(1, 600), rng.choice([8, 16, 32, 64]), rng.choice([64, 128]), rng.randint(1, 70000)
        bound = K.decode_workspace_bytes(S, nq, d, ctx)
        g = rng.choice([1, 2, 4, 8])
        bs = rng.choice([8, 16, 256, 1024])
        plan = K._Plan()
        st = L.pkv_plan_decode(S, nq, nq // g, d, bs, ctx, rng.choice([0, 1, 2]), 0, ctypes.byref(plan))
        if st == K.PKV_OK:
            assert plan.workspace_bytes <= bound, (S, nq, d, ctx, g, bs)
    assert K.decode_workspace_bytes(0, 32, 128, 4096) == 0
    assert K.decode_workspace_bytes(4, 32, 128, 1024) == 0
    assert K.decode_workspace_bytes(4, 32, 128, 1025) > 0


def test_binding_refuses_to_run_without_library(tmp_path):
    from paged_kv_cache_482_b200 import pagedkv

    with pytest.raises(RuntimeError):
        pagedkv._lib_saved = pagedkv._lib
        try:
            pagedkv._lib = None
            pagedkv.lib(str(tmp_path / "missing.so"))
        finally:
            pagedkv._lib = pagedkv._lib_saved


def test_prefill_host_checks(K):
    L = K.lib()
    ok = dict(q=0x10000, kc=0x20000, vc=0x30000, bt=0x40000, maxb=8, cu=0x50000, cl=0x60000, S=4, T=100, nq=32,
              nkv=8, d=128, bs=256, nblk=100, scale=0.088, dt=0, ks=None, vs=None, mq=64, ws=None, wsb=0,
              out=0x70000)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return L.pkv_paged_attention_prefill(a["q"], a["kc"], a["vc"], a["bt"], a["maxb"], a["cu"], a["cl"], a["S"],
                                             a["T"], a["nq"], a["nkv"], a["d"], a["bs"], a["nblk"], a["scale"],
                                             a["dt"], a["ks"], a["vs"], a["mq"], a["ws"], a["wsb"], a["out"], None,
                                             None)

    assert call(q=None) == K.PKV_ERR_INVALID_ARG
    assert call(cu=None) == K.PKV_ERR_INVALID_ARG
    assert call(out=0x70008) == K.PKV_ERR_INVALID_ARG  # misaligned
    assert call(d=96) == K.PKV_ERR_UNSUPPORTED
    assert call(nq=24) == K.PKV_ERR_UNSUPPORTED  # group 3
    assert call(nq=30) == K.PKV_ERR_INVALID_ARG
    assert call(bs=100) == K.PKV_ERR_INVALID_ARG
    assert call(dt=1) == K.PKV_ERR_INVALID_ARG  # FP8 without scales
    assert call(dt=5) == K.PKV_ERR_INVALID_ARG
    assert call(scale=float("nan")) == K.PKV_ERR_INVALID_ARG
    assert call(scale=-0.1) == K.PKV_ERR_INVALID_ARG and call(scale=0.0) == K.PKV_ERR_INVALID_ARG
    assert call(mq=0) == K.PKV_ERR_INVALID_ARG
    assert call(nblk=2**31) == K.PKV_ERR_INVALID_ARG
    assert call(S=0) == K.PKV_OK and call(T=0) == K.PKV_OK  # nothing to do, nothing launched
    # the E4M3 widening workspace: checked before anything is launched
    fp8 = dict(dt=1, ks=0x80000, vs=0x90000)
    assert call(ws=0xA0000, wsb=4096, **fp8) == K.PKV_ERR_WORKSPACE
    assert call(ws=0xA0000, wsb=4096, dt=2, ks=0x80000, vs=0x90000) == K.PKV_ERR_WORKSPACE
    assert call(ws=0xA0008, wsb=1 << 40, **fp8) == K.PKV_ERR_INVALID_ARG  # misaligned
    assert call(ws=0xA0000, wsb=0, S=0, **fp8) == K.PKV_OK  # no sequences: no bound


def test_prefill_workspace_bytes(K):
    L = K.lib()
    wb = K.prefill_workspace_bytes
    # rows per (sequence, KV head): the table capacity rounded up to 128
    assert wb(4, 8, 128, 8, 256, K.PKV_CACHE_FP8_E4M3) == 4 * 8 * 2048 * (4 * 128)
    assert wb(4, 8, 128, 8, 256, K.PKV_CACHE_FP8_E4M3_TOKEN) == 4 * 8 * 2048 * (4 * 128 + 4)
    assert wb(3, 2, 64, 3, 16, K.PKV_CACHE_FP8_E4M3) == 3 * 2 * 128 * (4 * 64)
    assert wb(1, 1, 128, 9, 16, K.PKV_CACHE_FP8_E4M3) == 256 * 512  # 144 -> 256 rows
    assert wb(4, 8, 128, 8, 256, K.PKV_CACHE_BF16) == 0
    assert wb(0, 8, 128, 8, 256, K.PKV_CACHE_FP8_E4M3) == 0 and wb(4, 8, 128, 0, 256, 1) == 0
    assert wb(4, 8, 128, 8, 256, 7) == 0  # unknown cache type
    # 2^20 sequences x 8 heads x 16384 rows: beyond int32 tensor-map rows
    assert wb(1 << 20, 8, 128, 1024, 16, K.PKV_CACHE_FP8_E4M3) == 0
    assert L.pkv_prefill_workspace_bytes(2, 2, 128, 1, 128, 1) == 2 * 2 * 128 * 512


def test_norm_host_checks(K):
    L = K.lib()
    ok = dict(x=0x10000, r=0x20000, w=0x30000, out=0x40000, T=4, H=4096, eps=1e-6)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return L.pkv_fused_add_rmsnorm(a["x"], a["r"], a["w"], a["out"], a["T"], a["H"], a["eps"], None)

    assert call(x=None) == K.PKV_ERR_INVALID_ARG
    assert call(w=None) == K.PKV_ERR_INVALID_ARG
    assert call(r=0x20008) == K.PKV_ERR_INVALID_ARG  # misaligned
    assert call(H=12) == K.PKV_ERR_INVALID_ARG  # not a multiple of 8
    assert call(H=0) == K.PKV_ERR_INVALID_ARG
    assert call(H=16384 + 8) == K.PKV_ERR_UNSUPPORTED
    assert call(eps=-1.0) == K.PKV_ERR_INVALID_ARG
    assert call(eps=float("nan")) == K.PKV_ERR_INVALID_ARG
    assert call(eps=float("inf")) == K.PKV_ERR_INVALID_ARG
    assert call(T=-1) == K.PKV_ERR_INVALID_ARG
    assert call(T=0) == K.PKV_OK  # nothing launched


def test_rope_store_host_checks(K):
    L = K.lib()
    ok = dict(q=0x10000, qo=0x11000, k=0x20000, v=0x30000, kc=0x40000, vc=0x50000, sm=0x60000, pos=0x70000,
              cs=0x80000, mp=4096, style=0, N=4, nq=32, nkv=8, d=128, bs=16, nblk=10, dt=0, ks=None, vs=None)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return L.pkv_store_kvcache_rope(a["q"], a["qo"], a["k"], a["v"], a["kc"], a["vc"], a["sm"], a["pos"],
                                        a["cs"], a["mp"], a["style"], a["N"], a["nq"], a["nkv"], a["d"], a["bs"],
                                        a["nblk"], a["dt"], a["ks"], a["vs"], None, None)

    assert call(d=24) == K.PKV_ERR_INVALID_ARG          # not a multiple of 16
    assert call(d=48) == K.PKV_ERR_UNSUPPORTED          # 3 lanes per row
    assert call(style=2) == K.PKV_ERR_INVALID_ARG
    assert call(qo=None) == K.PKV_ERR_INVALID_ARG        # q without q_out
    assert call(mp=0) == K.PKV_ERR_INVALID_ARG
    assert call(cs=0x80008) == K.PKV_ERR_INVALID_ARG     # table not 16-byte aligned
    assert call(dt=1) == K.PKV_ERR_INVALID_ARG           # E4M3 without scales
    assert call(pos=None) == K.PKV_ERR_INVALID_ARG
    assert call(N=0) == K.PKV_OK
    assert call(N=0, q=None, qo=None, k=None, v=None, pos=None, cs=None, sm=None) == K.PKV_OK


def test_shared_prefix_plan_and_host_checks(K):
    L = K.lib()
    for dt in (K.PKV_CACHE_BF16, K.PKV_CACHE_FP8_E4M3, K.PKV_CACHE_FP8_E4M3_TOKEN):
        for part in (0, 256, -1):
            plain = K.plan_decode(512, 32, 8, 128, 256, 1536, dt != K.PKV_CACHE_BF16, part)
            shared = K.plan_decode_shared_prefix(512, 32, 8, 128, 256, 1536, dt, part)
            np_suffix = plain["max_partitions"] if plain["partition_tokens"] else 1
            assert shared["max_partitions"] == np_suffix + 1  # slot 0 holds the shared prefix
            assert shared["workspace_bytes"] >= 512 * 32 * shared["max_partitions"] * 130 * 4
            assert shared["partition_tokens"] == (plain["partition_tokens"] or 1536)
    # head_dim 64 has no prefix kernel: the plan is the ordinary one
    assert K.plan_decode_shared_prefix(8, 8, 2, 64, 16, 900) == K.plan_decode(8, 8, 2, 64, 16, 900)

    def call(**kw):
        a = dict(q=0x10000, kc=0x20000, vc=0x30000, bt=0x40000, maxb=8, cl=0x50000, S=4, nq=32, nkv=8, d=128,
                 bs=256, nblk=100, scale=0.088, dt=0, ks=None, vs=None, maxctx=2048, cu=0x60000, pre=0x61000,
                 ng=2, mg=3, part=0, ws=None, wsb=0, out=0x70000)
        a.update(kw)
        return L.pkv_paged_attention_decode_shared_prefix(
            a["q"], a["kc"], a["vc"], a["bt"], a["maxb"], a["cl"], None, a["S"], a["nq"], a["nkv"], a["d"], a["bs"],
            a["nblk"], a["scale"], a["dt"], a["ks"], a["vs"], a["maxctx"], a["cu"], a["pre"], a["ng"], a["mg"],
            a["part"], a["ws"], a["wsb"], a["out"], None, None)

    assert call(ng=-1) == K.PKV_ERR_INVALID_ARG
    assert call(cu=None) == K.PKV_ERR_INVALID_ARG
    assert call(mg=0) == K.PKV_ERR_INVALID_ARG
    assert call(ws=None) == K.PKV_ERR_WORKSPACE           # the prefix slot always needs scratch
    assert call(ws=0x90000, wsb=64) == K.PKV_ERR_WORKSPACE
    assert call(ws=0x90010, wsb=1 << 30) == K.PKV_ERR_INVALID_ARG  # not 256-byte aligned
    assert call(q=0x10008, ws=0x90000, wsb=1 << 30) == K.PKV_ERR_INVALID_ARG
    assert call(S=0, ws=0x90000, wsb=1 << 30) == K.PKV_OK


def test_longest_first_is_a_stable_descending_order(K):
    """The host order helper: lengths non-increasing along the order, equal
    lengths in their original order, every sequence exactly once."""
    g = torch.Generator().manual_seed(3)
    for n in (1, 7, 512, 1025):
        lens = torch.randint(0, 40, (n,), generator=g, dtype=torch.int32)  # many ties
        order = K.longest_first(lens)
        assert order.dtype == torch.int32 and sorted(order.tolist()) == list(range(n))
        sl = lens[order.long()]
        assert bool((sl[:-1] >= sl[1:]).all())
        for a, b in zip(order[:-1].tolist(), order[1:].tolist()):
            if lens[a] == lens[b]:
                assert a < b

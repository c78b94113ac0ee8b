"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each ``pin_*`` function takes a loaded oracle library and raises
AssertionError when the oracle disagrees with:

* brute-force attention over the sequence's tokens laid out contiguously,
  taken straight from the drawn rows (no pool, no block table) and evaluated
  with scipy's softmax and numpy einsum (a library special case);
* the invariants the pages' block-table definition implies: any relabelling
  of physical blocks, or a shared prefix copied into private blocks, changes
  nothing ("DeepSeek复刻vLLM反超原版", section "vLLM：大模型推理的加速引擎与挑战":
  logical blocks map to physical blocks through a block table, and KV blocks
  can be shared within and across requests);
* closed forms: one token returns its V row; identical keys return the mean
  of V; a dominating key returns its own V row (pins token order and the
  block / offset split at every block boundary);
* the OCP E4M3 format points (tests/golden/e4m3_ocp_points.txt) and torch's
  own float8_e4m3fn cast (a library routine) for the FP8 codec.

The same functions run against deliberately broken copies of the oracle
(tests/test_oracle_mutants.py) to show that each plausible mistake trips at
least one of them.
"""

from __future__ import annotations

import copy
import os

import numpy as np
import scipy.special
import torch

import oracle as O
from paged_kv_cache_482_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-12


def cfg(**kw) -> W.DecodeConfig:
    base = dict(name="pin", num_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=16, block_size=4, ctx_lo=1,
                ctx_hi=23)
    base.update(kw)
    return W.DecodeConfig(**base)


def dequant(x_bf16: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """bf16 rows [t, nkv, d] -> fp64 values of their E4M3 codes times scale (torch's cast)."""
    y = x_bf16.float() / scale.float()[None, :, None]
    codes = y.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return codes.double() * scale.double()[None, :, None]


def token_scale(x_bf16: torch.Tensor) -> torch.Tensor:
    """The per-(token, head) scale of rows [t, nkv, d]: the row's largest
    magnitude / 448 in binary32, at least the smallest normal binary32."""
    s = x_bf16.float().abs().amax(dim=-1) / 448.0
    return torch.clamp(s, min=torch.finfo(torch.float32).tiny)


def token_codes(x_bf16: torch.Tensor) -> torch.Tensor:
    """E4M3 codes of rows [t, nkv, d] under their own per-token scales (torch's cast)."""
    y = x_bf16.float() / token_scale(x_bf16)[..., None]
    return y.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)


def dequant_token(x_bf16: torch.Tensor) -> torch.Tensor:
    return token_codes(x_bf16).double() * token_scale(x_bf16).double()[..., None]


def dequant_kv(wl, K, V):
    """The values a cache holds for logical rows K, V of workload wl."""
    if getattr(wl, "token_scales", False):
        return dequant_token(K), dequant_token(V)
    if wl.is_fp8:
        return dequant(K, wl.k_scale), dequant(V, wl.v_scale)
    return K, V


def brute_force(wl: W.Workload, i: int) -> np.ndarray:
    """Contiguous softmax attention for sequence i from its logical K/V rows."""
    c = wl.cfg
    K, V = W.logical_kv(wl, i)
    K, V = dequant_kv(wl, K, V)
    K = np.repeat(K.double().numpy(), c.group, axis=1)  # [ctx, nq, d]
    V = np.repeat(V.double().numpy(), c.group, axis=1)
    q = wl.q[i].double().numpy()  # [nq, d]
    scale = np.float64(np.float32(c.softmax_scale))
    s = np.einsum("hd,thd->ht", q, K) * scale
    p = scipy.special.softmax(s, axis=1)
    return np.einsum("ht,thd->hd", p, V)


def _assert_close(a, b, tol=TOL, what=""):
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert np.all(np.isfinite(a)), f"{what}: non-finite oracle output"
    assert err <= tol, f"{what}: max abs diff {err:.3e} > {tol:.1e}"


def _run(wl, lib):
    out, kp, vp, st = O.run_workload(wl, lib=lib)[:4]
    assert st == O.ORC_OK, f"oracle status {st}"
    return out, kp, vp


# ----------------------------------------------------------------- attention


def pin_bruteforce_bf16(lib):
    for c, seed in [
        (cfg(), 1),
        (cfg(num_seqs=2, num_q_heads=8, num_kv_heads=1, head_dim=8, block_size=8, ctx_lo=1, ctx_hi=40), 2),
        (cfg(num_seqs=2, num_q_heads=3, num_kv_heads=3, head_dim=12, block_size=16, ctx_lo=15, ctx_hi=33), 3),
        (cfg(num_seqs=3, block_size=4, prefix_tokens=8, ctx_lo=0, ctx_hi=6), 4),
    ]:
        wl = W.generate(c, seed)
        out, _, _ = _run(wl, lib)
        for i in range(c.num_seqs):
            _assert_close(out[i], brute_force(wl, i), what=f"bf16 seq {i} {c}")


def pin_bruteforce_fp8(lib):
    for c, seed in [
        (cfg(cache_dtype=W.CACHE_FP8), 5),
        (cfg(cache_dtype=W.CACHE_FP8, num_q_heads=8, num_kv_heads=2, head_dim=8, ctx_lo=30, ctx_hi=50), 6),
    ]:
        wl = W.generate(c, seed)
        out, _, _ = _run(wl, lib)
        for i in range(c.num_seqs):
            _assert_close(out[i], brute_force(wl, i), what=f"fp8 seq {i}")


def _relabel(wl: W.Workload, perm: torch.Tensor) -> W.Workload:
    """The same step with physical block b renamed perm[b] everywhere."""
    bs = wl.cfg.block_size
    w2 = copy.copy(wl)
    bt = wl.block_tables.long()
    w2.block_tables = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32)

    def slots(s):
        s = s.long()
        return torch.where(s >= 0, perm[(s // bs).clamp(min=0)] * bs + s % bs, s).to(torch.int32)

    w2.slot_hist = slots(wl.slot_hist)
    w2.slot_new = slots(wl.slot_new)
    return w2


def pin_permutation_invariance(lib):
    for c in (cfg(ctx_lo=5, ctx_hi=30), cfg(cache_dtype=W.CACHE_FP8), cfg(prefix_tokens=8, ctx_lo=0, ctx_hi=9)):
        wl = W.generate(c, 7)
        out, _, _ = _run(wl, lib)
        g = torch.Generator().manual_seed(11)
        for _ in range(2):
            perm = torch.randperm(wl.num_blocks, generator=g)
            out2, _, _ = _run(_relabel(wl, perm), lib)
            assert np.array_equal(out, out2), "block relabelling changed the result"


def pin_prefix_shared_equals_duplicated(lib):
    c = cfg(num_seqs=4, prefix_tokens=8, ctx_lo=0, ctx_hi=7)
    wl = W.generate(c, 8)
    out, _, _ = _run(wl, lib)
    bs, P = c.block_size, c.prefix_tokens
    nshared = P // bs
    S = c.num_seqs
    w2 = copy.copy(wl)
    w2.num_blocks = wl.num_blocks + S * nshared
    bt = wl.block_tables.clone()
    k_rows, v_rows, s_rows = [wl.k_hist], [wl.v_hist], [wl.slot_hist]
    for i in range(S):
        first = wl.num_blocks + i * nshared
        bt[i, :nshared] = torch.arange(first, first + nshared, dtype=torch.int32)
        k_rows.append(wl.k_hist[:P])
        v_rows.append(wl.v_hist[:P])
        s_rows.append(torch.arange(first * bs, first * bs + P, dtype=torch.int32))
    w2.block_tables = bt
    w2.k_hist = torch.cat(k_rows)
    w2.v_hist = torch.cat(v_rows)
    w2.slot_hist = torch.cat(s_rows)
    out2, _, _ = _run(w2, lib)
    assert np.array_equal(out, out2), "shared prefix differs from private copies"


def pin_single_token_returns_v(lib):
    for fp8 in (False, True):
        c = cfg(num_q_heads=6, num_kv_heads=3, ctx_lo=1, ctx_hi=1,
                cache_dtype=W.CACHE_FP8 if fp8 else W.CACHE_BF16)
        wl = W.generate(c, 9)
        out, _, _ = _run(wl, lib)
        for i in range(c.num_seqs):
            _, V = W.logical_kv(wl, i)
            Vd = dequant(V, wl.v_scale) if fp8 else V.double()
            expect = np.repeat(Vd[0].numpy(), c.group, axis=0)  # [nq, d]
            assert np.array_equal(out[i], expect), "context of one token must return its V row exactly"


def pin_identical_keys_mean_of_v(lib):
    c = cfg(ctx_lo=3, ctx_hi=29)
    wl = W.generate(c, 10)
    wl.k_hist[:] = wl.k_hist[0:1].clone()
    wl.k_new[:] = wl.k_hist[0:1]
    out, _, _ = _run(wl, lib)
    for i in range(c.num_seqs):
        _, V = W.logical_kv(wl, i)
        mean = np.repeat(V.double().numpy().mean(axis=0), c.group, axis=0)
        _assert_close(out[i], mean, what="identical keys")


def _logical_slot_row(wl, i, p):
    """(tensor, row) holding logical token p of sequence i in the drawn rows."""
    ctx = int(wl.context_lens[i])
    if p == ctx - 1 and int(wl.slot_new[i]) >= 0:
        return "new", i
    return "hist", int(wl.hist_rows[i][p])


def pin_dominant_key_returns_its_v(lib):
    c = cfg(num_seqs=2, num_q_heads=2, num_kv_heads=1, head_dim=16, block_size=4, ctx_lo=13, ctx_hi=13)
    for p in (0, 3, 4, 5, 8, 11, 12):
        wl = W.generate(c, 12)
        wl.q[:] = 1.0
        wl.k_hist.zero_()
        wl.k_new.zero_()
        for i in range(c.num_seqs):
            src, row = _logical_slot_row(wl, i, p)
            (wl.k_new if src == "new" else wl.k_hist)[row] = 32.0  # score 128 against 0 elsewhere
        out, _, _ = _run(wl, lib)
        for i in range(c.num_seqs):
            _, V = W.logical_kv(wl, i)
            expect = np.repeat(V[p].double().numpy(), c.group, axis=0)
            _assert_close(out[i], expect, what=f"dominant key at {p}")


def pin_bruteforce_fp8_token_scales(lib):
    for c, seed in [
        (cfg(cache_dtype=W.CACHE_FP8_TOKEN), 15),
        (cfg(cache_dtype=W.CACHE_FP8_TOKEN, num_q_heads=8, num_kv_heads=2, head_dim=8, ctx_lo=30, ctx_hi=50), 16),
        (cfg(cache_dtype=W.CACHE_FP8_TOKEN, prefix_tokens=8, ctx_lo=0, ctx_hi=9), 17),
    ]:
        wl = W.generate(c, seed)
        out, _, _ = _run(wl, lib)
        for i in range(c.num_seqs):
            _assert_close(out[i], brute_force(wl, i), what=f"fp8 per-token seq {i}")


def pin_token_scale_store(lib):
    """Codes and per-token scales at every stored slot equal torch's: the row
    amax / 448 in binary32 (floored at the smallest normal) and the E4M3 cast
    of x / s; an all-zero row gets the floor scale and zero codes; a row
    spanning the full range keeps its largest element at code 448."""
    c = cfg(cache_dtype=W.CACHE_FP8_TOKEN, num_seqs=2, ctx_lo=9, ctx_hi=14)
    wl = W.generate(c, 18)
    wl.k_hist[0] = 0.0  # an all-zero row (every head)
    wl.v_hist[1, 0, :] = torch.linspace(-3.0, 1.0, c.head_dim).to(torch.bfloat16)
    out, kp, vp, st, ks, vs = O.run_workload(wl, lib=lib)
    assert st == O.ORC_OK and np.all(np.isfinite(out))
    bs = c.block_size
    slots = wl.slot_hist.long()
    blk, off = slots // bs, slots % bs
    for pool, sp, rows in ((kp, ks, wl.k_hist), (vp, vs, wl.v_hist)):
        got_codes = pool[blk.numpy(), :, off.numpy(), :]  # [H, nkv, d]
        want_codes = token_codes(rows).view(torch.uint8).numpy()
        assert np.array_equal(got_codes, want_codes), "per-token E4M3 codes"
        got_s = sp[blk.numpy(), :, off.numpy()]
        assert np.array_equal(got_s, token_scale(rows).numpy()), "per-token scales"
    assert np.all(ks[blk[0], :, off[0]] == np.float32(torch.finfo(torch.float32).tiny))
    assert np.all(kp[blk[0], :, off[0]] == 0)
    assert vp[blk[1], 0, off[1], 0] == 0xFE  # -448: the row's largest magnitude


# --------------------------------------------------------------------- store


def pin_store_layout(lib):
    nblk, nkv, bs, d = 3, 2, 4, 4
    g = torch.Generator().manual_seed(13)
    k = torch.randn(6, nkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(6, nkv, d, generator=g).to(torch.bfloat16)
    slots = torch.tensor([0, 5, -1, 11, 6, 2], dtype=torch.int32)
    kp = O.new_pool(nblk, nkv, bs, d, False, W.CANARY_BF16)
    vp = O.new_pool(nblk, nkv, bs, d, False, W.CANARY_BF16)
    assert O.store_kvcache(k, v, kp, vp, slots, nblk, bs, lib=lib) == O.ORC_OK
    ek = np.full((nblk, nkv, bs, d), W.CANARY_BF16, np.uint16)
    ev = ek.copy()
    kb = k.view(torch.int16).numpy().view(np.uint16)
    vb = v.view(torch.int16).numpy().view(np.uint16)
    for t, s in enumerate(slots.tolist()):
        if s >= 0:
            blk, off = divmod(s, bs)
            ek[blk, :, off, :] = kb[t]
            ev[blk, :, off, :] = vb[t]
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev), "bf16 store layout"
    # A slot beyond the pool is refused and writes nothing.
    kp2, vp2 = kp.copy(), vp.copy()
    st = O.store_kvcache(k[:1], v[:1], kp2, vp2, torch.tensor([nblk * bs], dtype=torch.int32), nblk, bs, lib=lib)
    assert st == O.ORC_ERR_BOUNDS and np.array_equal(kp2, kp) and np.array_equal(vp2, vp)
    # FP8: the code in each slot is torch's E4M3 cast of x / scale (fp32 division).
    ks = torch.tensor([0.01, 0.003], dtype=torch.float32)
    vs = torch.tensor([0.02, 0.5], dtype=torch.float32)
    kq = O.new_pool(nblk, nkv, bs, d, True, W.CANARY_FP8)
    vq = O.new_pool(nblk, nkv, bs, d, True, W.CANARY_FP8)
    assert O.store_kvcache(k, v, kq, vq, slots, nblk, bs, ks, vs, lib=lib) == O.ORC_OK
    ck = (k.float() / ks[None, :, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    cv = (v.float() / vs[None, :, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ek = np.full((nblk, nkv, bs, d), W.CANARY_FP8, np.uint8)
    ev = ek.copy()
    for t, s in enumerate(slots.tolist()):
        if s >= 0:
            blk, off = divmod(s, bs)
            ek[blk, :, off, :] = ck[t]
            ev[blk, :, off, :] = cv[t]
    assert np.array_equal(kq, ek) and np.array_equal(vq, ev), "fp8 store layout / codes"


# ---------------------------------------------------------------- FP8 codec


def read_golden_points():
    pts = []
    with open(os.path.join(GOLDEN, "e4m3_ocp_points.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                code, val = line.split()[:2]
                pts.append((int(code, 16), float(val)))
    return pts


def pin_e4m3_decode_table(lib):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        got = O.e4m3_to_double(c, lib=lib)
        want = lib_vals[c]
        if np.isnan(want):
            assert np.isnan(got), f"code {c:#x} must be NaN"
        else:
            assert got == want and np.signbit(got) == np.signbit(want), f"code {c:#x}: {got} != {want}"
    for c, val in read_golden_points():
        got = O.e4m3_to_double(c, lib=lib)
        if np.isnan(val):
            assert np.isnan(got)
        else:
            assert got == val and np.signbit(got) == np.signbit(val), f"OCP point {c:#x}"
        if not np.isnan(val):
            assert O.e4m3_from_float(val, lib=lib) == c, f"OCP point {c:#x} must encode back to itself"


def _torch_encode(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(x.astype(np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_e4m3_encode(lib):
    # a dense grid through the whole range, past saturation, both signs
    grid = np.arange(-470 * 1024, 470 * 1024 + 1, dtype=np.float64) / 1024.0
    # every exact midpoint between neighbouring codes (ties go to the even code)
    vals = torch.arange(0, 0x7F, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (vals[:-1] + vals[1:]) / 2.0
    # the subnormal range in fine steps, and a spread of magnitudes
    fine = np.arange(0, 4097, dtype=np.float64) * 2.0**-18
    spread = np.float32(np.exp(np.linspace(-30, 8, 3001)))
    x = np.concatenate([grid, mids, -mids, fine, -fine, spread, -spread]).astype(np.float32)
    want = _torch_encode(x)
    got = np.fromiter((O.e4m3_from_float(float(v), lib=lib) for v in x), dtype=np.uint8, count=x.size)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} encodings differ, first x={x[bad[0]]!r}: {got[bad[0]]:#x} vs {want[bad[0]]:#x}"
    # ties: the even neighbour, checked directly
    for j, m in enumerate(mids):
        assert O.e4m3_from_float(float(m), lib=lib) == (j if j % 2 == 0 else j + 1), f"tie at {m}"
    assert O.e4m3_from_float(1e9, lib=lib) == 0x7E and O.e4m3_from_float(-1e9, lib=lib) == 0xFE
    assert O.e4m3_from_float(float("nan"), lib=lib) & 0x7F == 0x7F


def pin_bf16_widening(lib):
    bits = np.arange(0, 65536, 97, dtype=np.uint16)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    for b, w in zip(bits, want):
        got = O.bf16_to_double(int(b), lib=lib)
        assert (np.isnan(got) and np.isnan(w)) or got == w, f"bf16 {b:#x}"


# ------------------------------------------------------------------ errors


def pin_bounds_errors(lib):
    c = cfg(ctx_lo=5, ctx_hi=20)
    wl = W.generate(c, 14)
    out, kp, vp = _run(wl, lib)
    bt = wl.block_tables.clone()
    bt[1, 0] = wl.num_blocks  # outside the pool
    out2, st = O.paged_attention_decode(wl.q, kp, vp, bt, wl.context_lens, c.num_kv_heads, c.block_size,
                                        c.softmax_scale, lib=lib)
    assert st == O.ORC_ERR_BOUNDS
    assert np.all(out2[1] == 0) and np.array_equal(out2[0], out[0]) and np.array_equal(out2[2], out[2])
    # a middle row, so that a length check that lets one extra token through
    # reads the next row's (valid) entry instead of memory past the table
    # Row 1 gets a full row of valid ids, so only the length check can refuse
    # a length one past the table.
    full = wl.block_tables.clone()
    full[1, :] = full[1, 0]
    for bad_len in (0, c.max_blocks_per_seq * c.block_size + 1):
        cl = wl.context_lens.clone()
        cl[1] = bad_len
        out3, st = O.paged_attention_decode(wl.q, kp, vp, full, cl, c.num_kv_heads, c.block_size,
                                            c.softmax_scale, lib=lib)
        assert st == O.ORC_ERR_BOUNDS and np.all(out3[1] == 0)
        assert np.array_equal(out3[0], out[0]) and np.array_equal(out3[2], out[2])


# ------------------------------------------------------------------ prefill


def pcfg(**kw) -> W.PrefillConfig:
    base = dict(name="ppin", num_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=16, block_size=4, hist_lo=0,
                hist_hi=13, chunk_lo=1, chunk_hi=9)
    base.update(kw)
    return W.PrefillConfig(**base)


def _run_prefill(wl, lib):
    out, kp, vp, st = O.run_prefill_workload(wl, lib=lib)[:4]
    assert st == O.ORC_OK, f"oracle status {st}"
    return out, kp, vp


def prefill_brute_force(wl: W.PrefillWorkload, i: int) -> np.ndarray:
    """Causal softmax attention of sequence i's chunk from its logical K/V rows
    (no pool): query token j of a chunk of c sits at position ctx - c + j."""
    c = wl.cfg
    K, V = W.prefill_logical_kv(wl, i)
    K, V = dequant_kv(wl, K, V)
    K = np.repeat(K.double().numpy(), c.group, axis=1)  # [ctx, nq, d]
    V = np.repeat(V.double().numpy(), c.group, axis=1)
    a, b = int(wl.cu_q_lens[i]), int(wl.cu_q_lens[i + 1])
    q = wl.q[a:b].double().numpy()  # [c, nq, d]
    ctx, n = K.shape[0], b - a
    scale = np.float64(np.float32(c.softmax_scale))
    s = np.einsum("jhd,thd->hjt", q, K) * scale
    pos = ctx - n + np.arange(n)
    s = np.where(np.arange(ctx)[None, None, :] <= pos[None, :, None], s, -np.inf)
    p = scipy.special.softmax(s, axis=2)
    return np.einsum("hjt,thd->jhd", p, V)


def pin_prefill_bruteforce(lib):
    for c, seed in [
        (pcfg(), 21),
        (pcfg(num_q_heads=8, num_kv_heads=1, head_dim=8, block_size=8, hist_hi=30, chunk_lo=5, chunk_hi=20), 22),
        (pcfg(num_q_heads=3, num_kv_heads=3, head_dim=12, block_size=16, hist_lo=15, hist_hi=33), 23),
        (pcfg(cache_dtype=W.CACHE_FP8, chunk_hi=12), 24),
        (pcfg(cache_dtype=W.CACHE_FP8_TOKEN, chunk_hi=12, hist_hi=30), 31),
        (pcfg(num_seqs=2, decode_seqs=3, decode_hist_lo=1, decode_hist_hi=20), 25),
    ]:
        wl = W.generate_prefill(c, seed)
        out, _, _ = _run_prefill(wl, lib)
        for i in range(c.total_seqs):
            a, b = int(wl.cu_q_lens[i]), int(wl.cu_q_lens[i + 1])
            _assert_close(out[a:b], prefill_brute_force(wl, i), what=f"prefill seq {i} {c}")


def pin_prefill_one_token_is_decode(lib):
    """A chunk of one token is a decode step: the decode oracle's result (the
    decode function is pinned on its own above)."""
    c = pcfg(num_seqs=0, decode_seqs=5, decode_hist_lo=0, decode_hist_hi=21)
    for fp8 in (False, True):
        wl = W.generate_prefill(c.with_(cache_dtype=W.CACHE_FP8 if fp8 else W.CACHE_BF16), 26)
        out, kp, vp = _run_prefill(wl, lib)
        dec, st = O.paged_attention_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens, c.num_kv_heads,
                                           c.block_size, c.softmax_scale, wl.k_scale, wl.v_scale, lib=lib)
        assert st == O.ORC_OK
        assert np.array_equal(out, dec), "a one-token chunk differs from decode"


def pin_prefill_chunking_invariance(lib):
    """A prompt prefilled as one chunk or as two consecutive chunks gives every
    token the same output (each token's result depends on its prefix only)."""
    c = pcfg(num_seqs=3, hist_lo=0, hist_hi=9, chunk_lo=6, chunk_hi=14)
    wl = W.generate_prefill(c, 27)
    out, kp, vp = _run_prefill(wl, lib)
    cu, cl = wl.cu_q_lens.long(), wl.context_lens.long()
    n = cu[1:] - cu[:-1]
    first = n // 2  # first chunk: the leading half of each sequence's chunk
    rows1 = torch.cat([torch.arange(int(cu[i]), int(cu[i] + first[i])) for i in range(c.total_seqs)])
    rows2 = torch.cat([torch.arange(int(cu[i] + first[i]), int(cu[i + 1])) for i in range(c.total_seqs)])
    cu1 = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(first, 0)]).to(torch.int32)
    cu2 = torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(n - first, 0)]).to(torch.int32)
    o1, st1 = O.paged_attention_prefill(wl.q[rows1], kp, vp, wl.block_tables, cu1, (cl - (n - first)).to(torch.int32),
                                        c.num_kv_heads, c.block_size, c.softmax_scale, lib=lib)
    o2, st2 = O.paged_attention_prefill(wl.q[rows2], kp, vp, wl.block_tables, cu2, wl.context_lens,
                                        c.num_kv_heads, c.block_size, c.softmax_scale, lib=lib)
    assert st1 == O.ORC_OK and st2 == O.ORC_OK
    assert np.array_equal(out[rows1.numpy()], o1) and np.array_equal(out[rows2.numpy()], o2), "chunking changed a result"


def pin_prefill_causal_mask(lib):
    """A key that dominates every score takes over exactly the queries at or
    after its position and leaves the earlier ones unchanged."""
    c = pcfg(num_seqs=2, num_q_heads=2, num_kv_heads=1, head_dim=16, block_size=4, hist_lo=3, hist_hi=3,
             chunk_lo=9, chunk_hi=9)
    for p in (3, 4, 7, 8, 11):  # positions inside the chunk (positions 3 .. 11)
        wl = W.generate_prefill(c, 28)
        wl.q[:] = 1.0
        base, _, _ = _run_prefill(wl, lib)
        for i in range(c.total_seqs):
            a = int(wl.cu_q_lens[i])
            wl.k_new[a + p - 3] = 32.0  # chunk row of position p
        out, _, _ = _run_prefill(wl, lib)
        for i in range(c.total_seqs):
            a = int(wl.cu_q_lens[i])
            _, V = W.prefill_logical_kv(wl, i)
            for j in range(9):
                pos = 3 + j
                if pos < p:
                    assert np.array_equal(out[a + j], base[a + j]), f"query {pos} saw the key at {p}"
                else:
                    expect = np.repeat(V[p].double().numpy()[None], c.group, axis=0)[:, 0]
                    _assert_close(out[a + j], expect, what=f"query {pos}, dominant key {p}")


def pin_prefill_relabel_invariance(lib):
    c = pcfg(hist_hi=20)
    wl = W.generate_prefill(c, 29)
    out, _, _ = _run_prefill(wl, lib)
    perm = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(3))
    bs = c.block_size
    w2 = copy.copy(wl)
    bt = wl.block_tables.long()
    w2.block_tables = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32)
    w2.slot_hist = (perm[wl.slot_hist.long() // bs] * bs + wl.slot_hist.long() % bs).to(torch.int32)
    w2.slot_new = (perm[wl.slot_new.long() // bs] * bs + wl.slot_new.long() % bs).to(torch.int32)
    out2, _, _ = _run_prefill(w2, lib)
    assert np.array_equal(out, out2), "block relabelling changed the prefill result"


def pin_prefill_errors(lib):
    c = pcfg(hist_lo=4, hist_hi=12)
    wl = W.generate_prefill(c, 30)
    out, kp, vp = _run_prefill(wl, lib)
    cu, T = wl.cu_q_lens, wl.total_q

    def call(bt=None, cu_=None, cl=None):
        return O.paged_attention_prefill(wl.q, kp, vp, wl.block_tables if bt is None else bt,
                                         cu if cu_ is None else cu_, wl.context_lens if cl is None else cl,
                                         c.num_kv_heads, c.block_size, c.softmax_scale, lib=lib)

    rows1 = slice(int(cu[1]), int(cu[2]))
    others = np.r_[0:int(cu[1]), int(cu[2]):T]
    bt = wl.block_tables.clone()
    bt[1, 0] = wl.num_blocks
    o, st = call(bt=bt)
    assert st == O.ORC_ERR_BOUNDS and np.all(o[rows1] == 0) and np.array_equal(o[others], out[others])
    cl = wl.context_lens.clone()
    cl[1] = int(cu[2] - cu[1]) - 1  # a chunk longer than its context
    o, st = call(cl=cl)
    assert st == O.ORC_ERR_BOUNDS and np.all(o[rows1] == 0) and np.array_equal(o[others], out[others])
    full = wl.block_tables.clone()
    full[1, :] = full[1, 0]
    cl = wl.context_lens.clone()
    cl[1] = c.max_blocks_per_seq * c.block_size + 1
    o, st = call(bt=full, cl=cl)
    assert st == O.ORC_ERR_BOUNDS and np.all(o[rows1] == 0)
    bad = cu.clone()
    bad[1] = int(cu[2]) + 1  # decreasing from entry 1 to entry 2
    assert call(cu_=bad)[1] == O.ORC_ERR_ARG
    bad = cu.clone()
    bad[-1] -= 1  # does not end at total_q
    assert call(cu_=bad)[1] == O.ORC_ERR_ARG


# ----------------------------------------------------------- add + RMSNorm


def pin_rmsnorm_library(lib):
    """out against torch's rms_norm (a library routine) in fp64 on the exact
    sum, for several widths, eps values and with / without a residual."""
    for T, H, eps, res, seed in ((3, 64, 1e-6, True, 1), (4, 1000, 1e-5, True, 2), (2, 8, 0.5, False, 3),
                                 (5, 4096, 1e-6, True, 4)):
        wl = W.generate_norm(W.NormConfig("p", T, H, eps, res), seed)
        out, _, st = O.fused_add_rmsnorm(wl.x, wl.residual, wl.weight, eps, lib=lib)
        assert st == O.ORC_OK
        h = wl.x.double() + (wl.residual.double() if res else 0)
        want = torch.nn.functional.rms_norm(h, (H,), wl.weight.double(), eps).numpy()
        rel = np.abs(out - want).max() / np.abs(want).max()
        assert rel <= 1e-13, f"rms_norm T={T} H={H}: rel {rel:.2e}"


def pin_rmsnorm_residual_is_rounded_sum(lib):
    """residual_out is the bf16 (round to nearest even) of x + r: torch's own
    bf16 cast of the fp64 sum; and the bf16 rounding itself on arbitrary
    binary32 values against torch's cast."""
    wl = W.generate_norm(W.NormConfig("p", 16, 256), 5)
    wl.residual[0, :8] = torch.tensor([1.0, -1.0, 2.0 ** -130, 3.0e38, 65504.0, 0.0, -0.0, 1e-3]).to(torch.bfloat16)
    wl.x[0, :8] = torch.tensor([2.0 ** -8, -(2.0 ** -8), 2.0 ** -131, 3.0e38, 1.0, -0.0, -0.0, 3.0]).to(torch.bfloat16)
    _, rout, st = O.fused_add_rmsnorm(wl.x, wl.residual, wl.weight, 1e-6, lib=lib)
    want = (wl.x.double() + wl.residual.double()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert st == O.ORC_OK and np.array_equal(rout, want), "residual_out is not bf16(x + r)"
    g = torch.Generator().manual_seed(6)
    bits = torch.randint(-(2 ** 31), 2 ** 31 - 1, (20000,), generator=g, dtype=torch.int64).to(torch.int32)
    f = bits.view(torch.float32)
    f = f[torch.isfinite(f)]
    ties = (torch.randint(0, 2 ** 16, (2000,), generator=g).to(torch.int32) << 16 | 0x8000).view(torch.float32)
    vals = torch.cat([f, ties[torch.isfinite(ties)]])
    want = vals.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.bf16_from_double(float(v), lib=lib) for v in vals.tolist()], dtype=np.uint16)
    assert np.array_equal(got, want), "bf16 rounding differs from torch's cast"


def pin_rmsnorm_closed_forms(lib):
    H = 32
    w = torch.linspace(0.5, 1.5, H).to(torch.bfloat16)
    for c in (0.75, -3.0, 1e-3):
        x = torch.full((1, H), c).to(torch.bfloat16)
        out, _, _ = O.fused_add_rmsnorm(x, None, w, 1e-6, lib=lib)
        cb = float(x[0, 0])
        want = w.double().numpy() * cb / np.sqrt(cb * cb + 1e-6)
        _assert_close(out[0], want, tol=1e-14, what=f"constant row {c}")
    z = torch.zeros((2, H), dtype=torch.bfloat16)
    out, _, _ = O.fused_add_rmsnorm(z, z, w, 1e-6, lib=lib)
    assert np.array_equal(out, np.zeros_like(out)), "a zero row normalises to zeros"
    wl = W.generate_norm(W.NormConfig("p", 3, H, 0.0, False), 7)
    o1, _, _ = O.fused_add_rmsnorm(wl.x, None, wl.weight, 0.0, lib=lib)
    o2, _, _ = O.fused_add_rmsnorm((wl.x.float() * -4.0).to(torch.bfloat16), None, wl.weight, 0.0, lib=lib)
    _assert_close(o1, -o2, tol=1e-14, what="eps 0: scaling the row by -4 flips the sign only")
    r0 = torch.zeros_like(wl.x)
    o3, _, _ = O.fused_add_rmsnorm(wl.x, r0, wl.weight, 0.0, lib=lib)
    assert np.array_equal(o1, o3), "a zero residual is no residual"


# ------------------------------------------------ rotary embedding + store
# The rotation of the RoFormer paper (Su et al., 2021): pair i of a token at
# position m turns by m * theta_i, theta_i = base^(-2i/d). The references
# below recompute the angles from that definition in fp64, independently of
# the fp32 table the oracle reads.


def _rope_pairs(d, style):
    i = np.arange(d // 2)
    return (2 * i, 2 * i + 1) if style == W.ROPE_INTERLEAVED else (i, i + d // 2)


def rope_fp64(x_bf16, positions, d, base, style):
    """fp64 rotation of bf16 rows [N, H, d] from the definition."""
    x = x_bf16.float().double().numpy()
    m = positions.long().numpy().astype(np.float64)[:, None, None]
    i = np.arange(d // 2, dtype=np.float64)
    ang = m * base ** (-2.0 * i / d)[None, None, :]
    a, b = _rope_pairs(d, style)
    out = np.empty_like(x)
    out[..., a] = x[..., a] * np.cos(ang) - x[..., b] * np.sin(ang)
    out[..., b] = x[..., a] * np.sin(ang) + x[..., b] * np.cos(ang)
    return out


def _bf16_bits_to_f64(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).double().numpy()


def rcfg(**kw) -> W.RopeConfig:
    base = dict(name="rope", num_tokens=7, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                max_position=5000)
    base.update(kw)
    return W.RopeConfig(**base)


def pin_rope_position_zero_is_identity(lib):
    for style in (W.ROPE_HALF, W.ROPE_INTERLEAVED):
        wl = W.generate_rope(rcfg(style=style), 31)
        pos = torch.zeros_like(wl.positions)
        out, st = O.rope(wl.k, pos, wl.cos_sin, style, lib=lib)
        assert st == O.ORC_OK and np.array_equal(out, wl.k.view(torch.int16).numpy().view(np.uint16)), \
            "position 0 must leave every element unchanged"


def pin_rope_fp64_rotation(lib):
    """Within one bf16 rounding (plus binary32 slack) of the fp64 rotation,
    for both pairings, head sizes 64 and 128, positions up to 32767."""
    for style in (W.ROPE_HALF, W.ROPE_INTERLEAVED):
        for d, mp, base in ((64, 5000, 10000.0), (128, 32768, 1_000_000.0)):
            wl = W.generate_rope(rcfg(style=style, head_dim=d, max_position=mp, base=base, num_tokens=40), 32)
            out, st = O.rope(wl.q, wl.positions, wl.cos_sin, style, lib=lib)
            assert st == O.ORC_OK
            got = _bf16_bits_to_f64(out)
            ref = rope_fp64(wl.q, wl.positions, d, base, style)
            x = wl.q.float().double().numpy()
            a, b = _rope_pairs(d, style)
            pair = np.abs(x[..., a]) + np.abs(x[..., b])  # binary32 slack scales with the pair's size
            slack_full = np.empty_like(x)
            slack_full[..., a] = pair
            slack_full[..., b] = pair
            err = np.abs(got - ref)
            assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -18 * slack_full + 1e-30), \
                f"style {style} d {d}: max err {err.max():.3e}"


def pin_rope_styles_are_a_permutation(lib):
    """The two pairings are the same rotation on permuted coordinates: moving
    element i + d/2 next to element i turns the half pairing into the
    neighbour pairing, bit for bit."""
    d = 128
    wl = W.generate_rope(rcfg(head_dim=d, num_tokens=20), 33)
    perm = np.empty(d, dtype=np.int64)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    half, st1 = O.rope(wl.k, wl.positions, wl.cos_sin, W.ROPE_HALF, lib=lib)
    inter, st2 = O.rope(wl.k[..., torch.from_numpy(perm)].contiguous(), wl.positions, wl.cos_sin,
                        W.ROPE_INTERLEAVED, lib=lib)
    assert st1 == st2 == O.ORC_OK
    assert np.array_equal(half[..., perm], inter), "pairings differ by more than a permutation"


def pin_rope_relative_positions(lib):
    """<R_m q, R_n k> depends only on n - m: it equals <q, R_{n-m} k>
    evaluated in fp64 from the definition (within bf16 rounding)."""
    d, base = 128, 10000.0
    for style in (W.ROPE_HALF, W.ROPE_INTERLEAVED):
        wl = W.generate_rope(rcfg(head_dim=d, base=base, style=style, num_tokens=24, num_q_heads=2,
                                  num_kv_heads=2), 34)
        pos_q = wl.positions
        pos_k = torch.flip(wl.positions, [0])
        rq, st1 = O.rope(wl.q, pos_q, wl.cos_sin, style, lib=lib)
        rk, st2 = O.rope(wl.k, pos_k, wl.cos_sin, style, lib=lib)
        assert st1 == st2 == O.ORC_OK
        dots = (_bf16_bits_to_f64(rq) * _bf16_bits_to_f64(rk)).sum(-1)
        rel = rope_fp64(wl.k, pos_k - pos_q, d, base, style)  # R_{n-m} k (negative angles allowed)
        ref = (wl.q.float().double().numpy() * rel).sum(-1)
        nq = np.linalg.norm(wl.q.float().double().numpy(), axis=-1)
        nk = np.linalg.norm(wl.k.float().double().numpy(), axis=-1)
        assert np.all(np.abs(dots - ref) <= 2.0 ** -7 * nq * nk), np.abs(dots - ref).max()


def pin_rope_bounds(lib):
    wl = W.generate_rope(rcfg(max_position=100), 35)
    pos = wl.positions.clone() % 100
    pos[1] = -1
    pos[3] = 100
    out, st = O.rope(wl.k, pos, wl.cos_sin[:100], W.ROPE_HALF, lib=lib)
    assert st == O.ORC_ERR_BOUNDS
    assert not out[1].any() and not out[3].any(), "rows with a bad position must stay unwritten"
    good, st2 = O.rope(wl.k[[0, 2]], pos[[0, 2]], wl.cos_sin[:100], W.ROPE_HALF, lib=lib)
    assert st2 == O.ORC_OK and np.array_equal(out[[0, 2]], good)


def pin_store_rope_is_rope_then_store(lib):
    """The fused call equals rope of q and k followed by the plain store, for
    every cache type; a bad position stores nothing, slot -1 is skipped."""
    for dt in (W.CACHE_BF16, W.CACHE_FP8, W.CACHE_FP8_TOKEN):
        wl = W.generate_rope(rcfg(cache_dtype=dt, num_tokens=9, max_position=64), 36)
        pos = wl.positions.clone()
        pos[2] = 64  # out of range
        slots = wl.slot_mapping.clone()
        slots[4] = -1
        nb, bs, nkv, d = wl.num_blocks, wl.cfg.block_size, wl.cfg.num_kv_heads, wl.cfg.head_dim
        fp8 = dt != W.CACHE_BF16
        fill = W.CANARY_FP8 if fp8 else W.CANARY_BF16
        pools = [O.new_pool(nb, nkv, bs, d, fp8, fill) for _ in range(4)]
        if dt == W.CACHE_FP8_TOKEN:
            sc = [O.new_scale_pool(nb, nkv, bs) for _ in range(4)]
        else:
            sc = [wl.k_scale, wl.v_scale, wl.k_scale, wl.v_scale]
        q_out, st = O.store_kvcache_rope(wl.q, wl.k, wl.v, pools[0], pools[1], slots, pos, wl.cos_sin, nb, bs,
                                         sc[0], sc[1], lib=lib)
        assert st == O.ORC_ERR_BOUNDS
        rq, _ = O.rope(wl.q, pos, wl.cos_sin, lib=lib)
        rk, _ = O.rope(wl.k, pos, wl.cos_sin, lib=lib)
        slots2 = slots.clone()
        slots2[2] = -1
        st2 = O.store_kvcache(torch.from_numpy(rk.view(np.int16)).view(torch.bfloat16), wl.v, pools[2], pools[3],
                              slots2, nb, bs, sc[2], sc[3], lib=lib)
        assert st2 == O.ORC_OK
        assert np.array_equal(q_out, rq)
        assert np.array_equal(pools[0], pools[2]) and np.array_equal(pools[1], pools[3]), dt
        if dt == W.CACHE_FP8_TOKEN:
            assert np.array_equal(sc[0], sc[2], equal_nan=True) and np.array_equal(sc[1], sc[3], equal_nan=True)


def pin_rope_table(lib):
    """The workload's table is the definition's cos and sin in binary32."""
    cs = W.rope_cache(300, 64, 10000.0).double().numpy()
    i = np.arange(32)
    for m in (0, 1, 7, 299):
        ang = m * 10000.0 ** (-2.0 * i / 64)
        assert np.all(np.abs(cs[m, :32] - np.cos(ang)) <= 2.0 ** -24)
        assert np.all(np.abs(cs[m, 32:] - np.sin(ang)) <= 2.0 ** -24)


ALL_PINS = [
    pin_rope_position_zero_is_identity,
    pin_rope_fp64_rotation,
    pin_rope_styles_are_a_permutation,
    pin_rope_relative_positions,
    pin_rope_bounds,
    pin_store_rope_is_rope_then_store,
    pin_rope_table,
    pin_rmsnorm_library,
    pin_rmsnorm_residual_is_rounded_sum,
    pin_rmsnorm_closed_forms,
    pin_prefill_bruteforce,
    pin_prefill_one_token_is_decode,
    pin_prefill_chunking_invariance,
    pin_prefill_causal_mask,
    pin_prefill_relabel_invariance,
    pin_prefill_errors,
    pin_bruteforce_bf16,
    pin_bruteforce_fp8,
    pin_bruteforce_fp8_token_scales,
    pin_token_scale_store,
    pin_permutation_invariance,
    pin_prefix_shared_equals_duplicated,
    pin_single_token_returns_v,
    pin_identical_keys_mean_of_v,
    pin_dominant_key_returns_its_v,
    pin_store_layout,
    pin_e4m3_decode_table,
    pin_e4m3_encode,
    pin_bf16_widening,
    pin_bounds_errors,
]


def run_all(lib) -> list[str]:
    """Names of the pins that fail (or crash) against ``lib``."""
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except Exception as e:  # noqa: BLE001 - any failure counts
            failed.append(f"{pin.__name__}: {type(e).__name__}: {str(e)[:120]}")
    return failed

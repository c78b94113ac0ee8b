"""CPU oracle for paged decode attention -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never does; it has
no CPU path at all.

The arithmetic lives in ``pkv_oracle.c`` (plain C, fp64), compiled here with
gcc into ``liboracle.so`` next to it. This module only converts numpy/torch
arrays to pointers.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

ORC_OK = 0
ORC_ERR_ARG = 1
ORC_ERR_BOUNDS = 5

GCC_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC"]


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle (gcc, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _bind(lib):
    c = ctypes
    lib.orc_bf16_to_double.argtypes = [c.c_uint16]
    lib.orc_bf16_to_double.restype = c.c_double
    lib.orc_e4m3_to_double.argtypes = [c.c_uint8]
    lib.orc_e4m3_to_double.restype = c.c_double
    lib.orc_e4m3_from_float.argtypes = [c.c_float]
    lib.orc_e4m3_from_float.restype = c.c_uint8
    lib.orc_store_kvcache.argtypes = [c.c_void_p] * 5 + [c.c_int64, c.c_int, c.c_int, c.c_int, c.c_int64,
                                                          c.c_int, c.c_void_p, c.c_void_p]
    lib.orc_store_kvcache.restype = c.c_int
    lib.orc_paged_attention_decode.argtypes = (
        [c.c_void_p] * 4 + [c.c_int, c.c_void_p] + [c.c_int] * 5 + [c.c_int64, c.c_float, c.c_int]
        + [c.c_void_p] * 3 + [c.c_int]
    )
    lib.orc_paged_attention_decode.restype = c.c_int
    lib.orc_paged_attention_prefill.argtypes = (
        [c.c_void_p] * 4 + [c.c_int, c.c_void_p, c.c_void_p] + [c.c_int] * 6 + [c.c_int64, c.c_float, c.c_int]
        + [c.c_void_p] * 3 + [c.c_int]
    )
    lib.orc_paged_attention_prefill.restype = c.c_int
    lib.orc_bf16_from_double.argtypes = [c.c_double]
    lib.orc_bf16_from_double.restype = c.c_uint16
    lib.orc_fused_add_rmsnorm.argtypes = [c.c_void_p, c.c_void_p, c.c_void_p, c.c_int, c.c_int, c.c_double,
                                          c.c_void_p, c.c_void_p, c.c_int]
    lib.orc_fused_add_rmsnorm.restype = c.c_int
    lib.orc_rope.argtypes = [c.c_void_p] * 3 + [c.c_int64, c.c_int, c.c_int, c.c_void_p, c.c_int64, c.c_int]
    lib.orc_rope.restype = c.c_int
    lib.orc_store_kvcache_rope.argtypes = ([c.c_void_p] * 8 + [c.c_int64, c.c_int, c.c_int, c.c_int, c.c_int,
                                                                c.c_int64, c.c_int, c.c_void_p, c.c_void_p,
                                                                c.c_void_p, c.c_int64, c.c_int])
    lib.orc_store_kvcache_rope.restype = c.c_int
    return lib


def load(path: str | None = None):
    """Load (building first if needed) and return the ctypes library."""
    global _lib
    with _lock:
        if path is not None:
            return _bind(ctypes.CDLL(path))
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _np(x, dtype):
    """Host, C-contiguous numpy view of a torch tensor or array (bit-cast)."""
    if hasattr(x, "detach"):
        import torch

        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            x = x.view(torch.int16)
        elif x.dtype == getattr(torch, "float8_e4m3fn", None):
            x = x.view(torch.uint8)
        x = x.numpy()
    a = np.ascontiguousarray(x)
    if a.dtype != np.dtype(dtype):
        if a.dtype.itemsize == np.dtype(dtype).itemsize and a.dtype.kind in "iuV" and np.dtype(dtype).kind in "iu":
            a = a.view(dtype)
        else:
            a = a.astype(dtype)
    return a


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def new_pool(num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int, fp8: bool, fill: int):
    """A host KV pool filled with ``fill`` (bf16 bits or an E4M3 code)."""
    shape = (num_blocks, num_kv_heads, block_size, head_dim)
    return np.full(shape, fill, dtype=np.uint8 if fp8 else np.uint16)


def fp8_mode(k_cache, k_scale) -> int:
    """0: bf16 pool; 1: E4M3 with a scale per KV head ([nkv]); 2: E4M3 with
    a scale per token and KV head (scale pools [num_blocks, nkv, block_size])."""
    if k_cache.dtype != np.uint8:
        return 0
    return 2 if k_scale is not None and np.ndim(k_scale) == 3 else 1


def new_scale_pool(num_blocks: int, num_kv_heads: int, block_size: int):
    """A per-token scale pool, NaN where no token was stored."""
    return np.full((num_blocks, num_kv_heads, block_size), np.nan, dtype=np.float32)


def store_kvcache(k, v, k_cache, v_cache, slot_mapping, num_blocks, block_size, k_scale=None, v_scale=None,
                  lib=None) -> int:
    """Write rows of k/v ``[N, nkv, d]`` (bf16) into host pools, in place.
    With per-token scale pools (numpy, 3-D) the scales are written too."""
    lib = lib or load()
    k = _np(k, np.uint16)
    v = _np(v, np.uint16)
    sm = _np(slot_mapping, np.int32)
    N, nkv, d = k.shape
    mode = fp8_mode(k_cache, k_scale)
    if mode == 2:
        assert k_scale.dtype == np.float32 and k_scale.flags.c_contiguous and v_scale.flags.c_contiguous
        ks, vs = k_scale, v_scale  # written in place
    else:
        ks = _np(k_scale, np.float32) if mode else None
        vs = _np(v_scale, np.float32) if mode else None
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    return lib.orc_store_kvcache(_p(k), _p(v), _p(k_cache), _p(v_cache), _p(sm), N, nkv, d, block_size,
                                 num_blocks, mode, _p(ks), _p(vs))


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, num_kv_heads, block_size,
                           scale, k_scale=None, v_scale=None, num_threads=1, lib=None):
    """fp64 attention of each sequence's query heads over its paged K/V.

    Returns ``(out [S, nq, d] float64, status)``.
    """
    lib = lib or load()
    q = _np(q, np.uint16)
    bt = _np(block_tables, np.int32)
    cl = _np(context_lens, np.int32)
    S, nq, d = q.shape
    fp8 = fp8_mode(k_cache, k_scale)
    ks = _np(k_scale, np.float32) if fp8 else None
    vs = _np(v_scale, np.float32) if fp8 else None
    out = np.zeros((S, nq, d), dtype=np.float64)
    nblk = k_cache.shape[0]
    st = lib.orc_paged_attention_decode(_p(q), _p(k_cache), _p(v_cache), _p(bt), bt.shape[1], _p(cl), S, nq,
                                        num_kv_heads, d, block_size, nblk, float(scale), int(fp8), _p(ks),
                                        _p(vs), _p(out), int(num_threads))
    return out, st


def paged_attention_prefill(q, k_cache, v_cache, block_tables, cu_q_lens, context_lens, num_kv_heads, block_size,
                            scale, k_scale=None, v_scale=None, num_threads=1, lib=None):
    """fp64 causal attention of each sequence's chunk of query tokens over its
    paged K/V (the chunk is the last ``c`` of its ``context_lens`` positions).

    ``q`` is ``[total_q, nq, d]`` bf16, ``cu_q_lens`` ``[S + 1]``. Returns
    ``(out [total_q, nq, d] float64, status)``.
    """
    lib = lib or load()
    q = _np(q, np.uint16)
    bt = _np(block_tables, np.int32)
    cu = _np(cu_q_lens, np.int32)
    cl = _np(context_lens, np.int32)
    T, nq, d = q.shape
    S = cl.shape[0]
    assert cu.shape == (S + 1,)
    fp8 = fp8_mode(k_cache, k_scale)
    ks = _np(k_scale, np.float32) if fp8 else None
    vs = _np(v_scale, np.float32) if fp8 else None
    out = np.zeros((T, nq, d), dtype=np.float64)
    nblk = k_cache.shape[0]
    st = lib.orc_paged_attention_prefill(_p(q), _p(k_cache), _p(v_cache), _p(bt), bt.shape[1], _p(cu), _p(cl), S,
                                         T, nq, num_kv_heads, d, block_size, nblk, float(scale), int(fp8), _p(ks),
                                         _p(vs), _p(out), int(num_threads))
    return out, st


def rope(x, positions, cos_sin, style=0, lib=None):
    """bf16 rows ``[N, heads, d]`` rotated at ``positions`` with the binary32
    table ``cos_sin [max_position, d]`` (cos of the d/2 angles, then sin).
    Returns ``(out uint16 [N, heads, d], status)``; rows with an out-of-range
    position stay zero."""
    lib = lib or load()
    x = _np(x, np.uint16)
    pos = _np(positions, np.int32)
    cs = _np(cos_sin, np.float32)
    N, H, d = x.shape
    out = np.zeros_like(x)
    st = lib.orc_rope(_p(x), _p(out), _p(pos), N, H, d, _p(cs), cs.shape[0], int(style))
    return out, st


def store_kvcache_rope(q, k, v, k_cache, v_cache, slot_mapping, positions, cos_sin, num_blocks, block_size,
                       k_scale=None, v_scale=None, style=0, lib=None):
    """orc_rope of q and k, then orc_store_kvcache of the rotated k and of v
    into the host pools (in place). ``q`` may be None. Returns
    ``(q_out uint16 or None, status)``."""
    lib = lib or load()
    k = _np(k, np.uint16)
    v = _np(v, np.uint16)
    sm = _np(slot_mapping, np.int32)
    pos = _np(positions, np.int32)
    cs = _np(cos_sin, np.float32)
    N, nkv, d = k.shape
    mode = fp8_mode(k_cache, k_scale)
    if mode == 2:
        ks, vs = k_scale, v_scale
    else:
        ks = _np(k_scale, np.float32) if mode else None
        vs = _np(v_scale, np.float32) if mode else None
    qn = _np(q, np.uint16) if q is not None else None
    q_out = np.zeros_like(qn) if qn is not None else None
    nq = qn.shape[1] if qn is not None else 0
    st = lib.orc_store_kvcache_rope(_p(qn), _p(q_out), _p(k), _p(v), _p(k_cache), _p(v_cache), _p(sm), _p(pos), N,
                                    nq, nkv, d, block_size, num_blocks, mode, _p(ks), _p(vs), _p(cs), cs.shape[0],
                                    int(style))
    return q_out, st


def e4m3_from_float(y: float, lib=None) -> int:
    return (lib or load()).orc_e4m3_from_float(float(y))


def e4m3_to_double(code: int, lib=None) -> float:
    return (lib or load()).orc_e4m3_to_double(int(code))


def bf16_to_double(bits: int, lib=None) -> float:
    return (lib or load()).orc_bf16_to_double(int(bits))


def run_workload(wl, num_threads=1, seq_ids=None, lib=None):
    """Fill host pools from a workload's history and step tokens, then decode.

    With ``seq_ids`` only those sequences' blocks are filled and decoded (a
    sample of a full-size step). Returns ``(out, k_pool, v_pool, status)``
    where ``out`` rows follow ``seq_ids`` (or all sequences).
    """
    from paged_kv_cache_482_b200 import workloads as W

    cfg = wl.cfg
    fp8 = wl.is_fp8
    fill = W.CANARY_FP8 if fp8 else W.CANARY_BF16
    kp = new_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size, cfg.head_dim, fp8, fill)
    vp = new_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size, cfg.head_dim, fp8, fill)
    ks, vs = wl.k_scale, wl.v_scale
    if wl.token_scales:
        ks = new_scale_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size)
        vs = new_scale_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size)
    if seq_ids is None:
        sub = dict(k_hist=wl.k_hist, v_hist=wl.v_hist, slot_hist=wl.slot_hist, q=wl.q, k_new=wl.k_new,
                   v_new=wl.v_new, slot_new=wl.slot_new, block_tables=wl.block_tables,
                   context_lens=wl.context_lens)
    else:
        sub = W.subset_for_seqs(wl, seq_ids)
    st1 = store_kvcache(sub["k_hist"], sub["v_hist"], kp, vp, sub["slot_hist"], wl.num_blocks, cfg.block_size,
                        ks, vs, lib=lib)
    st2 = store_kvcache(sub["k_new"], sub["v_new"], kp, vp, sub["slot_new"], wl.num_blocks, cfg.block_size,
                        ks, vs, lib=lib)
    out, st3 = paged_attention_decode(sub["q"], kp, vp, sub["block_tables"], sub["context_lens"],
                                      cfg.num_kv_heads, cfg.block_size, cfg.softmax_scale, ks, vs,
                                      num_threads=num_threads, lib=lib)
    if wl.token_scales:
        return out, kp, vp, st1 | st2 | st3, ks, vs
    return out, kp, vp, st1 | st2 | st3


def run_prefill_workload(wl, num_threads=1, lib=None):
    """Fill host pools from a prefill workload's history, store its chunk
    tokens, then attend. Returns ``(out [T, nq, d], k_pool, v_pool, status)``."""
    from paged_kv_cache_482_b200 import workloads as W

    cfg = wl.cfg
    fp8 = wl.is_fp8
    fill = W.CANARY_FP8 if fp8 else W.CANARY_BF16
    kp = new_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size, cfg.head_dim, fp8, fill)
    vp = new_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size, cfg.head_dim, fp8, fill)
    ks, vs = wl.k_scale, wl.v_scale
    if wl.token_scales:
        ks = new_scale_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size)
        vs = new_scale_pool(wl.num_blocks, cfg.num_kv_heads, cfg.block_size)
    st1 = store_kvcache(wl.k_hist, wl.v_hist, kp, vp, wl.slot_hist, wl.num_blocks, cfg.block_size, ks, vs, lib=lib)
    st2 = store_kvcache(wl.k_new, wl.v_new, kp, vp, wl.slot_new, wl.num_blocks, cfg.block_size, ks, vs, lib=lib)
    out, st3 = paged_attention_prefill(wl.q, kp, vp, wl.block_tables, wl.cu_q_lens, wl.context_lens,
                                       cfg.num_kv_heads, cfg.block_size, cfg.softmax_scale, ks, vs,
                                       num_threads=num_threads, lib=lib)
    if wl.token_scales:
        return out, kp, vp, st1 | st2 | st3, ks, vs
    return out, kp, vp, st1 | st2 | st3


def bf16_from_double(v: float, lib=None) -> int:
    return (lib or load()).orc_bf16_from_double(float(v))


def fused_add_rmsnorm(x, residual, weight, eps, num_threads=1, lib=None):
    """fp64 residual add + RMSNorm of rows ``x`` ``[T, H]`` (bf16).

    Returns ``(out [T, H] float64, residual_out [T, H] bf16 bits or None, status)``.
    """
    lib = lib or load()
    x = _np(x, np.uint16)
    T, H = x.shape
    r = _np(residual, np.uint16) if residual is not None else None
    w = _np(weight, np.uint16)
    out = np.zeros((T, H), dtype=np.float64)
    rout = np.zeros((T, H), dtype=np.uint16) if r is not None else None
    st = lib.orc_fused_add_rmsnorm(_p(x), _p(r), _p(w), T, H, float(eps), _p(out), _p(rout), int(num_threads))
    return out, rout, st

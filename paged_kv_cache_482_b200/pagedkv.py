"""Python binding of libpagedkv.so (ctypes).

Argument marshalling only: tensors become device pointers, shapes become
sizes, the current torch CUDA stream becomes the ``stream`` argument. Every
step of the computation runs in the library's CUDA kernels. There is no CPU
path: if ``libpagedkv.so`` is missing or cannot load, ``lib()`` raises.

The functions mirror ``include/pagedkv.h``:

* ``store_kvcache`` -- ``pkv_store_kvcache``
* ``store_kvcache_rope`` -- ``pkv_store_kvcache_rope``
* ``plan_decode`` -- ``pkv_plan_decode``
* ``decode_workspace_bytes`` -- ``pkv_decode_workspace_bytes``
* ``paged_attention_decode`` -- ``pkv_paged_attention_decode``
* ``plan_decode_shared_prefix`` / ``paged_attention_decode_shared_prefix`` --
  ``pkv_plan_decode_shared_prefix`` / ``pkv_paged_attention_decode_shared_prefix``
* ``paged_attention_prefill`` -- ``pkv_paged_attention_prefill``
* ``prefill_workspace_bytes`` -- ``pkv_prefill_workspace_bytes``
* ``fused_add_rmsnorm`` -- ``pkv_fused_add_rmsnorm``
* ``read_device_error`` -- ``pkv_read_device_error``
"""

from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedkv.so")

PKV_OK = 0
PKV_ERR_INVALID_ARG = 1
PKV_ERR_UNSUPPORTED = 2
PKV_ERR_WORKSPACE = 3
PKV_ERR_CUDA = 4
PKV_ERR_DEVICE_BOUNDS = 5
PKV_ERR_DEVICE_TIMEOUT = 6

PKV_CACHE_BF16 = 0
PKV_CACHE_FP8_E4M3 = 1  # k_scale / v_scale: [num_kv_heads] fp32
PKV_CACHE_FP8_E4M3_TOKEN = 2  # k_scale / v_scale: scale pools [num_blocks, num_kv_heads, block_size] fp32

EXPORTED = ("pkv_store_kvcache", "pkv_store_kvcache_rope", "pkv_plan_decode", "pkv_decode_workspace_bytes",
            "pkv_plan_decode_shared_prefix", "pkv_paged_attention_decode_shared_prefix",
            "pkv_paged_attention_decode", "pkv_status_string", "pkv_read_device_error", "pkv_version",
            "pkv_paged_attention_decode_static_scratch", "pkv_paged_attention_prefill",
            "pkv_prefill_workspace_bytes", "pkv_fused_add_rmsnorm")


class PagedKVError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class _Plan(ctypes.Structure):
    _fields_ = [("partition_tokens", ctypes.c_int), ("max_partitions", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t)]


_lock = threading.Lock()
_lib = None


def lib(path: str = LIB_PATH):
    """The loaded library; raises if it is not built."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = load_library(path)
        return _lib


def load_library(path: str):
    """Load and declare a libpagedkv.so at ``path`` (not cached)."""
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m paged_kv_cache_482_b200.build` "
                           "(there is no CPU fallback)")
    L = ctypes.CDLL(path)
    c = ctypes
    vp, i32, i64, f32, sz = c.c_void_p, c.c_int, c.c_int64, c.c_float, c.c_size_t
    L.pkv_store_kvcache.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i64, i32, vp, vp, vp, vp]
    L.pkv_store_kvcache.restype = i32
    L.pkv_store_kvcache_rope.argtypes = [vp] * 9 + [i32] * 7 + [i64, i32, vp, vp, vp, vp]
    L.pkv_store_kvcache_rope.restype = i32
    L.pkv_plan_decode.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, c.POINTER(_Plan)]
    L.pkv_plan_decode.restype = i32
    L.pkv_plan_decode_shared_prefix.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, c.POINTER(_Plan)]
    L.pkv_plan_decode_shared_prefix.restype = i32
    L.pkv_paged_attention_decode_shared_prefix.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32,
                                                           i64, f32, i32, vp, vp, i32, vp, vp, i32, i32, i32, vp,
                                                           sz, vp, vp, vp]
    L.pkv_paged_attention_decode_shared_prefix.restype = i32
    L.pkv_decode_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.pkv_decode_workspace_bytes.restype = sz
    L.pkv_paged_attention_decode.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i64, f32, i32,
                                             vp, vp, i32, i32, vp, sz, vp, vp, vp]
    L.pkv_paged_attention_decode.restype = i32
    L.pkv_status_string.argtypes = [i32]
    L.pkv_status_string.restype = c.c_char_p
    L.pkv_read_device_error.argtypes = [vp, vp]
    L.pkv_read_device_error.restype = i32
    L.pkv_version.argtypes = []
    L.pkv_version.restype = i32
    L.pkv_paged_attention_prefill.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, i32, i64, f32,
                                              i32, vp, vp, i32, vp, sz, vp, vp, vp]
    L.pkv_paged_attention_prefill.restype = i32
    L.pkv_prefill_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    L.pkv_prefill_workspace_bytes.restype = sz
    L.pkv_fused_add_rmsnorm.argtypes = [vp, vp, vp, vp, i32, i32, f32, vp]
    L.pkv_fused_add_rmsnorm.restype = i32
    if hasattr(L, "pkv_paged_attention_decode_static_scratch"):
        L.pkv_paged_attention_decode_static_scratch.argtypes = [vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32,
                                                                i32, i64, f32, i32, vp, vp, i32, i32, vp, vp, vp]
        L.pkv_paged_attention_decode_static_scratch.restype = i32
    return L


def status_string(status: int) -> str:
    return lib().pkv_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _cache_dtype(t: torch.Tensor, k_scale=None) -> int:
    """The pool's cache type; an E4M3 pool whose scales are 3-D scale pools
    ([num_blocks, num_kv_heads, block_size]) has one scale per token."""
    if t.dtype == torch.bfloat16:
        return PKV_CACHE_BF16
    if t.dtype in (torch.uint8, getattr(torch, "float8_e4m3fn", torch.uint8)):
        if k_scale is not None and k_scale.dim() == 3:
            if k_scale.shape != t.shape[:3] or k_scale.dtype != torch.float32 or not k_scale.is_contiguous():
                raise ValueError("per-token scale pools must be contiguous fp32 [num_blocks, num_kv_heads, block_size]")
            return PKV_CACHE_FP8_E4M3_TOKEN
        return PKV_CACHE_FP8_E4M3
    raise TypeError(f"KV pool dtype {t.dtype}: expected bfloat16 or an 8-bit E4M3 container")


def _check(status: int, where: str):
    if status != PKV_OK:
        raise PagedKVError(status, where)


def store_kvcache(k, v, k_cache, v_cache, slot_mapping, k_scale=None, v_scale=None, dev_err=None, stream=None):
    """Write k/v ``[N, nkv, d]`` bf16 rows into pool slots ``slot_mapping`` (-1 skips)."""
    if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("k and v must be bfloat16")
    if not (k.is_contiguous() and v.is_contiguous() and k_cache.is_contiguous() and v_cache.is_contiguous()):
        raise ValueError("k, v and the pools must be contiguous")
    if slot_mapping.dtype != torch.int32:
        raise TypeError("slot_mapping must be int32")
    N, nkv, d = k.shape
    nblk, nkv2, bs, d2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or nkv2 != nkv or d2 != d or slot_mapping.numel() != N:
        raise ValueError("shape mismatch between k/v, pools and slot_mapping")
    st = lib().pkv_store_kvcache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), N, nkv, d, bs,
                                 nblk, _cache_dtype(k_cache, k_scale), _ptr(k_scale), _ptr(v_scale), _ptr(dev_err),
                                 _stream(stream))
    _check(st, "pkv_store_kvcache")


def store_kvcache_rope(k, v, k_cache, v_cache, slot_mapping, positions, cos_sin, q=None, q_out=None, style=0,
                       k_scale=None, v_scale=None, dev_err=None, stream=None):
    """Rotate k (and q into ``q_out``) at ``positions`` with the fp32 table
    ``cos_sin [max_position, d]``, then store the rotated k and v like
    ``store_kvcache``. Returns ``q_out`` (allocated when q is given without it)."""
    if k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("k and v must be bfloat16")
    if slot_mapping.dtype != torch.int32 or positions.dtype != torch.int32:
        raise TypeError("slot_mapping and positions must be int32")
    if cos_sin.dtype != torch.float32 or cos_sin.dim() != 2 or not cos_sin.is_contiguous():
        raise TypeError("cos_sin must be a contiguous fp32 [max_position, head_dim] table")
    for t in (k, v, k_cache, v_cache):
        if not t.is_contiguous():
            raise ValueError("k, v and the pools must be contiguous")
    N, nkv, d = k.shape
    nblk, nkv2, bs, d2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or nkv2 != nkv or d2 != d:
        raise ValueError("shape mismatch between k/v and the pools")
    if slot_mapping.numel() != N or positions.numel() != N or cos_sin.shape[1] != d:
        raise ValueError("slot_mapping / positions / cos_sin do not match k")
    nq = 0
    if q is not None:
        if q.dtype != torch.bfloat16 or not q.is_contiguous() or q.shape[0] != N or q.shape[2] != d:
            raise ValueError("q must be contiguous bf16 [N, nq, head_dim]")
        nq = q.shape[1]
        if q_out is None:
            q_out = torch.empty_like(q)
    st = lib().pkv_store_kvcache_rope(_ptr(q), _ptr(q_out), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(slot_mapping), _ptr(positions), _ptr(cos_sin), cos_sin.shape[0], style, N,
                                      nq, nkv, d, bs, nblk, _cache_dtype(k_cache, k_scale), _ptr(k_scale),
                                      _ptr(v_scale), _ptr(dev_err), _stream(stream))
    _check(st, "pkv_store_kvcache_rope")
    return q_out


def plan_decode(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len, fp8=False,
                partition_request=0) -> dict:
    plan = _Plan()
    st = lib().pkv_plan_decode(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                               PKV_CACHE_FP8_E4M3 if fp8 else PKV_CACHE_BF16, partition_request,
                               ctypes.byref(plan))
    _check(st, "pkv_plan_decode")
    return dict(partition_tokens=plan.partition_tokens, max_partitions=plan.max_partitions,
                workspace_bytes=plan.workspace_bytes)


def plan_decode_shared_prefix(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_context_len,
                              cache_dtype=PKV_CACHE_BF16, partition_request=0) -> dict:
    plan = _Plan()
    st = lib().pkv_plan_decode_shared_prefix(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                             max_context_len, int(cache_dtype), partition_request,
                                             ctypes.byref(plan))
    _check(st, "pkv_plan_decode_shared_prefix")
    return dict(partition_tokens=plan.partition_tokens, max_partitions=plan.max_partitions,
                workspace_bytes=plan.workspace_bytes)


def paged_attention_decode_shared_prefix(q, k_cache, v_cache, block_tables, context_lens, scale, cu_group_seqs,
                                         group_prefix_tokens, max_group_seqs, out=None, k_scale=None, v_scale=None,
                                         max_context_len=None, partition_request=0, workspace=None, dev_err=None,
                                         stream=None, seq_order=None):
    """Decode of a batch whose consecutive groups of sequences share cached
    prefixes (int32 device tensors ``cu_group_seqs [G+1]`` and
    ``group_prefix_tokens [G]``); same result as ``paged_attention_decode``.
    ``seq_order`` (optional, as there) orders the suffix decode."""
    S, nq, d = q.shape
    nblk, nkv, bs, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("q and the pools disagree")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if cu_group_seqs.dtype != torch.int32 or group_prefix_tokens.dtype != torch.int32:
        raise TypeError("cu_group_seqs and group_prefix_tokens must be int32")
    G = group_prefix_tokens.numel()
    if cu_group_seqs.numel() != G + 1:
        raise ValueError("cu_group_seqs must have one more entry than group_prefix_tokens")
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    dt = _cache_dtype(k_cache, k_scale)
    plan = plan_decode_shared_prefix(S, nq, nkv, d, bs, max_context_len, dt, partition_request)
    if out is None:
        out = torch.empty_like(q)
    if plan["workspace_bytes"] and workspace is None:
        workspace = torch.empty(plan["workspace_bytes"], dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if seq_order is not None and (seq_order.dtype != torch.int32 or seq_order.numel() != S):
        raise ValueError("seq_order must be an int32 permutation of the sequences")
    st = lib().pkv_paged_attention_decode_shared_prefix(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), maxb, _ptr(context_lens), _ptr(seq_order), S,
        nq, nkv, d, bs, nblk,
        float(scale), dt, _ptr(k_scale), _ptr(v_scale), int(max_context_len), _ptr(cu_group_seqs),
        _ptr(group_prefix_tokens), G, int(max_group_seqs), int(partition_request), _ptr(workspace), ws_bytes,
        _ptr(out), _ptr(dev_err), _stream(stream))
    _check(st, "pkv_paged_attention_decode_shared_prefix")
    return out


def decode_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len) -> int:
    """Scratch bytes that suffice for any automatic split-K plan of these sizes."""
    return int(lib().pkv_decode_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len))


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out=None, k_scale=None,
                           v_scale=None, max_context_len=None, partition_request=0, workspace=None, dev_err=None,
                           stream=None, seq_order=None):
    """One decode step of paged attention; returns ``out`` ``[S, nq, d]`` bf16.

    ``max_context_len`` defaults to the block-table capacity (no device
    sync). A workspace is allocated with torch when the plan needs one and
    none is given. ``seq_order`` (optional int32 device permutation of the
    sequences) sets the order in which they are scheduled; longest first
    shortens the tail (see ``longest_first``).
    """
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise TypeError("q must be contiguous bfloat16")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    if not block_tables.is_contiguous():
        raise ValueError("block_tables must be contiguous")
    S, nq, d = q.shape
    nblk, nkv, bs, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("shape mismatch")
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    dt = _cache_dtype(k_cache, k_scale)
    if out is None:
        out = torch.empty_like(q)
    plan = plan_decode(S, nq, nkv, d, bs, max_context_len, dt != PKV_CACHE_BF16, partition_request)
    if plan["workspace_bytes"] and workspace is None:
        workspace = torch.empty(plan["workspace_bytes"], dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if seq_order is not None and (seq_order.dtype != torch.int32 or seq_order.numel() != S):
        raise ValueError("seq_order must be an int32 permutation of the sequences")
    st = lib().pkv_paged_attention_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), maxb,
                                          _ptr(context_lens), _ptr(seq_order), S, nq, nkv, d, bs, nblk, float(scale),
                                          dt, _ptr(k_scale),
                                          _ptr(v_scale), int(max_context_len), int(partition_request),
                                          _ptr(workspace), ws_bytes, _ptr(out), _ptr(dev_err), _stream(stream))
    _check(st, "pkv_paged_attention_decode")
    return out


def paged_attention_decode_static_scratch(q, k_cache, v_cache, block_tables, context_lens, scale, out=None,
                                          k_scale=None, v_scale=None, max_context_len=None, partition_request=0,
                                          dev_err=None, stream=None, seq_order=None):
    """``paged_attention_decode`` for callers that cannot allocate device memory.

    The split-K scratch comes from a fixed array inside the library
    (``STATIC_SCRATCH_BYTES`` per GPU, held until exit) instead of a
    workspace; nothing is allocated by the library. Pass ``out`` to avoid the
    one allocation this wrapper would otherwise make for the result. Calls
    that overlap on the GPU share the array and must be serialised; the first
    call on a device should come before any stream capture.
    """
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise TypeError("q must be contiguous bfloat16")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32 or not block_tables.is_contiguous():
        raise TypeError("block_tables and context_lens must be contiguous int32")
    S, nq, d = q.shape
    nblk, nkv, bs, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape or block_tables.shape[0] != S or context_lens.numel() != S:
        raise ValueError("shape mismatch")
    maxb = block_tables.shape[1]
    if max_context_len is None:
        max_context_len = maxb * bs
    if out is None:
        out = torch.empty_like(q)
    dt = _cache_dtype(k_cache, k_scale)
    st = lib().pkv_paged_attention_decode_static_scratch(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                                         maxb, _ptr(context_lens), _ptr(seq_order), S, nq, nkv, d,
                                                         bs, nblk,
                                                         float(scale), dt, _ptr(k_scale), _ptr(v_scale),
                                                         int(max_context_len), int(partition_request), _ptr(out),
                                                         _ptr(dev_err), _stream(stream))
    _check(st, "pkv_paged_attention_decode_static_scratch")
    return out


STATIC_SCRATCH_BYTES = 32 << 20  # PKV_STATIC_SCRATCH_BYTES


def prefill_workspace_bytes(num_seqs, num_kv_heads, head_dim, max_blocks_per_seq, block_size, cache_dtype) -> int:
    """Bytes of the optional E4M3 widening workspace of ``paged_attention_prefill``
    (0 for a bf16 cache, or when the staging does not fit int32 rows)."""
    return int(lib().pkv_prefill_workspace_bytes(num_seqs, num_kv_heads, head_dim, max_blocks_per_seq, block_size,
                                                 cache_dtype))


def paged_attention_prefill(q, k_cache, v_cache, block_tables, cu_q_lens, context_lens, scale, max_q_len,
                            out=None, k_scale=None, v_scale=None, dev_err=None, stream=None, workspace=None):
    """Chunked prefill: each sequence's chunk of query tokens (rows
    ``cu_q_lens[i]`` .. ``cu_q_lens[i+1] - 1`` of ``q``, ``[total_q, nq, d]``
    bf16) attends causally over its paged context; returns ``out`` like ``q``.
    ``max_q_len`` is a host-known bound on every chunk length. ``workspace``
    (E4M3 cache, optional): a device buffer of at least
    ``prefill_workspace_bytes(...)`` bytes into which the codes of the long
    chunks' contexts are widened once per call (same result, fewer conversions)."""
    if q.dtype != torch.bfloat16 or not q.is_contiguous():
        raise TypeError("q must be contiguous bfloat16")
    for t, n in ((block_tables, "block_tables"), (cu_q_lens, "cu_q_lens"), (context_lens, "context_lens")):
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous int32")
    if not (k_cache.is_contiguous() and v_cache.is_contiguous()):
        raise ValueError("the pools must be contiguous")
    T, nq, d = q.shape
    nblk, nkv, bs, d2 = k_cache.shape
    if d2 != d or v_cache.shape != k_cache.shape:
        raise ValueError("pool shape does not match q")
    S = context_lens.shape[0]
    if cu_q_lens.shape[0] != S + 1 or block_tables.shape[0] != S:
        raise ValueError("cu_q_lens must have num_seqs + 1 entries and block_tables num_seqs rows")
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().pkv_paged_attention_prefill(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), block_tables.shape[1], _ptr(cu_q_lens),
        _ptr(context_lens), S, T, nq, nkv, d, bs, nblk, float(scale), _cache_dtype(k_cache, k_scale), _ptr(k_scale),
        _ptr(v_scale), int(max_q_len), _ptr(workspace), ws_bytes, _ptr(out), _ptr(dev_err), _stream(stream))
    _check(st, "pkv_paged_attention_prefill")
    return out


def fused_add_rmsnorm(x, residual, weight, eps, out=None, stream=None):
    """Residual add + RMSNorm over the last dimension of ``x`` ``[T, H]`` bf16:
    ``residual`` (or None) is updated in place to bf16(x + residual) and the
    normalised rows are returned (in ``out``; ``out=x`` works in place)."""
    for t, n in ((x, "x"), (weight, "weight")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous bfloat16")
    if residual is not None and (residual.dtype != torch.bfloat16 or not residual.is_contiguous()
                                 or residual.shape != x.shape):
        raise TypeError("residual must be contiguous bfloat16 shaped like x")
    if x.dim() != 2 or weight.shape != (x.shape[1],):
        raise ValueError("x must be [T, H] and weight [H]")
    if out is None:
        out = torch.empty_like(x)
    st = lib().pkv_fused_add_rmsnorm(_ptr(x), _ptr(residual), _ptr(weight), _ptr(out), x.shape[0], x.shape[1],
                                     float(eps), _stream(stream))
    _check(st, "pkv_fused_add_rmsnorm")
    return out


def longest_first(context_lens_host: torch.Tensor) -> torch.Tensor:
    """Host helper: the order that schedules the longest sequences first
    (stable: equal lengths keep their order; int32). Engines know their
    lengths on the host."""
    return torch.from_numpy(_longest_first_np(context_lens_host.numpy()))


def _longest_first_np(lens) -> np.ndarray:
    return np.argsort(-lens.astype(np.int64), kind="stable").astype(np.int32)


def read_device_error(dev_err, stream=None) -> int:
    """Synchronise the stream and map the device error word to a status."""
    return lib().pkv_read_device_error(_ptr(dev_err), _stream(stream))


def version() -> int:
    return lib().pkv_version()


def graphed(fn):
    """Record ``fn()`` (library calls on fixed device tensors) once as a CUDA
    graph and return a function that replays it on the current stream. ``fn``
    runs once first, outside the capture, so that one-time set-up (kernel
    attributes, the library's side stream) is done before recording."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()

    def replay():
        g.replay()

    replay.graph = g
    return replay


class DecodeStep:
    """A decode step bound to resident pools: store the step's K/V, then attend.

    Holds the plan and workspace for a fixed shape, so repeated steps launch
    only the library's kernels. ``run_host`` takes the step's inputs from host
    (pinned) memory, copies them to the device, runs the step and copies the
    output back: the end-to-end form of the call.
    """

    def __init__(self, k_cache, v_cache, num_seqs, num_q_heads, max_blocks_per_seq, scale, k_scale=None,
                 v_scale=None, max_context_len=None, partition_request=0, device=None, groups=None):
        """``groups`` = (cu_group_seqs, group_prefix_tokens, max_group_seqs):
        consecutive sequences that share cached prefixes, attended through
        ``paged_attention_decode_shared_prefix``."""
        self.k_cache, self.v_cache = k_cache, v_cache
        self.k_scale, self.v_scale = k_scale, v_scale
        nblk, nkv, bs, d = k_cache.shape
        self.shape = (num_seqs, num_q_heads, nkv, d, bs)
        self.max_blocks = max_blocks_per_seq
        self.max_context_len = max_context_len or max_blocks_per_seq * bs
        self.scale = scale
        self.partition_request = partition_request
        dev = device or k_cache.device
        self.groups = None
        if groups is not None:
            cu, pre, mg = groups
            host_cu = torch.as_tensor(cu, dtype=torch.int32).cpu()
            host_pre = torch.as_tensor(pre, dtype=torch.int32).cpu()
            if torch.cuda.is_available():
                host_cu, host_pre = host_cu.pin_memory(), host_pre.pin_memory()
            self._host_groups = (host_cu, host_pre)
            self.groups = (host_cu.to(dev), host_pre.to(dev), int(mg))
            self.plan = plan_decode_shared_prefix(num_seqs, num_q_heads, nkv, d, bs, self.max_context_len,
                                                  _cache_dtype(k_cache, k_scale), partition_request)
        else:
            self.plan = plan_decode(num_seqs, num_q_heads, nkv, d, bs, self.max_context_len,
                                    _cache_dtype(k_cache, k_scale) != PKV_CACHE_BF16, partition_request)
        self.workspace = (torch.empty(self.plan["workspace_bytes"], dtype=torch.uint8, device=dev)
                          if self.plan["workspace_bytes"] else None)
        self.out = torch.empty((num_seqs, num_q_heads, d), dtype=torch.bfloat16, device=dev)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)
        self._dev_inputs = None

    def run(self, q, k_new, v_new, slot_mapping, block_tables, context_lens, stream=None, seq_order=None):
        """Device inputs -> device output (no host traffic, no sync)."""
        store_kvcache(k_new, v_new, self.k_cache, self.v_cache, slot_mapping, self.k_scale, self.v_scale,
                      self.dev_err, stream)
        if self.groups is not None:
            cu, pre, mg = self.groups
            return paged_attention_decode_shared_prefix(
                q, self.k_cache, self.v_cache, block_tables, context_lens, self.scale, cu, pre, mg, out=self.out,
                k_scale=self.k_scale, v_scale=self.v_scale, max_context_len=self.max_context_len,
                partition_request=self.partition_request, workspace=self.workspace, dev_err=self.dev_err,
                stream=stream, seq_order=seq_order)
        return paged_attention_decode(q, self.k_cache, self.v_cache, block_tables, context_lens, self.scale,
                                      out=self.out, k_scale=self.k_scale, v_scale=self.v_scale,
                                      max_context_len=self.max_context_len,
                                      partition_request=self.partition_request, workspace=self.workspace,
                                      dev_err=self.dev_err, stream=stream, seq_order=seq_order)

    def run_host(self, q, k_new, v_new, slot_mapping, block_tables, context_lens, out_host, stream=None):
        """One step from host (pinned) inputs to a host output: the end-to-end
        form of the call. The longest-first order is computed from the host
        lengths; the inputs are copied in on a copy stream into one of two sets
        of device buffers, the step runs on ``stream`` (default: the current
        stream), and the output is copied out on a second copy stream from one
        of two device outputs. So the copies of one step overlap the kernels of
        the steps around it, and nothing waits on the host unless it runs two
        steps ahead of the GPU. The store and the attention on buffer set i are
        recorded as a CUDA graph the first time set i is used (that first step
        also runs them once eagerly; a repeated store writes the same values)
        and replayed after that, so a step costs the host one graph launch
        besides the copies. Returns once queued; ``flush(stream)`` makes
        ``stream`` wait for every queued output copy."""
        cs = stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.current_stream()
        dev = self.k_cache.device
        if self._dev_inputs is None:
            self._h2d, self._d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
            self._dev_inputs, self._outs, self._order_host, self._graphs = [], [], [], [None, None]
            for _ in range(2):
                self._dev_inputs.append([torch.empty(t.shape, dtype=t.dtype, device=dev)
                                         for t in (q, k_new, v_new, slot_mapping, block_tables, context_lens)] +
                                        [torch.empty(context_lens.shape, dtype=torch.int32, device=dev)])
                self._outs.append(torch.empty_like(self.out))
                self._order_host.append(torch.empty(context_lens.shape, dtype=torch.int32).pin_memory())
            # events reused step after step (re-recording one is safe once its
            # earlier waits are queued); "used" marks a set's first round
            self._ev_ready = [torch.cuda.Event(), torch.cuda.Event()]
            self._ev_free = [torch.cuda.Event(), torch.cuda.Event()]
            self._ev_out = [torch.cuda.Event(), torch.cuda.Event()]
            self._used = [False, False]
            self._flip = 0
            self._primed = False
        if not self._primed:  # the first copies start after what is already queued on cs
            start = torch.cuda.Event()
            start.record(cs)
            self._h2d.wait_event(start)
            self._primed = True
        i = self._flip
        self._flip ^= 1
        used = self._used[i]
        if used:
            self._ev_ready[i].synchronize()  # the pinned order buffer of two steps ago has been copied
        self._order_host[i].numpy()[:] = _longest_first_np(context_lens.numpy())
        bufs = self._dev_inputs[i]
        if used:
            self._h2d.wait_event(self._ev_free[i])  # the step two back is done reading set i
        with torch.cuda.stream(self._h2d):
            for d_, h_ in zip(bufs, (q, k_new, v_new, slot_mapping, block_tables, context_lens, self._order_host[i])):
                d_.copy_(h_, non_blocking=True)
            if self.groups is not None:  # the step's groups come from the host too
                self.groups[0].copy_(self._host_groups[0], non_blocking=True)
                self.groups[1].copy_(self._host_groups[1], non_blocking=True)
        self._ev_ready[i].record(self._h2d)
        cs.wait_event(self._ev_ready[i])
        if used:
            cs.wait_event(self._ev_out[i])  # the output copy of two steps ago is done with output i
        with torch.cuda.stream(cs):
            if self._graphs[i] is None:
                dq, dk, dv, ds, dbt, dcl, dord = bufs

                def device_step(i=i):
                    keep = self.out
                    self.out = self._outs[i]
                    try:
                        # the cascade's suffixes keep the batch order: longest first
                        # measured slower there (short suffixes leave little tail to
                        # remove)
                        self.run(dq, dk, dv, ds, dbt, dcl, seq_order=None if self.groups is not None else dord)
                    finally:
                        self.out = keep

                self._graphs[i] = graphed(device_step)
            self._graphs[i]()
        self._ev_free[i].record(cs)
        self._d2h.wait_event(self._ev_free[i])
        with torch.cuda.stream(self._d2h):
            out_host.copy_(self._outs[i], non_blocking=True)
        self._ev_out[i].record(self._d2h)
        self._used[i] = True
        return out_host

    def flush(self, stream=None):
        """Make ``stream`` (default: current) wait for every output copy that
        ``run_host`` queued; the next ``run_host`` starts a new pipeline."""
        cs = stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.current_stream()
        if self._dev_inputs is not None:
            cs.wait_stream(self._d2h)
            cs.wait_stream(self._h2d)
            self._primed = False

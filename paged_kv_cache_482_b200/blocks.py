"""Python binding of the block manager in libpagedkv.so (ctypes; C ABI in
``include/pagedkv_blocks.h``).

Argument marshalling only: the manager's state and every step of it live in
the native library. The single-sequence methods return the C statuses the
way the header defines them; the per-step batch calls raise
:class:`PagedKVError` and hand back numpy arrays ready to copy to the device
(``slot_mapping`` for ``store_kvcache``; ``block_tables`` and
``context_lens`` for ``paged_attention_decode``).
"""

from __future__ import annotations

import ctypes

import numpy as np

from . import pagedkv as _K
from .pagedkv import PKV_OK, PagedKVError

_declared = set()


def _lib():
    L = _K.lib()
    if id(L) not in _declared:
        c = ctypes
        vp, i32, i64 = c.c_void_p, c.c_int, c.c_int64
        L.pkv_bm_create.argtypes = [i64, i32]
        L.pkv_bm_create.restype = vp
        L.pkv_bm_destroy.argtypes = [vp]
        L.pkv_bm_destroy.restype = None
        L.pkv_bm_add_sequence.argtypes = [vp, i64, vp, i32, c.POINTER(i32)]
        L.pkv_bm_append_token.argtypes = [vp, i64, c.c_int32, c.POINTER(i64)]
        L.pkv_bm_free_sequence.argtypes = [vp, i64]
        L.pkv_bm_block_table.argtypes = [vp, i64, vp, i32, c.POINTER(i32)]
        L.pkv_bm_slots.argtypes = [vp, i64, i32, i32, vp]
        L.pkv_bm_num_free_blocks.argtypes = [vp]
        L.pkv_bm_num_free_blocks.restype = i64
        L.pkv_bm_block_refcount.argtypes = [vp, i64, c.POINTER(i32)]
        L.pkv_bm_append_tokens.argtypes = [vp, vp, vp, i32, vp]
        L.pkv_bm_block_tables.argtypes = [vp, vp, i32, vp, i32, vp]
        for n in ("pkv_bm_add_sequence", "pkv_bm_append_token", "pkv_bm_free_sequence", "pkv_bm_block_table",
                  "pkv_bm_slots", "pkv_bm_block_refcount", "pkv_bm_append_tokens", "pkv_bm_block_tables"):
            getattr(L, n).restype = i32
        _declared.add(id(L))
    return L


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _i64(a):
    return np.ascontiguousarray(a, dtype=np.int64)


def _p(a):
    """Address of a contiguous array's data (None when empty). A ctypes view of
    the buffer is the cheapest route for a writable array (a third of the cost
    of ``a.ctypes.data``, which read-only arrays still take)."""
    if not a.size:
        return None
    try:
        return ctypes.addressof(ctypes.c_char.from_buffer(a))
    except (TypeError, ValueError):
        return a.ctypes.data


class BlockManager:
    """Physical blocks of one paged KV pool (``num_blocks`` blocks of
    ``block_size`` tokens), shared between sequences with equal prefixes."""

    def __init__(self, num_blocks: int, block_size: int):
        self._L = _lib()
        self._h = self._L.pkv_bm_create(int(num_blocks), int(block_size))
        if not self._h:
            raise PagedKVError(_K.PKV_ERR_INVALID_ARG, "pkv_bm_create")
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)

    def close(self):
        if getattr(self, "_h", None):
            self._L.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    # ---------------------------------------------- one sequence (statuses)
    def add_sequence(self, seq_id, tokens):
        """(status, number of leading tokens whose KV is already cached)."""
        t = _i32(tokens)
        cached = ctypes.c_int(0)
        st = self._L.pkv_bm_add_sequence(self._h, int(seq_id), _p(t), int(t.size), ctypes.byref(cached))
        return st, cached.value

    def append_token(self, seq_id, token):
        """(status, slot of the new token, -1 on failure)."""
        slot = ctypes.c_int64(-1)
        st = self._L.pkv_bm_append_token(self._h, int(seq_id), int(token), ctypes.byref(slot))
        return st, slot.value if st == PKV_OK else -1

    def free_sequence(self, seq_id):
        return self._L.pkv_bm_free_sequence(self._h, int(seq_id))

    def block_table(self, seq_id):
        """(list of block ids, sequence length); raises for an unknown id."""
        n = ctypes.c_int(0)
        st = self._L.pkv_bm_block_table(self._h, int(seq_id), None, 0, ctypes.byref(n))
        if st != PKV_OK and n.value == 0:
            raise PagedKVError(st, "pkv_bm_block_table")
        nb = -(-n.value // self.block_size)
        row = np.empty(max(nb, 1), np.int32)
        st = self._L.pkv_bm_block_table(self._h, int(seq_id), _p(row), nb, ctypes.byref(n))
        if st != PKV_OK:
            raise PagedKVError(st, "pkv_bm_block_table")
        return row[:nb].tolist(), n.value

    def slots(self, seq_id, start, count):
        out = np.empty(max(int(count), 1), np.int32)
        st = self._L.pkv_bm_slots(self._h, int(seq_id), int(start), int(count), _p(out))
        if st != PKV_OK:
            raise PagedKVError(st, "pkv_bm_slots")
        return out[: int(count)].tolist()

    def num_free(self):
        return int(self._L.pkv_bm_num_free_blocks(self._h))

    def refcount(self, block):
        r = ctypes.c_int(0)
        st = self._L.pkv_bm_block_refcount(self._h, int(block), ctypes.byref(r))
        if st != PKV_OK:
            raise PagedKVError(st, "pkv_bm_block_refcount")
        return r.value

    # ------------------------------------------------- one step (raising)
    def append_tokens(self, seq_ids, tokens, out=None):
        """Append tokens[i] to seq_ids[i] for all i; returns the int32 slots."""
        ids, tok = _i64(seq_ids), _i32(tokens)
        if ids.shape != tok.shape or ids.ndim != 1:
            raise ValueError("seq_ids and tokens must be 1-D of equal length")
        slots = np.empty(ids.size, np.int32) if out is None else out
        st = self._L.pkv_bm_append_tokens(self._h, _p(ids), _p(tok), int(ids.size), _p(slots))
        if st != PKV_OK:
            raise PagedKVError(st, "pkv_bm_append_tokens")
        return slots

    def block_tables(self, seq_ids, max_blocks, tables=None, context_lens=None):
        """([n, max_blocks] int32 tables padded with -1, [n] int32 lengths)."""
        ids = _i64(seq_ids)
        n = ids.size
        if tables is None:
            tables = np.empty((n, int(max_blocks)), np.int32)
        if context_lens is None:
            context_lens = np.empty(n, np.int32)
        assert tables.dtype == np.int32 and tables.flags.c_contiguous and tables.shape == (n, int(max_blocks))
        assert context_lens.dtype == np.int32 and context_lens.shape == (n,)
        st = self._L.pkv_bm_block_tables(self._h, _p(ids), int(n), _p(tables), int(max_blocks), _p(context_lens))
        if st != PKV_OK:
            raise PagedKVError(st, "pkv_bm_block_tables")
        return tables, context_lens

"""Plain-Python reference block manager -- test infrastructure only.

Only ``tests/`` (and nothing in the product) use this module. It restates,
as directly as possible, what the pages say a block manager with prefix
caching does: the KV memory is cut into fixed-size blocks; a request gets the
blocks it needs and gives them back when it ends, so that others can reuse
them ("Nano-vLLM：轻量高效的大模型推理框架", section 三.1 块管理器); requests that
share a prefix reuse its cached KV instead of recomputing it -- hit: reuse the
cached blocks, miss: compute and cache them (same page, section 三.2 (1)
前缀缓存); block tables map logical blocks to physical ones and blocks are
shared within and across requests ("DeepSeek复刻vLLM反超原版", section
"vLLM：大模型推理的加速引擎与挑战").

No hashing here: a full block is identified by the exact tuple of every
token from position 0 through its own last token, so sharing happens exactly
when two prefixes are equal. It also records which tokens each physical
block holds, so tests can read a sequence's token stream back through its
block table.

Readings (the same as the C++ manager's, stated in include/pagedkv_blocks.h):
only full blocks are shared and matching stops at the first miss; free
blocks form a FIFO queue (initially 0..N-1, freed blocks to the back, new
blocks from the front); a freed full block keeps its cache entry until it is
taken again; registering a prefix that is already cached moves the entry to
the new block; a sequence's blocks are freed last block first.
"""

from __future__ import annotations

OK = 0
ERR_INVALID_ARG = 1
ERR_NO_BLOCKS = 3  # PKV_ERR_WORKSPACE


class BlockManagerOracle:
    def __init__(self, num_blocks: int, block_size: int):
        assert num_blocks >= 1 and block_size >= 1
        self.num_blocks = num_blocks
        self.bs = block_size
        self.free = list(range(num_blocks))  # front = index 0
        self.ref = [0] * num_blocks
        self.content = [()] * num_blocks  # tokens each block holds
        self.cached = {}  # full prefix tuple -> block id
        self.key_of = {}  # block id -> its prefix tuple (if cached)
        self.seqs = {}  # seq id -> {"tokens": [...], "table": [...]}

    # -------------------------------------------------------------- helpers
    def _register(self, block: int, prefix: tuple):
        old = self.cached.get(prefix)
        if old is not None and old != block:
            del self.key_of[old]
        if block in self.key_of:
            del self.cached[self.key_of[block]]
        self.cached[prefix] = block
        self.key_of[block] = prefix

    def _take_free(self) -> int:
        b = self.free.pop(0)
        if b in self.key_of:  # its cached content is about to be overwritten
            del self.cached[self.key_of.pop(b)]
        self.content[b] = ()
        return b

    # ------------------------------------------------------------------ API
    def add_sequence(self, seq_id, tokens):
        """Returns (status, cached_token_count)."""
        tokens = [int(t) for t in tokens]
        if seq_id in self.seqs or len(tokens) < 1:
            return ERR_INVALID_ARG, 0
        bs = self.bs
        n_blocks = -(-len(tokens) // bs)
        hits = []
        for i in range(len(tokens) // bs):
            b = self.cached.get(tuple(tokens[: (i + 1) * bs]))
            if b is None:
                break
            hits.append(b)
        free_hits = sum(1 for b in hits if self.ref[b] == 0)
        if len(self.free) - free_hits < n_blocks - len(hits):
            return ERR_NO_BLOCKS, 0
        for b in hits:
            if self.ref[b] == 0:
                self.free.remove(b)
            self.ref[b] += 1
        table = list(hits)
        for i in range(len(hits), n_blocks):
            b = self._take_free()
            self.ref[b] = 1
            self.content[b] = tuple(tokens[i * bs : (i + 1) * bs])
            if len(self.content[b]) == bs:
                self._register(b, tuple(tokens[: (i + 1) * bs]))
            table.append(b)
        self.seqs[seq_id] = {"tokens": tokens, "table": table}
        return OK, len(hits) * bs

    def append_token(self, seq_id, token):
        """Returns (status, slot)."""
        s = self.seqs.get(seq_id)
        if s is None:
            return ERR_INVALID_ARG, -1
        bs = self.bs
        n = len(s["tokens"])
        if n % bs == 0:
            if not self.free:
                return ERR_NO_BLOCKS, -1
            b = self._take_free()
            self.ref[b] = 1
            s["table"].append(b)
        b = s["table"][n // bs]
        self.content[b] = self.content[b] + (int(token),)
        s["tokens"].append(int(token))
        if len(self.content[b]) == bs:
            self._register(b, tuple(s["tokens"]))
        return OK, b * bs + n % bs

    def free_sequence(self, seq_id):
        s = self.seqs.pop(seq_id, None)
        if s is None:
            return ERR_INVALID_ARG
        for b in reversed(s["table"]):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        return OK

    def block_table(self, seq_id):
        s = self.seqs[seq_id]
        return list(s["table"]), len(s["tokens"])

    def slots(self, seq_id, start, count):
        s = self.seqs[seq_id]
        return [s["table"][p // self.bs] * self.bs + p % self.bs for p in range(start, start + count)]

    def num_free(self):
        return len(self.free)

    def refcount(self, block):
        return self.ref[block]

    def tokens_through_table(self, seq_id):
        """The sequence's tokens as read back from the blocks its table names."""
        s = self.seqs[seq_id]
        out = []
        for b in s["table"]:
            out.extend(self.content[b])
        return out[: len(s["tokens"])]

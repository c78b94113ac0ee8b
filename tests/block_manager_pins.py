"""Pins of the reference block manager (oracle/block_manager.py).

Each ``pin_*`` takes a block-manager class with the oracle's interface and
raises AssertionError on a violation of what the pages fix:

* the paged mapping itself ("DeepSeek复刻vLLM反超原版", section "vLLM：大模型推理
  的加速引擎与挑战": block tables map logical blocks to physical ones): a
  simulated physical pool receives every token at the slot the manager gives
  for it, cached prefix tokens are not written again, and every live
  sequence must read its exact token stream back through its block table;
* prefix caching ("Nano-vLLM：轻量高效的大模型推理框架", section 三.2 (1)): equal
  prefixes share their full blocks, the hit length is reported, different
  prefixes share nothing even when later blocks happen to be equal;
* block reuse (same page, section 三.1): freed blocks go back for reuse,
  reference counts equal the number of sequences using a block, and no block
  is lost or handed out twice;
* the stated policy readings (FIFO free queue, freed prefix blocks stay
  cached until taken again, last block freed first, appended blocks become
  shareable once full, failures change nothing).

tests/test_block_manager_oracle.py runs them against the oracle and against
planted mistakes in copies of it.
"""

from __future__ import annotations

import random

OK, ERR_INVALID_ARG, ERR_NO_BLOCKS = 0, 1, 3


class Checked:
    """Drives a manager and checks the pool / refcount invariants after every step."""

    def __init__(self, cls, num_blocks, bs):
        self.m = cls(num_blocks, bs)
        self.nb, self.bs = num_blocks, bs
        self.pool = [None] * (num_blocks * bs)  # token id held by each slot
        self.live = {}  # seq id -> tokens

    def add(self, sid, tokens):
        st, cached = self.m.add_sequence(sid, tokens)
        if st != OK:
            return st, cached
        assert cached % self.bs == 0 and 0 <= cached <= len(tokens)
        for p, s in enumerate(self.m.slots(sid, cached, len(tokens) - cached), start=cached):
            self.pool[s] = tokens[p]
        self.live[sid] = list(tokens)
        self.check()
        return st, cached

    def append(self, sid, tok):
        st, slot = self.m.append_token(sid, tok)
        if st != OK:
            return st, slot
        self.pool[slot] = tok
        self.live[sid].append(tok)
        self.check()
        return st, slot

    def free(self, sid):
        st = self.m.free_sequence(sid)
        if st == OK:
            del self.live[sid]
            self.check()
        return st

    def check(self):
        users = [0] * self.nb
        for sid, toks in self.live.items():
            table, n = self.m.block_table(sid)
            assert n == len(toks), "sequence length"
            assert len(table) == -(-n // self.bs), "one block per started block of tokens"
            assert len(set(table)) == len(table), "a block twice in one table"
            got = [self.pool[table[p // self.bs] * self.bs + p % self.bs] for p in range(n)]
            assert got == toks, f"sequence {sid} does not read back through its table"
            for b in table:
                users[b] += 1
        for b in range(self.nb):
            assert self.m.refcount(b) == users[b], f"refcount of block {b}"
        in_use = sum(1 for u in users if u > 0)
        assert self.m.num_free() + in_use == self.nb, "blocks lost or double-counted"


def _random_trace(cls, seed, nb=48, bs=4, steps=400):
    rng = random.Random(seed)
    c = Checked(cls, nb, bs)
    prompts = [[rng.randrange(50) for _ in range(rng.randrange(1, 14))] for _ in range(4)]
    next_id = 0
    for _ in range(steps):
        op = rng.random()
        if op < 0.35 or not c.live:
            base = rng.choice(prompts)
            toks = base[: rng.randrange(0, len(base) + 1)] + [rng.randrange(50) for _ in range(rng.randrange(0, 7))]
            if not toks:
                toks = [rng.randrange(50)]
            st, _ = c.add(next_id, toks)
            assert st in (OK, ERR_NO_BLOCKS)
            next_id += 1
        elif op < 0.8:
            sid = rng.choice(list(c.live))
            st, _ = c.append(sid, rng.randrange(50))
            assert st in (OK, ERR_NO_BLOCKS)
        else:
            assert c.free(rng.choice(list(c.live))) == OK
    return c


def pin_tables_read_back_their_tokens(cls):
    for seed in range(6):
        _random_trace(cls, seed)


def pin_equal_prefixes_share_full_blocks(cls):
    bs = 4
    c = Checked(cls, 32, bs)
    p = list(range(100, 112))  # three full blocks
    st, cached = c.add(0, p + [1, 2])
    assert st == OK and cached == 0
    st, cached = c.add(1, p + [3])
    assert st == OK and cached == 12, "the three shared blocks are a hit"
    t0, _ = c.m.block_table(0)
    t1, _ = c.m.block_table(1)
    assert t0[:3] == t1[:3] and t0[3] != t1[3]
    # a different first block: nothing is shared, even though blocks 2 and 3 are equal
    q = [999] + p[1:]
    st, cached = c.add(2, q + [1, 2])
    t2, _ = c.m.block_table(2)
    assert cached == 0 and not set(t2) & set(t0), "sharing needs the whole prefix to be equal"
    # a partial block is never shared
    st, cached = c.add(3, [7, 7, 7, 7, 7, 7])
    st, cached = c.add(4, [7, 7, 7, 7, 7, 7])
    t3, _ = c.m.block_table(3)
    t4, _ = c.m.block_table(4)
    assert cached == 4 and t3[0] == t4[0] and t3[1] != t4[1]


def pin_fifo_free_queue(cls):
    c = Checked(cls, 8, 2)
    c.add(0, [1, 2, 3])  # blocks 0, 1
    c.add(1, [4, 5, 6, 7, 8])  # blocks 2, 3, 4
    assert c.m.block_table(0)[0] == [0, 1] and c.m.block_table(1)[0] == [2, 3, 4]
    c.free(0)  # last block first: queue 5 6 7 1 0
    c.add(2, [9, 9, 9, 9, 9, 9, 9])  # four blocks: 5 6 7 1
    assert c.m.block_table(2)[0] == [5, 6, 7, 1]


def pin_freed_prefix_stays_cached_until_taken(cls):
    bs = 4
    c = Checked(cls, 4, bs)
    pre = [1, 2, 3, 4, 5, 6, 7, 8]
    c.add(0, pre + [9, 9, 9, 9])  # three full blocks
    c.free(0)  # queue: tail block, block 2, block 1
    st, cached = c.add(1, [42])  # takes the freed tail block
    assert st == OK and cached == 0
    st, cached = c.add(2, pre + [5])  # the prefix blocks were freed but not taken: a hit
    assert st == OK and cached == 8
    assert c.free(1) == OK and c.free(2) == OK
    # now force every block to be taken again: the prefix is gone
    c.add(3, [50] * 16)
    c.free(3)
    st, cached = c.add(4, pre + [5])
    assert cached == 0, "a block that was taken again no longer holds the prefix"


def pin_matching_stops_at_the_first_miss(cls):
    bs = 4
    c = Checked(cls, 4, bs)
    x, y = [1, 2, 3, 4], [5, 6, 7, 8]
    c.add(0, x + y)  # blocks 0, 1 cache X and XY
    c.add(1, x[:3])  # block 2
    c.append(1, x[3])  # block 2 now holds X too: the entry for X moves to it
    c.free(1)  # queue: 3, 2
    c.add(2, [9] * 8)  # takes 3 and 2: X is no longer cached, XY still is
    c.free(2)
    st, cached = c.add(3, x + y)
    assert st == OK and cached == 0, "a later block cannot hit once an earlier one missed"


def pin_appended_blocks_become_shareable(cls):
    bs = 4
    c = Checked(cls, 16, bs)
    c.add(0, [1, 2, 3])
    st, slot = c.append(0, 4)  # fills block 0
    st, slot = c.append(0, 5)  # starts a new block
    t0, n = c.m.block_table(0)
    assert n == 5 and len(t0) == 2 and slot == t0[1] * bs + 0
    st, cached = c.add(1, [1, 2, 3, 4, 8])
    assert cached == 4 and c.m.block_table(1)[0][0] == t0[0]


def pin_failures_change_nothing(cls):
    c = Checked(cls, 3, 2)
    c.add(0, [1, 2, 3, 4])
    before = (c.m.num_free(), c.m.block_table(0))
    st, _ = c.add(1, [5, 6, 7, 8, 9])  # needs three blocks, one is free
    assert st == ERR_NO_BLOCKS and (c.m.num_free(), c.m.block_table(0)) == before
    assert c.add(0, [1])[0] == ERR_INVALID_ARG, "id in use"
    c.add(2, [5, 6])
    st, _ = c.append(2, 7)  # needs a block, none free
    assert st == ERR_NO_BLOCKS and c.m.block_table(2) == ([c.m.block_table(2)[0][0]], 2)
    assert c.m.free_sequence(9) == ERR_INVALID_ARG
    assert c.m.append_token(9, 1)[0] == ERR_INVALID_ARG
    c.check()


ALL_PINS = [
    pin_tables_read_back_their_tokens,
    pin_equal_prefixes_share_full_blocks,
    pin_fifo_free_queue,
    pin_freed_prefix_stays_cached_until_taken,
    pin_matching_stops_at_the_first_miss,
    pin_appended_blocks_become_shareable,
    pin_failures_change_nothing,
]


def run_all(cls):
    failed = []
    for pin in ALL_PINS:
        try:
            pin(cls)
        except Exception as e:  # noqa: BLE001
            failed.append(f"{pin.__name__}: {type(e).__name__}: {str(e)[:100]}")
    return failed

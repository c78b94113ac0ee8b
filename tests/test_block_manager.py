"""The native block manager (libpagedkv.so, include/pagedkv_blocks.h) on the
host: its pins, and bit-exact agreement with the reference block manager on
random operation traces (every status, cached length, slot, table row,
refcount and free count). No GPU."""

import random

import numpy as np
import pytest

import block_manager_pins as P
from oracle.block_manager import BlockManagerOracle, ERR_INVALID_ARG, ERR_NO_BLOCKS, OK


@pytest.fixture(scope="module")
def BM():
    from paged_kv_cache_482_b200 import build as B

    B.build()
    from paged_kv_cache_482_b200.blocks import BlockManager

    return BlockManager


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(BM, pin):
    pin(BM)


def _oracle_append_batch(o, ids, toks):
    """The batch call's meaning, spelled out with the oracle's single steps."""
    if len(set(ids)) != len(ids) or any(i not in o.seqs for i in ids):
        return ERR_INVALID_ARG, None
    need = sum(1 for i in ids if len(o.seqs[i]["tokens"]) % o.bs == 0)
    if need > o.num_free():
        return ERR_NO_BLOCKS, None
    out = []
    for i, t in zip(ids, toks):
        st, s = o.append_token(i, t)
        assert st == OK
        out.append(s)
    return OK, out


def _compare_state(o, m, nb):
    assert o.num_free() == m.num_free()
    for b in range(nb):
        assert o.refcount(b) == m.refcount(b), b
    ids = sorted(o.seqs)
    for i in ids:
        assert o.block_table(i) == m.block_table(i), i
    if ids:
        maxb = max(len(o.block_table(i)[0]) for i in ids) + 1
        tabs, lens = m.block_tables(ids, maxb)
        for r, i in enumerate(ids):
            t, n = o.block_table(i)
            assert lens[r] == n and tabs[r, : len(t)].tolist() == t and (tabs[r, len(t):] == -1).all()


def _trace(BM, seed, nb, bs, steps, vocab, n_prompts, check_every):
    rng = random.Random(seed)
    o, m = BlockManagerOracle(nb, bs), BM(nb, bs)
    prompts = [[rng.randrange(vocab) for _ in range(rng.randrange(1, 6 * bs + 3))] for _ in range(n_prompts)]
    next_id = 0
    counts = {"hit": 0, "nospace": 0}
    for step in range(steps):
        op = rng.random()
        if op < 0.3 or not o.seqs:
            base = rng.choice(prompts)
            toks = base[: rng.randrange(0, len(base) + 1)] + [rng.randrange(vocab) for _ in range(rng.randrange(0, 2 * bs))]
            toks = toks or [rng.randrange(vocab)]
            sid = next_id if rng.random() > 0.03 or not o.seqs else rng.choice(list(o.seqs))  # sometimes an id in use
            a, b = o.add_sequence(sid, toks), m.add_sequence(sid, toks)
            assert a == b, (step, "add", a, b)
            if a[0] == OK:
                next_id += 1
                counts["hit"] += a[1] > 0
                assert o.slots(sid, 0, len(toks)) == m.slots(sid, 0, len(toks))
            counts["nospace"] += a[0] == ERR_NO_BLOCKS
        elif op < 0.55:
            sid = rng.choice(list(o.seqs)) if rng.random() > 0.02 else 10**9
            t = rng.randrange(vocab)
            assert o.append_token(sid, t) == m.append_token(sid, t), (step, "append")
        elif op < 0.75:
            live = list(o.seqs)
            ids = rng.sample(live, rng.randrange(1, len(live) + 1))
            if rng.random() < 0.05:
                ids.append(ids[0])  # a repeated id: refused as a whole
            toks = [rng.randrange(vocab) for _ in ids]
            st, want = _oracle_append_batch(o, ids, toks)
            try:
                got = m.append_tokens(ids, toks).tolist()
                gst = OK
            except Exception as e:  # noqa: BLE001
                gst, got = e.status, None
            assert (st, want) == (gst, got), (step, "batch", st, gst)
        else:
            sid = rng.choice(list(o.seqs)) if rng.random() > 0.02 else -5
            assert o.free_sequence(sid) == m.free_sequence(sid), (step, "free")
        if step % check_every == 0:
            _compare_state(o, m, nb)
    _compare_state(o, m, nb)
    return counts


@pytest.mark.parametrize("seed,nb,bs,steps,vocab", [
    (0, 64, 4, 3000, 8),      # tiny vocabulary: many equal blocks
    (1, 64, 16, 3000, 50),
    (2, 300, 1, 3000, 4),     # every token a full block: heavy table churn
    (3, 40, 2, 3000, 3),      # tight pool: frequent out-of-blocks
    (4, 2048, 8, 6000, 1000),
])
def test_random_traces_match_the_oracle(BM, seed, nb, bs, steps, vocab):
    c = _trace(BM, seed, nb, bs, steps, vocab, n_prompts=6, check_every=97)
    assert c["hit"] > 0


def test_prefix_hits_at_scale(BM):
    """A pool of Qwen3-8B-decode size with block size 256: 64 requests over 4
    shared 3000-token prompts, then a few hundred decode steps in batches."""
    rng = np.random.default_rng(7)
    nb, bs = 2048, 256
    o, m = BlockManagerOracle(nb, bs), BM(nb, bs)
    prompts = [rng.integers(0, 150000, 3000).tolist() for _ in range(4)]
    for sid in range(64):
        toks = prompts[sid % 4][: 1024 + 256 * (sid % 8)] + rng.integers(0, 150000, sid % 300).tolist()
        assert o.add_sequence(sid, toks) == m.add_sequence(sid, toks)
    ids = list(range(64))
    for _ in range(300):
        toks = rng.integers(0, 150000, 64).tolist()
        st, want = _oracle_append_batch(o, ids, toks)
        assert st == OK and m.append_tokens(ids, toks).tolist() == want
    _compare_state(o, m, nb)
    assert o.refcount(o.block_table(0)[0][0]) == 16  # the first block of prompt 0 is shared 16 ways


def test_host_checks(BM):
    from paged_kv_cache_482_b200 import pagedkv as K
    from paged_kv_cache_482_b200.blocks import _lib

    L = _lib()
    assert not L.pkv_bm_create(0, 16) and not L.pkv_bm_create(4, 0) and not L.pkv_bm_create(2**40, 16)
    assert not L.pkv_bm_create(2**27, 16)  # slots would overflow int32
    m = BM(8, 4)
    assert m.add_sequence(0, []) == (K.PKV_ERR_INVALID_ARG, 0)
    assert m.add_sequence(0, list(range(33)))[0] == K.PKV_ERR_WORKSPACE  # more blocks than the pool has
    assert m.add_sequence(0, [1, 2, 3]) == (OK, 0)
    with pytest.raises(K.PagedKVError):
        m.slots(0, 2, 5)
    with pytest.raises(K.PagedKVError):
        m.refcount(8)
    with pytest.raises(K.PagedKVError):
        m.block_tables([0, 1], 4)
    with pytest.raises(K.PagedKVError):
        m.block_tables([0], 0)  # one block does not fit in zero
    assert m.slots(0, 3, 0) == []
    assert m.append_tokens([], []).size == 0
    assert m.num_free() == 7
    m.close()
    m.close()

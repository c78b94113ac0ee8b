"""The block manager's table of live sequences under churn: thousands of
adds, appends and frees over scattered 64-bit ids (negative, huge, and
multiples of large powers of two that collide in a hash table's low bits),
checked after every step against a Python dict of ids and lengths. Block
contents are checked against the reference manager by test_block_manager."""

import numpy as np

from paged_kv_cache_482_b200 import pagedkv as K
from paged_kv_cache_482_b200.blocks import BlockManager


def _ids(rng, n):
    base = [int(x) for x in rng.integers(-(2**62), 2**62, n // 2)]
    coll = [int(k) << s for k, s in zip(rng.integers(1, 1000, n // 2), rng.integers(6, 40, n // 2))]
    out = list(dict.fromkeys(base + coll + [0, -1, 2**63 - 1, -(2**63)]))
    rng.shuffle(out)
    return out


def test_churn_matches_a_dict():
    rng = np.random.default_rng(5)
    bs, nb = 4, 4096
    m = BlockManager(nb, bs)
    ids = _ids(rng, 3000)
    live = {}
    for step in range(20000):
        sid = ids[int(rng.integers(0, len(ids)))]
        op = int(rng.integers(0, 4))
        if op == 0:
            toks = rng.integers(0, 3, int(rng.integers(1, 10)))  # a small vocabulary: shared prefixes
            st, _ = m.add_sequence(sid, toks)
            if sid in live:
                assert st == K.PKV_ERR_INVALID_ARG
            elif st == K.PKV_OK:
                live[sid] = len(toks)
            else:
                assert st == K.PKV_ERR_WORKSPACE
        elif op == 1:
            st, slot = m.append_token(sid, int(rng.integers(0, 3)))
            if sid not in live:
                assert st == K.PKV_ERR_INVALID_ARG
            elif st == K.PKV_OK:
                live[sid] += 1
                assert 0 <= slot < nb * bs
            else:
                assert st == K.PKV_ERR_WORKSPACE
        elif op == 2:
            st = m.free_sequence(sid)
            assert (st == K.PKV_OK) == (sid in live)
            live.pop(sid, None)
        else:
            if sid in live:
                table, n = m.block_table(sid)
                assert n == live[sid] and len(table) == -(-n // bs)
            else:
                try:
                    m.block_table(sid)
                    raise AssertionError("unknown id answered")
                except K.PagedKVError:
                    pass
    # every live sequence at once, in the batch calls
    keys = np.array(list(live), dtype=np.int64)
    maxb = max(-(-n // bs) for n in live.values())
    tables, lens = m.block_tables(keys, maxb)
    assert lens.tolist() == [live[int(k)] for k in keys]
    for k in keys:
        assert m.free_sequence(int(k)) == K.PKV_OK
    assert m.num_free() == nb


def _home(sid: int, mask: int) -> int:
    """Home slot of an id in the manager's live-sequence table (a multiply by
    the 64-bit golden ratio, an xor-shift, a mask), restated here only to pick
    ids that collide on purpose."""
    h = (sid * 0x9E3779B97F4A7C15) & (2**64 - 1)
    return (h ^ (h >> 29)) & mask


def _ids_with_home(slot: int, n: int, mask: int = 63, start: int = 1):
    out, x = [], start
    while len(out) < n:
        if _home(x, mask) == slot:
            out.append(x)
        x += 1
    return out


def test_probe_runs_that_wrap_and_erase_from_their_middle():
    """With at most 32 live sequences the table has 64 slots. Ids whose home
    slots are 60, 62, 63, 0 and 1 build one long probe run that wraps past the
    end of the table; erasing from its middle must shift the right entries
    back (backward-shift deletion) so that every remaining id is still found,
    and an erased id is gone."""
    groups = [_ids_with_home(60, 10), _ids_with_home(62, 4), _ids_with_home(63, 3), _ids_with_home(0, 4),
              _ids_with_home(1, 3)]
    ids = [i for g in groups for i in g]
    assert len(set(ids)) == len(ids) <= 32
    rng = np.random.default_rng(11)
    m = BlockManager(512, 4)
    live = {}

    def check_all():
        for sid in ids:
            if sid in live:
                table, n = m.block_table(sid)
                assert n == live[sid]
            else:
                try:
                    m.block_table(sid)
                    raise AssertionError(f"erased id {sid} still found")
                except K.PagedKVError:
                    pass

    # interleaved inserts: the run starting at 60 wraps and absorbs the others
    order = [g[i] for i in range(10) for g in groups if i < len(g)]
    for k, sid in enumerate(order):
        st, _ = m.add_sequence(sid, np.array([k % 3] * (1 + k % 5)))
        assert st == K.PKV_OK
        live[sid] = 1 + k % 5
        check_all()
    # erase from the middle of the run, then churn
    for sid in (groups[0][4], groups[3][1], groups[0][0], groups[2][1], groups[1][3]):
        assert m.free_sequence(sid) == K.PKV_OK
        live.pop(sid)
        check_all()
    for step in range(3000):
        sid = ids[int(rng.integers(0, len(ids)))]
        if sid in live:
            assert m.free_sequence(sid) == K.PKV_OK
            live.pop(sid)
        else:
            n = int(rng.integers(1, 6))
            st, _ = m.add_sequence(sid, rng.integers(0, 3, n))
            assert st == K.PKV_OK
            live[sid] = n
        check_all()

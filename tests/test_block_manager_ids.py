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

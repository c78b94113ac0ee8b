"""The CPU oracle against its pins (no GPU)."""

import pytest

import oracle as O
import oracle_pins as P


@pytest.fixture(scope="module")
def lib():
    return O.load()


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(lib, pin):
    pin(lib)


def test_threads_do_not_change_results(lib):
    from paged_kv_cache_482_b200 import workloads as W

    wl = W.generate(P.cfg(num_seqs=9, ctx_lo=1, ctx_hi=60, cache_dtype=W.CACHE_FP8), 21)
    out1, _, _, st1 = O.run_workload(wl, num_threads=1, lib=lib)
    out4, _, _, st4 = O.run_workload(wl, num_threads=4, lib=lib)
    assert st1 == st4 == O.ORC_OK
    assert (out1 == out4).all()


def test_sampled_rebuild_matches_full(lib):
    """Rebuilding only a few sequences' blocks gives those sequences' full result."""
    from paged_kv_cache_482_b200 import workloads as W

    for c in (P.cfg(num_seqs=6, ctx_lo=1, ctx_hi=30), P.cfg(num_seqs=5, prefix_tokens=8, ctx_lo=0, ctx_hi=6)):
        wl = W.generate(c, 22)
        full, kp, vp, st = O.run_workload(wl, lib=lib)
        ids = [4, 1]
        part, kp2, vp2, st2 = O.run_workload(wl, seq_ids=ids, lib=lib)
        assert st == st2 == O.ORC_OK
        assert (part == full[ids]).all()
        for i in ids:
            for b in wl.block_tables[i].tolist():
                if b >= 0:
                    assert (kp2[b] == kp[b]).all() and (vp2[b] == vp[b]).all()

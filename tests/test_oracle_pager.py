"""Pins of the oracle's paged-cache bookkeeping (oracle/pager.py) against the
page's own unit tests (combs-models 0.2.2, src/kv.rs; restated in
tests/golden/pager_scripts.txt) and invariants any correct allocator keeps."""
import random

import pytest

from oracle.pager import OraclePager, PagerError, num_pages_for
from pager_scripts import load_scripts, run_script

CASES = load_scripts()


@pytest.mark.parametrize("name", list(CASES))
def test_page_tests(name):
    run_script(lambda n, ps, w: OraclePager(n, ps, 1, n, w), num_pages_for, name, CASES[name],
               PagerError)


def test_failed_append_changes_nothing():
    p = OraclePager(3, 16, 2, 8)
    p.append(0, 40)                      # 3 pages
    before = (p.table(), list(p.lens), list(p.free))
    with pytest.raises(PagerError):
        p.append(1, 1)                   # no page left
    with pytest.raises(PagerError):
        p.append(0, 16 * 8)              # beyond the table
    assert (p.table(), list(p.lens), list(p.free)) == before


def test_random_operations_keep_pages_disjoint_and_counted():
    rng = random.Random(7)
    npg, ps, S, mp = 40, 16, 5, 12
    p = OraclePager(npg, ps, S, mp)
    for _ in range(3000):
        s = rng.randrange(S)
        r = rng.random()
        if r < 0.55:
            try:
                pos = p.append(s, rng.randrange(0, 40))
                assert pos <= p.seq_len(s)
            except PagerError:
                pass
        elif r < 0.9:
            n = rng.randrange(0, 50)
            before = p.seq_len(s)
            assert p.popn(s, n) == min(n, before)
        elif r < 0.97:
            p.release(s)
        else:
            p.reset()
        used = [pg for t in p.tables for pg in t]
        # every page is either free or in exactly one table
        assert sorted(used + p.free) == list(range(npg))
        for q in range(S):
            assert p.pages_used(q) == -(-p.seq_len(q) // ps)

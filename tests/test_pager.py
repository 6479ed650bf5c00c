"""The library's native paged-cache bookkeeping (kvq_pager_*, host code, no
GPU needed) against the page's own unit tests and, operation by operation,
against the oracle's model (oracle/pager.py): same page ids in the same
order, same lengths, same free counts, same refusals."""
import random

import pytest
import torch

import oracle.pager as op
from pager_scripts import load_scripts, run_script

CASES = load_scripts()


def kvq():
    import decode_attention_kvq_b200 as m
    return m


def _native(n, ps, w, seqs=1, max_pages=None):
    return kvq().Pager(n, seqs, max_pages or n, ps, windows=w)


class _NativeView:
    """OraclePager-shaped view of the native pager for the script runner."""

    def __init__(self, p):
        self.p = p

    def append(self, s, n):
        return self.p.append(s, n)

    def popn(self, s, n):
        return self.p.popn(s, n)

    def reset(self):
        self.p.reset()

    def num_free(self):
        return self.p.num_free()

    def pages_used(self, s):
        return self.p.pages_used(s)

    def seq_len(self, s):
        return self.p.seq_len(s)

    def table(self):
        return self.p.table().tolist()


@pytest.mark.parametrize("name", list(CASES))
def test_page_tests_native(name):
    run_script(lambda n, ps, w: _NativeView(_native(n, ps, w)), op.num_pages_for, name,
               CASES[name], kvq().KvqError)


@pytest.mark.parametrize("seed,windows", [(1, ()), (2, ()), (3, (40,)), (4, (8, 200))])
def test_native_matches_oracle_on_random_operations(seed, windows):
    m = kvq()
    rng = random.Random(seed)
    npg, ps, S, mp = 37, 16, 6, 10
    nat = m.Pager(npg, S, mp, ps, windows=windows)
    ora = op.OraclePager(npg, ps, S, mp, windows)
    for step in range(4000):
        s = rng.randrange(S)
        r = rng.random()
        if r < 0.5:
            n = rng.randrange(0, 45)
            try:
                want = ora.append(s, n)
            except op.PagerError:
                want = None
            if want is None:
                with pytest.raises(m.KvqError) as ei:
                    nat.append(s, n)
                assert ei.value.status in (1, 6)
            else:
                assert nat.append(s, n) == want
        elif r < 0.85:
            n = rng.randrange(0, 60)
            assert nat.popn(s, n) == ora.popn(s, n), f"step {step}"
        elif r < 0.97:
            nat.release(s)
            ora.release(s)
        else:
            nat.reset()
            ora.reset()
        assert nat.table().tolist() == ora.table(), f"step {step}"
        assert nat.lens().tolist() == ora.lens
        assert nat.num_free() == ora.num_free()


def test_out_of_pages_status_and_no_change():
    m = kvq()
    p = m.Pager(3, 2, 8, 16)
    assert p.append(0, 40) == 0
    before = p.table().clone(), p.lens().clone(), p.num_free()
    with pytest.raises(m.KvqError) as ei:
        p.append(1, 1)
    assert ei.value.status == 6                                   # KVQ_ERR_OUT_OF_PAGES
    with pytest.raises(m.KvqError) as ei:
        p.append(0, 16 * 8)                                       # beyond the table
    assert ei.value.status == 1
    assert torch.equal(p.table(), before[0]) and torch.equal(p.lens(), before[1])
    assert p.num_free() == before[2]


def test_bad_arguments():
    m = kvq()
    with pytest.raises(ValueError):
        m.Pager(0, 1, 1)
    with pytest.raises(m.KvqError):
        m.Pager(4, 1, 4, windows=(1,))                            # a window must be >= 2
    assert m.lib.kvq_pager_bytes(4, 0, 4, 0) == 0
    p = m.Pager(4, 2, 4)
    assert p.popn(5, 3) == 0 and p.pages_used(-1) == 0
    with pytest.raises(m.KvqError):
        p.append(2, 1)                                            # no sequence 2

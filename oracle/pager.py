"""Plain model of the paged cache's host bookkeeping: free-page allocator,
per-sequence page tables, append (grow), rollback (popn), release, reset,
and the rollback rule of sliding-window layers.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): the tests compare
the library's native bookkeeping with this model, operation by operation.

What it follows: combs-models 0.2.2, src/kv.rs --
 * PageAllocator: a stack of free physical page ids, built reversed so that
   page 0 is handed out first; alloc pops, free pushes (LIFO reuse), reset
   rebuilds the full stack.
 * CacheConfig::num_pages: ceil(max_seq_len / page_size).
 * PagedKVCache::ensure_pages: the page table grows, one page from the
   allocator at a time, until it covers ceil(total / page_size) pages.
 * PagedKVCache::popn: n is clamped to the length; a cache with a sliding
   layer of window w refuses (returns 0, nothing changes) once its length
   exceeds w - 1 (tokens were evicted); otherwise the length drops by n and
   trailing pages beyond ceil(len / page_size) are popped from the table
   and pushed back onto the free stack, last page first.
 * PagedKVCache::reset: every page free, length 0.
The page's cache holds one sequence and notes that per-sequence tables can
be added; here every sequence has its own table and length and all share
one allocator.  Where the page panics (allocator exhausted, capacity
exceeded) the model raises and leaves its state unchanged.
"""
from __future__ import annotations


class PagerError(Exception):
    """An append the arena or the table cannot hold (state unchanged)."""


class OraclePager:
    def __init__(self, num_pages: int, page_size: int, max_seqs: int, max_pages: int,
                 windows=()):
        self.num_pages = num_pages
        self.page_size = page_size
        self.max_seqs = max_seqs
        self.max_pages = max_pages
        self.windows = [int(w) for w in windows]
        self.reset()

    # PageAllocator
    def reset(self):
        self.free = list(range(self.num_pages))[::-1]   # page 0 on top
        self.tables = [[] for _ in range(self.max_seqs)]
        self.lens = [0] * self.max_seqs

    def num_free(self) -> int:
        return len(self.free)

    def pages_used(self, s: int) -> int:
        return len(self.tables[s])

    def seq_len(self, s: int) -> int:
        return self.lens[s]

    # PagedKVCache::ensure_pages, with the length advanced by n
    def append(self, s: int, n: int) -> int:
        total = self.lens[s] + n
        need = -(-total // self.page_size)
        if need > self.max_pages:
            raise PagerError("sequence capacity exceeded")
        grow = need - len(self.tables[s])
        if grow > len(self.free):
            raise PagerError("page allocator exhausted")
        pos = self.lens[s]
        while len(self.tables[s]) < need:
            self.tables[s].append(self.free.pop())
        self.lens[s] = total
        return pos

    # PagedKVCache::popn
    def popn(self, s: int, n: int) -> int:
        n = min(n, self.lens[s])
        if n == 0:
            return 0
        for w in self.windows:
            if self.lens[s] > w - 1:
                return 0
        self.lens[s] -= n
        keep = -(-self.lens[s] // self.page_size)
        while len(self.tables[s]) > keep:
            self.free.append(self.tables[s].pop())
        return n

    def release(self, s: int):
        """Sequence s empty, its pages freed (a popn of everything that the
        sliding-layer rule does not apply to: the sequence is finished)."""
        while self.tables[s]:
            self.free.append(self.tables[s].pop())
        self.lens[s] = 0

    def table(self):
        """int32 rows [max_seqs][max_pages] padded with -1."""
        return [t + [-1] * (self.max_pages - len(t)) for t in self.tables]


def num_pages_for(max_seq_len: int, page_size: int) -> int:
    """CacheConfig::num_pages: ceil(max_seq_len / page_size)."""
    return -(-max_seq_len // page_size)

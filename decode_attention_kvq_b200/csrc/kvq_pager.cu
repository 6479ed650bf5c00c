// kvq_pager.cu -- host bookkeeping around the paged cache: the free-page
// allocator shared by all sequences, one page table and length per sequence,
// append (grow), rollback (popn), release and reset, and the rollback rule of
// sliding-window layers.  Host code only: nothing here touches a GPU.  The
// page tables it keeps are the int32 [max_seqs, max_pages] table that
// kvq_append_paged and the decode / chunk attention read once the caller has
// copied it to the device.
//
// Method: combs-models 0.2.2, src/kv.rs -- PageAllocator (a stack of free
// page ids built reversed, so page 0 is handed out first; pages come back
// last-in first-out), PagedKVCache::ensure_pages (grow the table a page at a
// time until it covers the length), PagedKVCache::popn (clamp to the length,
// refuse once a sliding layer has evicted, free trailing pages that no longer
// hold a token) and PagedKVCache::reset.  The page's cache holds one sequence;
// here every sequence has its own table and length, all drawing on one
// allocator.  Where the page panics (allocator exhausted, capacity exceeded)
// these calls return an error and change nothing.
//
// Memory: the pager lives in caller-provided host memory (kvq_pager_bytes),
// laid out as the header, the free stack int32[num_pages], the tables
// int32[max_seqs * max_pages], the lengths int32[max_seqs] and the windows
// int32[num_windows].
#include <stdint.h>
#include <string.h>

#include "kvq.h"

struct kvq_pager {
    int32_t num_pages, page_size, max_seqs, max_pages, num_windows;
    int32_t n_free;            // entries on the free stack (its top is free[n_free - 1])
    int32_t* free;             // [num_pages]
    int32_t* table;            // [max_seqs * max_pages], -1 past each sequence's pages
    int32_t* lens;             // [max_seqs]
    int32_t* windows;          // [num_windows]
};

namespace {

size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

bool sizes_ok(int num_pages, int max_seqs, int max_pages, int num_windows) {
    return num_pages >= 1 && max_seqs >= 1 && max_pages >= 1 && num_windows >= 0 &&
           static_cast<int64_t>(max_seqs) * max_pages < (int64_t{1} << 31);
}

int32_t pages_for(int64_t len, int page_size) {
    return static_cast<int32_t>((len + page_size - 1) / page_size);
}

int32_t used(const kvq_pager* p, int s) { return pages_for(p->lens[s], p->page_size); }

}  // namespace

extern "C" {

size_t kvq_pager_bytes(int num_pages, int max_seqs, int max_pages, int num_windows) {
    if (!sizes_ok(num_pages, max_seqs, max_pages, num_windows)) return 0;
    return align16(sizeof(kvq_pager)) +
           4 * (static_cast<size_t>(num_pages) + static_cast<size_t>(max_seqs) * max_pages +
                max_seqs + num_windows);
}

void kvq_pager_reset(kvq_pager* p) {
    if (!p) return;
    for (int i = 0; i < p->num_pages; ++i) p->free[i] = p->num_pages - 1 - i;   // page 0 on top
    p->n_free = p->num_pages;
    for (int64_t i = 0; i < static_cast<int64_t>(p->max_seqs) * p->max_pages; ++i) p->table[i] = -1;
    for (int s = 0; s < p->max_seqs; ++s) p->lens[s] = 0;
}

kvq_status kvq_pager_init(void* mem, size_t bytes, int num_pages, int page_size, int max_seqs,
                          int max_pages, const int32_t* windows, int num_windows,
                          kvq_pager** out) {
    if (!mem || !out || page_size < 1 || !sizes_ok(num_pages, max_seqs, max_pages, num_windows))
        return KVQ_ERR_INVALID_ARG;
    if (num_windows > 0 && !windows) return KVQ_ERR_INVALID_ARG;
    if (static_cast<int64_t>(max_pages) * page_size >= (int64_t{1} << 31)) return KVQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(mem) % 16 != 0) return KVQ_ERR_INVALID_ARG;
    if (bytes < kvq_pager_bytes(num_pages, max_seqs, max_pages, num_windows))
        return KVQ_ERR_INVALID_ARG;
    for (int i = 0; i < num_windows; ++i)
        if (windows[i] < 2) return KVQ_ERR_INVALID_ARG;   // a window of 1 keeps no past
    uint8_t* base = static_cast<uint8_t*>(mem);
    kvq_pager* p = reinterpret_cast<kvq_pager*>(base);
    int32_t* arr = reinterpret_cast<int32_t*>(base + align16(sizeof(kvq_pager)));
    p->num_pages = num_pages;
    p->page_size = page_size;
    p->max_seqs = max_seqs;
    p->max_pages = max_pages;
    p->num_windows = num_windows;
    p->free = arr;
    p->table = p->free + num_pages;
    p->lens = p->table + static_cast<int64_t>(max_seqs) * max_pages;
    p->windows = p->lens + max_seqs;
    if (num_windows > 0) memcpy(p->windows, windows, sizeof(int32_t) * num_windows);
    kvq_pager_reset(p);
    *out = p;
    return KVQ_OK;
}

kvq_status kvq_pager_append(kvq_pager* p, int seq, int64_t n, int64_t* pos) {
    if (!p || seq < 0 || seq >= p->max_seqs || n < 0) return KVQ_ERR_INVALID_ARG;
    const int64_t total = static_cast<int64_t>(p->lens[seq]) + n;
    if (total > static_cast<int64_t>(p->max_pages) * p->page_size) return KVQ_ERR_INVALID_ARG;
    const int32_t need = pages_for(total, p->page_size);
    const int32_t have = used(p, seq);
    if (need - have > p->n_free) return KVQ_ERR_OUT_OF_PAGES;
    int32_t* row = p->table + static_cast<int64_t>(seq) * p->max_pages;
    for (int32_t i = have; i < need; ++i) row[i] = p->free[--p->n_free];
    if (pos) *pos = p->lens[seq];
    p->lens[seq] = static_cast<int32_t>(total);
    return KVQ_OK;
}

int64_t kvq_pager_popn(kvq_pager* p, int seq, int64_t n) {
    if (!p || seq < 0 || seq >= p->max_seqs || n <= 0) return 0;
    if (n > p->lens[seq]) n = p->lens[seq];
    if (n == 0) return 0;
    // a sliding layer that already evicted cannot give back the tokens a
    // rollback would re-expose: the whole rollback is refused
    for (int i = 0; i < p->num_windows; ++i)
        if (p->lens[seq] > p->windows[i] - 1) return 0;
    const int32_t had = used(p, seq);
    p->lens[seq] -= static_cast<int32_t>(n);
    const int32_t keep = used(p, seq);
    int32_t* row = p->table + static_cast<int64_t>(seq) * p->max_pages;
    for (int32_t i = had - 1; i >= keep; --i) {   // last page first back onto the stack
        p->free[p->n_free++] = row[i];
        row[i] = -1;
    }
    return n;
}

kvq_status kvq_pager_release(kvq_pager* p, int seq) {
    if (!p || seq < 0 || seq >= p->max_seqs) return KVQ_ERR_INVALID_ARG;
    int32_t* row = p->table + static_cast<int64_t>(seq) * p->max_pages;
    for (int32_t i = used(p, seq) - 1; i >= 0; --i) {
        p->free[p->n_free++] = row[i];
        row[i] = -1;
    }
    p->lens[seq] = 0;
    return KVQ_OK;
}

int kvq_pager_free_pages(const kvq_pager* p) { return p ? p->n_free : 0; }

int kvq_pager_pages_used(const kvq_pager* p, int seq) {
    if (!p || seq < 0 || seq >= p->max_seqs) return 0;
    return used(p, seq);
}

int64_t kvq_pager_seq_len(const kvq_pager* p, int seq) {
    if (!p || seq < 0 || seq >= p->max_seqs) return 0;
    return p->lens[seq];
}

const int32_t* kvq_pager_table(const kvq_pager* p) { return p ? p->table : nullptr; }

const int32_t* kvq_pager_lens(const kvq_pager* p) { return p ? p->lens : nullptr; }

}  // extern "C"

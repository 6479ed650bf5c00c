"""GPU parity: kvq_window_attn (sliding-window attention on the INT8 cache,
decode steps and chunks) against the oracle's fp64 window attention over the
same dequantized cache (max-abs 2e-3, relative-L2 1e-3): windows smaller and
larger than the sequence, at and off the 16-token alignment, both scale
modes, both layouts, one item per CTA and blocks of items, forced splits,
empty and long sequences; and the ring store of a sliding layer decoded with
kvq_decode_attn."""
import random

import pytest
import torch

import oracle
from kvq_testutil import (ContigCache, PagedCache, assert_attn_close, bf16_randn, f32_scale,
                          kvq)

pytestmark = pytest.mark.gpu


def _contig(B, Hk, D, mode, lens, seed):
    S = max(max(lens), 1)
    c = ContigCache(B, Hk, S, D, mode)
    L = max(lens)
    if L > 0:
        k = bf16_randn((B, Hk, L, D), seed)
        v = bf16_randn((B, Hk, L, D), seed + 1)
        assert c.append(k, v, torch.zeros(B, dtype=torch.int32)) == 0
    return c


def _window_ref(c, q, sl, w, paged=False):
    if paged:
        return oracle.window_attn(q, c.ok, c.ov, c.oks, c.ovs, sl, w, f32_scale(q.shape[-1]),
                                  c.mode, page_size=16, table=c.table_cpu)
    return oracle.window_attn(q, c.ok, c.ov, c.oks, c.ovs, sl, w, f32_scale(q.shape[-1]), c.mode)


def _window(c, q, sl, hint, w, paged=False, **kw):
    m = kvq()
    extra = dict(page_table=c.table, page_size=16) if paged else {}
    return m.kvq_window_attn(q.cuda(), c.k, c.v, c.ks, c.vs, sl.cuda(), hint, w,
                             mode=c.mode, attn_scale=f32_scale(q.shape[-1]), err=c.err,
                             **extra, **kw)


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("w", [1, 5, 16, 17, 100, 5000])
def test_window_decode_contig(mode, D, w):
    B, Hk, G = 3, 2, 4
    lens = [1, 130, 3001]
    c = _contig(B, Hk, D, mode, lens, seed=w + D)
    q = bf16_randn((B, Hk * G, D), seed=w)
    sl = torch.tensor(lens, dtype=torch.int32)
    ref = _window_ref(c, q, sl, w)
    for ns in (0, 1, 3):
        out = _window(c, q, sl, max(lens), w, num_splits=ns)
        assert_attn_close(out, ref, f"w={w} D={D} {mode} ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("G,T,w", [(4, 2, 3), (4, 4, 7), (2, 8, 16), (1, 16, 40), (8, 2, 1)])
def test_window_chunk_contig(G, T, w):
    B, Hk, D = 3, 2, 128
    lens = [T, 90, 1500]
    c = _contig(B, Hk, D, "per_token", lens, seed=G * 7 + T)
    q = bf16_randn((B, Hk * G, T, D), seed=T + w)
    sl = torch.tensor(lens, dtype=torch.int32)
    ref = _window_ref(c, q, sl, w)
    for ns in (0, 2):
        assert_attn_close(_window(c, q, sl, max(lens), w, num_splits=ns), ref,
                          f"G={G} T={T} w={w} ns={ns}")


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_window_many_units_blocks_of_items(mode):
    rnd = random.Random(3)
    B, Hk, G, D = 48, 4, 4, 64
    lens = [rnd.choice([0, 1, 15, 16, 17, 300, 1024, 4000]) for _ in range(B)]
    c = _contig(B, Hk, D, mode, lens, seed=5)
    q = bf16_randn((B, Hk * G, D), seed=6)
    sl = torch.tensor(lens, dtype=torch.int32)
    for w in (33, 700):
        assert_attn_close(_window(c, q, sl, max(lens), w), _window_ref(c, q, sl, w),
                          f"many units w={w} {mode}")


@pytest.mark.parametrize("T", [1, 4])
def test_window_paged(T):
    B, Hk, G, D = 3, 2, 4, 128
    lens = [T, 77, 1000]
    need = [(L + 15) // 16 for L in lens]
    num_pages = sum(need) + 3
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(8)).to(torch.int32)
    table = torch.full((B, max(need)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    c = PagedCache(num_pages, Hk, D, "per_token", table)
    for b, L in enumerate(lens):
        assert c.append(bf16_randn((1, Hk, L, D), 20 + b), bf16_randn((1, Hk, L, D), 30 + b),
                        torch.zeros(1, dtype=torch.int32), rows=[b]) == 0
    shape = (B, Hk * G, D) if T == 1 else (B, Hk * G, T, D)
    q = bf16_randn(shape, seed=40 + T)
    sl = torch.tensor(lens, dtype=torch.int32)
    for w in (9, 48, 2000):
        for ns in (0, 3):
            assert_attn_close(_window(c, q, sl, max(lens), w, paged=True, num_splits=ns),
                              _window_ref(c, q, sl, w, paged=True), f"paged T={T} w={w}")


def test_window_long_sequence_small_window():
    """A 100k-token sequence with a 64-token window: only the window is
    walked, from a 16-aligned base far from position 0."""
    B, Hk, G, D, L = 1, 8, 4, 128, 100003
    c = _contig(B, Hk, D, "per_token", [L], seed=50)
    q = bf16_randn((B, Hk * G, D), seed=51)
    sl = torch.tensor([L], dtype=torch.int32)
    m = kvq()
    assert m.lib.kvq_window_workspace_bytes(B, Hk * G, Hk, 1, D, L, 64, 0) <= \
        m.kvq_decode_workspace_bytes(B, Hk * G, Hk, D, 64 + 15)
    assert_attn_close(_window(c, q, sl, L, 64), _window_ref(c, q, sl, 64), "100k, w=64")


@pytest.mark.parametrize("w", [8, 100])
def test_ring_store_sliding_layer(w):
    """A sliding layer's ring of w rows (position g in row g % w, appended one
    token per step) decoded with kvq_decode_attn over min(L, w) rows equals the
    oracle's window attention over the full history."""
    m = kvq()
    B, Hk, G, D, steps = 2, 2, 4, 128, 130
    ring = ContigCache(B, Hk, w, D, "per_token")
    full = ContigCache(B, Hk, steps, D, "per_token")
    for step in range(steps):
        kn = bf16_randn((B, Hk, 1, D), 1000 + step)
        vn = bf16_randn((B, Hk, 1, D), 5000 + step)
        assert ring.append(kn, vn, torch.full((B,), step % w, dtype=torch.int32)) == 0
        assert full.append(kn, vn, torch.full((B,), step, dtype=torch.int32)) == 0
        if step % 37 == 0 or step == steps - 1:
            L = step + 1
            q = bf16_randn((B, Hk * G, D), seed=step)
            n = torch.full((B,), min(L, w), dtype=torch.int32)
            out = m.kvq_decode_attn(q.cuda(), ring.k, ring.v, ring.ks, ring.vs, n.cuda(), w,
                                    attn_scale=f32_scale(D))
            ref = oracle.window_attn(q, full.ok, full.ov, full.oks, full.ovs,
                                     torch.full((B,), L, dtype=torch.int32), w, f32_scale(D))
            assert_attn_close(out, ref, f"ring w={w} L={L}")


def test_window_argument_errors():
    m = kvq()
    c = _contig(1, 1, 64, "per_token", [10], seed=1)
    q = bf16_randn((1, 4, 64), seed=2).cuda()
    sl = torch.tensor([10], dtype=torch.int32).cuda()
    for bad in (0, -3):
        with pytest.raises(m.KvqError):
            m.kvq_window_attn(q, c.k, c.v, c.ks, c.vs, sl, 10, bad)

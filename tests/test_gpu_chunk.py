"""GPU parity: kvq_chunk_attn (T queries per sequence and q head, causal
from the chunk's end) against the oracle's fp64 chunk attention over the same
dequantized cache (max-abs 2e-3, relative-L2 1e-3): both scale modes, both
layouts, one item per CTA and blocks of items, forced split counts, chunks
that fill the cache, and the length rule."""
import random

import pytest
import torch

from kvq_testutil import (ContigCache, PagedCache, assert_attn_close, bf16_randn, f32_scale,
                          kvq)

pytestmark = pytest.mark.gpu

KVQ_DEVERR_LEN = 4


def _contig(B, Hk, D, mode, lens, seed):
    S = max(lens) + 1
    c = ContigCache(B, Hk, S, D, mode)
    L = max(lens)
    if L > 0:
        k = bf16_randn((B, Hk, L, D), seed)
        v = bf16_randn((B, Hk, L, D), seed + 1)
        assert c.append(k, v, torch.zeros(B, dtype=torch.int32)) == 0
    return c


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G,T", [(1, 4), (4, 2), (4, 4), (8, 2), (2, 8), (1, 16)])
def test_chunk_contig_matches_oracle(mode, D, G, T):
    B, Hk = 3, 2
    lens = [T, 130, 517]                 # a chunk that fills its cache, ragged others
    c = _contig(B, Hk, D, mode, lens, seed=G * 11 + T + D)
    q = bf16_randn((B, Hk * G, T, D), seed=G + T)
    sl = torch.tensor(lens, dtype=torch.int32)
    sc = f32_scale(D)
    ref = c.oracle_chunk(q, sl, sc)
    for ns in (0, 1, 3):
        out = c.chunk(q, sl, max(lens), attn_scale=sc, num_splits=ns)
        assert_attn_close(out, ref, f"G={G} T={T} D={D} {mode} ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_chunk_many_units_blocks_of_items(mode):
    """Many (sequence, kv head) units of different lengths: one-stage chunks and
    the weighted partition (blocks of items, segments split over CTAs)."""
    rnd = random.Random(5 + (mode == "group32"))
    B, Hk, G, D, T = 40, 4, 2, 64, 3
    lens = [rnd.choice([0, 3, 17, 130, 600, 2000]) for _ in range(B)]
    c = _contig(B, Hk, D, mode, lens, seed=71)
    q = bf16_randn((B, Hk * G, T, D), seed=72)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = c.chunk(q, sl, max(lens), attn_scale=f32_scale(D))
    assert_attn_close(out, c.oracle_chunk(q, sl, f32_scale(D)), f"many units {mode}")


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_chunk_paged_matches_oracle(mode):
    B, Hk, G, D, T, ps = 3, 2, 4, 128, 4, 16
    lens = [4, 47, 300]
    need = [(L + ps - 1) // ps for L in lens]
    num_pages = sum(need) + 2
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(81)).to(torch.int32)
    table = torch.full((B, max(need)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    c = PagedCache(num_pages, Hk, D, mode, table)
    for b, L in enumerate(lens):
        k = bf16_randn((1, Hk, L, D), seed=82 + b)
        v = bf16_randn((1, Hk, L, D), seed=92 + b)
        assert c.append(k, v, torch.zeros(1, dtype=torch.int32), rows=[b]) == 0
    q = bf16_randn((B, Hk * G, T, D), seed=99)
    sl = torch.tensor(lens, dtype=torch.int32)
    for ns in (0, 2):
        out = c.chunk(q, sl, max(lens), attn_scale=f32_scale(D), num_splits=ns)
        assert_attn_close(out, c.oracle_chunk(q, sl, f32_scale(D)), f"paged {mode} ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


def test_chunk_of_one_equals_decode():
    B, Hk, G, D = 2, 2, 4, 128
    lens = [300, 1000]
    c = _contig(B, Hk, D, "per_token", lens, seed=101)
    q = bf16_randn((B, Hk * G, 1, D), seed=102)
    sl = torch.tensor(lens, dtype=torch.int32)
    a = c.chunk(q, sl, max(lens), attn_scale=f32_scale(D))
    b = c.decode(q[:, :, 0].contiguous(), sl, max(lens), attn_scale=f32_scale(D))
    assert torch.equal(a[:, :, 0], b)


def test_chunk_longer_than_its_sequence_is_a_length_error():
    B, Hk, G, D, T = 2, 1, 2, 64, 4
    lens = [3, 40]                       # sequence 0 cannot hold its 4-token chunk
    c = _contig(B, Hk, D, "per_token", lens, seed=111)
    q = bf16_randn((B, Hk * G, T, D), seed=112)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = c.chunk(q, sl, max(lens), attn_scale=f32_scale(D))
    assert kvq().kvq_read_error(c.err) & KVQ_DEVERR_LEN
    assert torch.count_nonzero(out[0]) == 0
    assert_attn_close(out[1:], c.oracle_chunk(q, sl, f32_scale(D))[1:], "valid sequence")


def test_chunk_rows_beyond_sixteen_per_kv_head_at_d64():
    """More than 16 rows per kv head at head_dim 64, a shape the dense kernel
    does not cover: the CUDA-core split kernel takes it."""
    c = _contig(1, 1, 64, "per_token", [40], seed=121)
    q = bf16_randn((1, 4, 5, 64), seed=122)      # G * T = 20
    sl = torch.tensor([40], dtype=torch.int32)
    assert_attn_close(c.chunk(q, sl, 40, attn_scale=f32_scale(64)),
                      c.oracle_chunk(q, sl, f32_scale(64)), "G*T=20 at D=64")
    assert kvq().kvq_read_error(c.err) == 0

"""GPU parity: kvq_decode_attn against the oracle's fp64 attention over the same
dequantized cache (max-abs 2e-3, relative-L2 1e-3), on small and ragged
shapes, both layouts, both scale modes, forced split counts, and the
degenerate cases (length 1, empty sequences, page-boundary lengths)."""
import pytest
import torch

from kvq_testutil import (ContigCache, PagedCache, assert_attn_close, bf16_randn, f32_scale,
                          kvq)

pytestmark = pytest.mark.gpu


def _fill_contig(B, Hq, Hk, D, mode, lens, seed, sigma=1.0, outlier=None):
    S = max(lens) + 1
    c = ContigCache(B, Hk, S, D, mode)
    L = max(lens)
    k = bf16_randn((B, Hk, L, D), seed, sigma)
    v = bf16_randn((B, Hk, L, D), seed + 1, sigma)
    if outlier is not None:
        k[:, :, :, outlier] = (k[:, :, :, outlier].float() * 10).to(torch.bfloat16)
        v[:, :, :, outlier] = (v[:, :, :, outlier].float() * 10).to(torch.bfloat16)
    if L > 0:
        assert c.append(k, v, torch.zeros(B, dtype=torch.int32)) == 0
    q = bf16_randn((B, Hq, D), seed + 2)
    return c, q


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 8, 12, 16])
def test_decode_contig_small(mode, D, G):
    B, Hk = 3, 2
    lens = [1, 130, 517]
    c, q = _fill_contig(B, Hk * G, Hk, D, mode, lens, seed=G * 7 + D)
    sl = torch.tensor(lens, dtype=torch.int32)
    sc = f32_scale(D)
    out = c.decode(q, sl, max(lens), attn_scale=sc)
    ref = c.oracle_decode(q, sl, sc)
    assert_attn_close(out, ref, f"G={G} D={D} {mode}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("num_splits", [1, 2, 3, 17, 64])
def test_decode_split_count_only_changes_rounding(num_splits):
    B, Hk, G, D = 2, 2, 4, 128
    lens = [1000, 333]
    c, q = _fill_contig(B, Hk * G, Hk, D, "per_token", lens, seed=11)
    sl = torch.tensor(lens, dtype=torch.int32)
    sc = f32_scale(D)
    ref = c.oracle_decode(q, sl, sc)
    out = c.decode(q, sl, max(lens), attn_scale=sc, num_splits=num_splits)
    assert_attn_close(out, ref, f"splits={num_splits}")
    base = c.decode(q, sl, max(lens), attn_scale=sc, num_splits=1)
    assert (out - base).abs().max().item() < 1e-4


@pytest.mark.parametrize("L", [1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 255, 256,
                               257, 1023, 1024, 1025])
def test_decode_tile_edges(L):
    c, q = _fill_contig(1, 8, 2, 128, "per_token", [L], seed=L)
    sl = torch.tensor([L], dtype=torch.int32)
    out = c.decode(q, sl, L, attn_scale=f32_scale(128))
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(128)), f"L={L}")


def test_decode_length_one_returns_the_value():
    c, q = _fill_contig(2, 4, 1, 64, "per_token", [1, 1], seed=3)
    sl = torch.tensor([1, 1], dtype=torch.int32)
    out = c.decode(q, sl, 1).cpu()
    vhat = kvq().kvq_dequant(c.v[:, :, :1].contiguous(), c.vs[:, :, :1].contiguous()).cpu()
    for h in range(4):
        assert torch.allclose(out[:, h], vhat[:, 0, 0], rtol=1e-6, atol=1e-7)


def test_decode_empty_sequences_give_zero_rows():
    c, q = _fill_contig(3, 8, 2, 64, "group32", [0, 50, 0], seed=4)
    sl = torch.tensor([0, 50, 0], dtype=torch.int32)
    for ns in (0, 1, 4):
        out = c.decode(q, sl, 50, attn_scale=f32_scale(64), num_splits=ns).cpu()
        assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
        assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(64)), f"ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


def test_decode_length_beyond_capacity_is_flagged():
    c, q = _fill_contig(2, 4, 1, 64, "per_token", [10, 10], seed=5)
    sl = torch.tensor([10, 999], dtype=torch.int32)     # capacity is 11
    out = c.decode(q, sl, 11).cpu()
    assert kvq().kvq_read_error(c.err) == kvq().DEVERR_LEN
    assert torch.all(out[1] == 0)


def test_decode_gqa_identical_queries_identical_outputs():
    c, q = _fill_contig(1, 16, 2, 128, "per_token", [700], seed=6)
    q[0, 8:16] = q[0, 8:9]                      # kv head 1's group: identical queries
    out = c.decode(q, torch.tensor([700], dtype=torch.int32), 700).cpu()
    for h in range(9, 16):
        assert torch.equal(out[0, h], out[0, 8])


def test_decode_outlier_channels():
    c, q = _fill_contig(1, 32, 8, 128, "per_token", [2000], seed=7, outlier=[3, 77])
    sl = torch.tensor([2000], dtype=torch.int32)
    assert_attn_close(c.decode(q, sl, 2000, attn_scale=f32_scale(128)),
                      c.oracle_decode(q, sl, f32_scale(128)), "outliers")


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("G,D", [(1, 128), (4, 128), (8, 128), (16, 128), (4, 64)])
def test_decode_paged_matches_oracle(mode, G, D):
    B, Hk, ps = 3, 2, 16
    lens = [16, 47, 300]
    need = [(L + ps - 1) // ps for L in lens]
    gen = torch.Generator().manual_seed(G)
    num_pages = sum(need) + 3
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = torch.full((B, max(need)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    c = PagedCache(num_pages, Hk, D, mode, table)
    for b, L in enumerate(lens):
        k = bf16_randn((1, Hk, L, D), seed=30 + b, sigma=0.5)
        v = bf16_randn((1, Hk, L, D), seed=40 + b, sigma=0.5)
        assert c.append(k, v, torch.zeros(1, dtype=torch.int32), rows=[b]) == 0
    c.assert_bit_exact()
    q = bf16_randn((B, Hk * G, D), seed=50)
    sl = torch.tensor(lens, dtype=torch.int32)
    for ns in (0, 1, 5):
        out = c.decode(q, sl, max(lens), attn_scale=f32_scale(D), num_splits=ns)
        assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), f"paged ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


def test_decode_paged_equals_contiguous_on_same_bytes():
    """The same logical cache read through a page table gives the same output."""
    D, Hk, G, L = 128, 2, 4, 200
    cc, q = _fill_contig(1, Hk * G, Hk, D, "per_token", [L], seed=9)
    npg = (L + 15) // 16
    table = torch.randperm(npg, generator=torch.Generator().manual_seed(1)).to(torch.int32)[None]
    pc = PagedCache(npg, Hk, D, "per_token", table)
    torch.cuda.synchronize()
    for t in range(L):
        p, s = int(table[0, t // 16]), t % 16
        pc.k[p, :, s] = cc.k[0, :, t]
        pc.v[p, :, s] = cc.v[0, :, t]
        pc.ks[p, :, s] = cc.ks[0, :, t]
        pc.vs[p, :, s] = cc.vs[0, :, t]
    sl = torch.tensor([L], dtype=torch.int32)
    a = cc.decode(q, sl, L, num_splits=3)
    b = pc.decode(q, sl, L, num_splits=3)
    assert torch.equal(a.cpu(), b.cpu())


def test_decode_bad_page_is_flagged_not_read():
    table = torch.tensor([[0, 1, 99]], dtype=torch.int32)
    c = PagedCache(3, 1, 64, "per_token", table)
    k = bf16_randn((1, 1, 32, 64), seed=1)
    v = bf16_randn((1, 1, 32, 64), seed=2)
    assert c.append(k, v, torch.zeros(1, dtype=torch.int32)) == 0
    q = bf16_randn((1, 2, 64), seed=3)
    c.decode(q, torch.tensor([40], dtype=torch.int32), 48)
    assert kvq().kvq_read_error(c.err) & kvq().DEVERR_PAGE


@pytest.mark.parametrize("G", [4, 8])
def test_decode_peaky_softmax(G):
    """One key per sequence aligned with the query dominates the softmax."""
    B, Hk, D, L = 2, 2, 128, 300
    c, q = _fill_contig(B, Hk * G, Hk, D, "per_token", [L, L], seed=21)
    kq = q.view(B, Hk, G, D)[:, :, 0]                       # first query head of each group
    k_hot = (kq.float() * 6).to(torch.bfloat16)[:, :, None]  # [B, Hk, 1, D]
    v_hot = bf16_randn((B, Hk, 1, D), seed=22, sigma=4.0)
    assert c.append(k_hot, v_hot, torch.tensor([137, 5], dtype=torch.int32)) == 0
    sl = torch.tensor([L, L], dtype=torch.int32)
    out = c.decode(q, sl, L, attn_scale=f32_scale(D))
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), "peaky")


@pytest.mark.parametrize("G", [4, 8])
def test_decode_large_query_magnitudes(G):
    """Query rows of very different magnitude (the per-head integer prescale;
    G = 4 also runs the group-pair packing of group-32 scales)."""
    B, Hk, D, L = 1, 2, 128, 200
    c, q = _fill_contig(B, Hk * G, Hk, D, "group32", [L], seed=23)
    qf = q.float()
    qf[0, 0] *= 1e-20
    qf[0, 1] *= 3e4
    qf[0, 2] = 0
    qf[0, 3, :5] = 1e-30
    q = qf.to(torch.bfloat16)
    sl = torch.tensor([L], dtype=torch.int32)
    out = c.decode(q, sl, L, attn_scale=1e-4)
    assert_attn_close(out, c.oracle_decode(q, sl, 1e-4), "q magnitudes")


@pytest.mark.parametrize("mode,D", [("per_token", 128), ("per_token", 64), ("group32", 64)])
@pytest.mark.parametrize("S", [257, 130, 131])
def test_decode_full_cache_unaligned_capacity(mode, D, S):
    """Every sequence fills its whole capacity S, and S * (scales per token) is
    not a multiple of 4: the scale rows of a (sequence, kv head) start off a
    16-byte boundary and the last tile ends at the end of the scale array."""
    B, Hk, G = 2, 3, 2
    c = ContigCache(B, Hk, S, D, mode)
    k = bf16_randn((B, Hk, S, D), seed=S, sigma=0.7)
    v = bf16_randn((B, Hk, S, D), seed=S + 1, sigma=0.7)
    assert c.append(k, v, torch.zeros(B, dtype=torch.int32)) == 0
    q = bf16_randn((B, Hk * G, D), seed=S + 2)
    sl = torch.tensor([S, S], dtype=torch.int32)
    for ns in (0, 1, 3):
        out = c.decode(q, sl, S, attn_scale=f32_scale(D), num_splits=ns)
        assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), f"S={S} ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0



def test_one_workspace_serves_calls_of_any_shape():
    """One workspace, reused across calls of different shapes and split counts,
    gives the oracle's answer every time (its contents on entry are ignored)."""
    m = kvq()
    ws = torch.full((8 << 20,), 0xFF, dtype=torch.uint8, device="cuda")   # NaN bit patterns
    cases = [(2, 8, 2, 128, "per_token", [1000, 333]), (3, 16, 2, 64, "group32", [517, 1, 130]),
             (1, 32, 8, 128, "per_token", [4097])]
    for rep in range(2):
        for i, (B, Hq, Hk, D, mode, lens) in enumerate(cases):
            c, q = _fill_contig(B, Hq, Hk, D, mode, lens, seed=100 + i)
            sl = torch.tensor(lens, dtype=torch.int32)
            need = m.kvq_decode_workspace_bytes(B, Hq, Hk, D, max(lens), 7)
            assert 0 < need <= ws.numel()
            out = c.decode(q, sl, max(lens), attn_scale=f32_scale(D), num_splits=7, workspace=ws)
            assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), f"case {i} rep {rep}")


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("num_splits,top", [(0, 4100), (40, 4100), (300, 4100), (0, 2000)])
def test_decode_many_units_ragged_with_empty_sequences(mode, num_splits, top):
    """Many (sequence, kv head) units of very different lengths, some empty:
    one-stage chunks, the weighted CTA partition, units split over several
    CTAs and units finished inside one, and the combine that finds a unit's
    partials from its m slots (within the first 128 slots and past them)."""
    import random
    rnd = random.Random(num_splits + (7 if mode == "group32" else 0))
    B, Hk, G, D = 40, 4, 2, 64
    lens = [rnd.choice([0, 1, 17, 130, 600, 2000, top]) for _ in range(B)]
    lens[3] = 0
    c, q = _fill_contig(B, Hk * G, Hk, D, mode, lens, seed=90 + num_splits)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = c.decode(q, sl, max(lens), attn_scale=f32_scale(D), num_splits=num_splits).cpu()
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), f"splits={num_splits} {mode}")
    for b, L in enumerate(lens):
        if L == 0:
            assert torch.all(out[b] == 0)
    assert kvq().kvq_read_error(c.err) == 0

"""GPU parity of the one-call decode step (kvq_append_decode).

kvq_append_decode quantises the step's new token into position L - 1 of the
cache inside the decode kernel, then attends.  Its cache bytes and scales
must equal the oracle's append bit for bit, and its output must be the
oracle's fp64 attention over that cache within the decode bar.  Against the
two-call step (kvq_append at L - 1, then kvq_decode_attn) it must agree
exactly: the same bytes reach the same arithmetic.
"""
import pytest
import torch

import oracle
from kvq_testutil import (ContigCache, PagedCache, assert_attn_close, bf16_randn, f32_scale,
                          kvq)

pytestmark = pytest.mark.gpu


def _contig_with_history(B, Hk, D, mode, lens, seed):
    """Contiguous cache holding max(lens) - 1 history tokens of every sequence."""
    S = max(max(lens), 1) + 3
    c = ContigCache(B, Hk, S, D, mode)
    H = max(lens) - 1
    if H > 0:
        k = bf16_randn((B, Hk, H, D), seed)
        v = bf16_randn((B, Hk, H, D), seed + 1)
        assert c.append(k, v, torch.zeros(B, dtype=torch.int32)) == 0
    return c


def _clone_contig(c):
    d = ContigCache(c.B, c.Hk, c.S, c.D, c.mode)
    for a in ("k", "v", "ks", "vs", "ok", "ov", "oks", "ovs"):
        getattr(d, a).copy_(getattr(c, a))
    return d


def _fused(c, q, k_new, v_new, sl, hint, paged=False, **kw):
    m = kvq()
    dev = c.k.device
    extra = dict(page_table=c.table, page_size=c.ps) if paged else {}
    return m.kvq_append_decode(q.to(dev), k_new.to(dev), v_new.to(dev), c.k, c.v, c.ks, c.vs,
                               sl.to(dev), hint, mode=c.mode, err=c.err, **extra, **kw)


def _oracle_append_new(c, k_new, v_new, sl, paged=False):
    """The oracle's append of the new token at L - 1 (L = 0: nothing)."""
    pos = (sl - 1).to(torch.int32)
    if paged:
        e1 = oracle.append_paged(k_new, pos, c.ok, c.oks, c.table_cpu, c.ps, c.mode)
        e2 = oracle.append_paged(v_new, pos, c.ov, c.ovs, c.table_cpu, c.ps, c.mode)
    else:
        e1 = oracle.append_contig(k_new, pos, c.ok, c.oks, c.mode)
        e2 = oracle.append_contig(v_new, pos, c.ov, c.ovs, c.mode)
    return e1 | e2


CASES = [
    # B, Hq, Hk, lens, num_splits
    (1, 32, 8, [4097], 0),           # one item per CTA, the new token alone in its chunk
    (2, 8, 2, [1, 129], 0),          # the new token is the whole sequence / starts a stage
    (3, 16, 2, [128, 129, 1000], 3),
    (2, 8, 2, [256, 257], 17),
    (4, 8, 2, [300, 17, 33, 257], 64),
]


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_append_decode_contig_matches_oracle_and_two_calls(mode, D, case):
    B, Hq, Hk, lens, ns = CASES[case]
    sc = f32_scale(D)
    c = _contig_with_history(B, Hk, D, mode, lens, seed=300 + case)
    two = _clone_contig(c)
    k_new = bf16_randn((B, Hk, 1, D), seed=400 + case)
    v_new = bf16_randn((B, Hk, 1, D), seed=500 + case)
    q = bf16_randn((B, Hq, D), seed=600 + case)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = _fused(c, q, k_new, v_new, sl, max(lens), num_splits=ns)
    assert _oracle_append_new(c, k_new, v_new, sl) == 0
    c.assert_bit_exact()
    assert_attn_close(out, c.oracle_decode(q, sl, sc), f"fused {mode} D={D} case {case}")
    assert kvq().kvq_read_error(c.err) == 0
    # the two-call step on a copy of the same cache
    m = kvq()
    m.kvq_append(k_new.cuda(), v_new.cuda(), (sl - 1).cuda(), two.k, two.v, two.ks, two.vs,
                 mode, err=two.err)
    ref = two.decode(q, sl, max(lens), attn_scale=sc, num_splits=ns)
    torch.cuda.synchronize()
    assert torch.equal(c.k, two.k) and torch.equal(c.v, two.v)
    assert torch.equal(c.ks.view(torch.int32), two.ks.view(torch.int32))
    assert torch.equal(c.vs.view(torch.int32), two.vs.view(torch.int32))
    assert torch.equal(out, ref), "fused step differs from append + decode"


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("ns", [0, 1, 5])
def test_append_decode_paged(mode, ns):
    B, Hk, G, D, ps = 3, 2, 4, 128, 16
    lens = [16, 17, 300]              # the new token ends a page / starts one
    need = [(L + ps - 1) // ps for L in lens]
    gen = torch.Generator().manual_seed(77 + ns)
    num_pages = sum(need) + 3
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = torch.full((B, max(need)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    c = PagedCache(num_pages, Hk, D, mode, table)
    for b, L in enumerate(lens):
        if L > 1:
            k = bf16_randn((1, Hk, L - 1, D), seed=30 + b, sigma=0.5)
            v = bf16_randn((1, Hk, L - 1, D), seed=40 + b, sigma=0.5)
            assert c.append(k, v, torch.zeros(1, dtype=torch.int32), rows=[b]) == 0
    k_new = bf16_randn((B, Hk, 1, D), seed=51, sigma=0.5)
    v_new = bf16_randn((B, Hk, 1, D), seed=52, sigma=0.5)
    q = bf16_randn((B, Hk * G, D), seed=53)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = _fused(c, q, k_new, v_new, sl, max(lens), paged=True, num_splits=ns)
    assert _oracle_append_new(c, k_new, v_new, sl, paged=True) == 0
    c.assert_bit_exact()
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), f"paged fused ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_append_decode_many_units_and_empty_sequences(mode):
    """Blocks of several items per CTA (more units than SMs), ragged lengths
    with empty sequences: zero rows and nothing written for those."""
    B, Hk, G, D = 40, 8, 4, 128
    gen = torch.Generator().manual_seed(5)
    lens = torch.randint(1, 700, (B,), generator=gen)
    lens[3] = 0
    lens[17] = 0
    lens[20] = 1
    lens = lens.tolist()
    c = _contig_with_history(B, Hk, D, mode, lens, seed=900)
    k_new = bf16_randn((B, Hk, 1, D), seed=901)
    v_new = bf16_randn((B, Hk, 1, D), seed=902)
    q = bf16_randn((B, Hk * G, D), seed=903)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = _fused(c, q, k_new, v_new, sl, max(lens))
    # the oracle flags the two empty sequences' position -1 and skips them
    _oracle_append_new(c, k_new, v_new, sl)
    c.assert_bit_exact()
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), "many units")
    assert out[3].abs().max().item() == 0 and out[17].abs().max().item() == 0
    assert kvq().kvq_read_error(c.err) == 0


def test_append_decode_length_beyond_capacity_writes_nothing():
    B, Hk, G, D = 2, 2, 4, 128
    c = _contig_with_history(B, Hk, D, "per_token", [100, 100], seed=11)
    before_k, before_ks = c.k.clone(), c.ks.clone()
    k_new = bf16_randn((B, Hk, 1, D), seed=12)
    q = bf16_randn((B, Hk * G, D), seed=13)
    sl = torch.tensor([100, c.S + 5], dtype=torch.int32)
    out = _fused(c, q, k_new, k_new, sl, c.S + 5)
    torch.cuda.synchronize()
    assert kvq().kvq_read_error(c.err) == 4            # KVQ_DEVERR_LEN
    assert torch.equal(c.k[1], before_k[1]) and torch.equal(c.ks[1], before_ks[1])
    assert out[1].abs().max().item() == 0
    assert not torch.equal(c.k[0, :, 99], before_k[0, :, 99])   # sequence 0 was appended


def test_one_workspace_serves_decode_chunk_window_and_fused_calls():
    """One workspace (scratch filled with NaN bit patterns) reused by decode,
    chunk, window and fused calls of different shapes and split counts."""
    m = kvq()
    ws = torch.full((8 << 20,), 0xFF, dtype=torch.uint8, device="cuda")
    B, Hk, G, D = 2, 2, 4, 128
    c = _contig_with_history(B, Hk, D, "per_token", [1500, 700], seed=21)
    sl = torch.tensor([1499, 700], dtype=torch.int32)
    q = bf16_randn((B, Hk * G, D), seed=22)
    sc = f32_scale(D)
    for ns in (0, 3, 40):
        out = c.decode(q, sl, 1500, attn_scale=sc, num_splits=ns, workspace=ws)
        assert_attn_close(out, c.oracle_decode(q, sl, sc), f"decode ns={ns}")
    qc = bf16_randn((B, Hk * G // 2, 2, D), seed=23)
    outc = c.chunk(qc, sl, 1500, attn_scale=sc, num_splits=5, workspace=ws)
    assert_attn_close(outc, c.oracle_chunk(qc, sl, sc), "chunk")
    outw = m.kvq_window_attn(q.cuda(), c.k, c.v, c.ks, c.vs, sl.cuda(), 1500, 300,
                             attn_scale=sc, num_splits=4, workspace=ws, err=c.err)
    assert_attn_close(outw, oracle.window_attn(q, c.ok, c.ov, c.oks, c.ovs, sl, 300, sc),
                      "window")
    k_new = bf16_randn((B, Hk, 1, D), seed=24)
    sl2 = sl + 1
    out = _fused(c, q, k_new, k_new, sl2, 1501, num_splits=6, workspace=ws)
    assert _oracle_append_new(c, k_new, k_new, sl2) == 0
    c.assert_bit_exact()
    assert_attn_close(out, c.oracle_decode(q, sl2, sc), "fused")
    assert m.kvq_read_error(c.err) == 0


def test_append_decode_many_short_sequences():
    """Thousands of (sequence, kv head) units with short ragged lengths."""
    B, Hk, G, D = 520, 8, 2, 64
    gen = torch.Generator().manual_seed(8)
    lens = torch.randint(1, 300, (B,), generator=gen).tolist()
    c = _contig_with_history(B, Hk, D, "per_token", lens, seed=31)
    k_new = bf16_randn((B, Hk, 1, D), seed=32)
    v_new = bf16_randn((B, Hk, 1, D), seed=33)
    q = bf16_randn((B, Hk * G, D), seed=34)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = _fused(c, q, k_new, v_new, sl, max(lens))
    assert _oracle_append_new(c, k_new, v_new, sl) == 0
    c.assert_bit_exact()
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), "many short sequences")
    assert kvq().kvq_read_error(c.err) == 0

"""The oracle's all-core baseline build (oracle/baseline_omp.c, OpenMP over
independent (sequence, kv head) units) gives exactly the pinned oracle's
results: each unit is one call of the pinned routine on a one-sequence,
one-kv-head view, so the outputs must be bit-identical for decode and chunk
attention, contiguous and paged, both scale modes."""
import math

import pytest
import torch

import oracle
import synth


def _contig(wl, B, lo, hi, mode):
    inp = synth.make_decode_inputs(wl, B=B, len_lo=lo, len_hi=hi)
    Hk, D = wl.Hk, wl.D
    n = 1 if mode == "per_token" else D // 32
    S = int(inp.seq_lens.max())
    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
    v = torch.zeros_like(k)
    ks, vs = torch.zeros(B, Hk, S, n), torch.zeros(B, Hk, S, n)
    zb = torch.zeros(B, dtype=torch.int32)
    Lm = int(inp.cached.max())
    oracle.append_contig(inp.k_hist[:, :, :Lm].contiguous(), zb, k, ks, mode)
    oracle.append_contig(inp.v_hist[:, :, :Lm].contiguous(), zb, v, vs, mode)
    oracle.append_contig(inp.k_new, inp.cached, k, ks, mode)
    oracle.append_contig(inp.v_new, inp.cached, v, vs, mode)
    return inp, k, v, ks, vs


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("T", [1, 3])
def test_units_equal_oracle_contiguous(mode, T):
    wl = synth.WORKLOADS["batched_group32"]
    inp, k, v, ks, vs = _contig(wl, 3, 20, 90, mode)
    sc = 1.0 / math.sqrt(wl.D)
    g = torch.Generator().manual_seed(5)
    q = inp.q if T == 1 else torch.randn(3, wl.Hq, T, wl.D, generator=g).to(torch.bfloat16)
    ref = (oracle.decode_attn if T == 1 else oracle.chunk_attn)(q, k, v, ks, vs, inp.seq_lens,
                                                                sc, mode)
    got, err = oracle.attn_units(q, k, v, ks, vs, inp.seq_lens, sc, mode, threads=4)
    assert err == 0 and torch.equal(ref, got)


def test_units_equal_oracle_paged():
    wl = synth.WORKLOADS["paged"]
    B = 3
    inp = synth.make_decode_inputs(wl, B=B, len_lo=25, len_hi=70)
    Hk, D = wl.Hk, wl.D
    k = torch.zeros(inp.num_pages, Hk, 16, D, dtype=torch.uint8)
    v = torch.zeros_like(k)
    ks, vs = torch.zeros(inp.num_pages, Hk, 16, 1), torch.zeros(inp.num_pages, Hk, 16, 1)
    z1 = torch.zeros(1, dtype=torch.int32)
    for b in range(B):
        L = int(inp.cached[b])
        tb = inp.page_table[b:b + 1].contiguous()
        oracle.append_paged(inp.k_hist[b:b + 1, :, :L].contiguous(), z1, k, ks, tb)
        oracle.append_paged(inp.v_hist[b:b + 1, :, :L].contiguous(), z1, v, vs, tb)
    oracle.append_paged(inp.k_new, inp.cached, k, ks, inp.page_table)
    oracle.append_paged(inp.v_new, inp.cached, v, vs, inp.page_table)
    sc = 1.0 / math.sqrt(D)
    ref = oracle.decode_attn(inp.q, k, v, ks, vs, inp.seq_lens, sc, page_size=16,
                             table=inp.page_table)
    ut = oracle.unit_tables(inp.page_table, Hk, inp.num_pages)
    got, err = oracle.attn_units(inp.q, k, v, ks, vs, inp.seq_lens, sc, page_size=16,
                                 utables=ut, num_pages=inp.num_pages, threads=3)
    assert err == 0 and torch.equal(ref, got)


def test_unit_tables_keep_bad_entries_bad():
    t = torch.tensor([[0, 2, -1, 5]], dtype=torch.int32)
    u = oracle.unit_tables(t, 2, 3)            # 3 pages: entry 5 is outside the arena
    assert u.tolist() == [[0, 4, -1, -1], [1, 5, -1, -1]]

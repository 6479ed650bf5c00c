"""Pins of the oracle's sliding-window attention (oracle_window_attn):
against torch fp64 scaled_dot_product_attention with the page's window mask
built here (combs-models 0.2.2, src/kv.rs, attend: a key at k is forbidden
when k > p or k + w - 1 < p), against the pinned decode / chunk attention
when the window covers everything, the closed form of a one-token window,
the ring store of a sliding layer (the last w tokens in any order give the
same decode: the page's sliding_layer_matches_masked_global property), and
paged = contiguous."""
import math

import pytest
import torch

import oracle


def _cache(B, Hk, S, D, mode, seed, L=None):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, Hk, S, D, generator=g).to(torch.bfloat16)
    y = torch.randn(B, Hk, S, D, generator=g).to(torch.bfloat16)
    n = 1 if mode == "per_token" else D // 32
    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
    v = torch.zeros_like(k)
    ks, vs = torch.zeros(B, Hk, S, n), torch.zeros(B, Hk, S, n)
    z = torch.zeros(B, dtype=torch.int32)
    oracle.append_contig(x, z, k, ks, mode)
    oracle.append_contig(y, z, v, vs, mode)
    return k, v, ks, vs


def _sdpa_window(q, k, v, ks, vs, lens, window, scale, mode):
    """torch fp64 SDPA over the dequantized cache with the page's window mask."""
    B, Hq, T, D = q.shape
    Hk = k.shape[1]
    G = Hq // Hk
    kd = oracle.dequant(k, ks, mode).double()
    vd = oracle.dequant(v, vs, mode).double()
    out = torch.zeros(B, Hq, T, D, dtype=torch.float64)
    for b in range(B):
        L = int(lens[b])
        if L == 0:
            continue
        kk = kd[b, :, :L].repeat_interleave(G, dim=0)
        vv = vd[b, :, :L].repeat_interleave(G, dim=0)
        qp = torch.arange(L - T, L).view(T, 1)
        kp = torch.arange(L).view(1, L)
        forbidden = (kp > qp) | (kp + window - 1 < qp)
        mask = (~forbidden).unsqueeze(0).expand(Hq, T, L)
        out[b] = torch.nn.functional.scaled_dot_product_attention(
            q[b].double(), kk, vv, attn_mask=mask, scale=scale)
    return out


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("T,window", [(1, 5), (1, 1), (1, 64), (4, 3), (7, 5), (6, 40)])
def test_window_vs_sdpa(mode, T, window):
    B, Hq, Hk, D, S = 2, 4, 2, 64, 50
    k, v, ks, vs = _cache(B, Hk, S, D, mode, seed=3)
    lens = torch.tensor([50, 23], dtype=torch.int32)
    g = torch.Generator().manual_seed(9)
    q = torch.randn(B, Hq, T, D, generator=g).to(torch.bfloat16)
    sc = 1.0 / math.sqrt(D)
    got = oracle.window_attn(q if T > 1 else q[:, :, 0], k, v, ks, vs, lens, window, sc, mode)
    ref = _sdpa_window(q, k, v, ks, vs, lens, window, sc, mode)
    assert torch.allclose(got.reshape(ref.shape), ref, atol=1e-12, rtol=1e-10)


def test_window_covering_everything_is_plain_attention():
    B, Hq, Hk, D, S = 2, 8, 2, 64, 70
    k, v, ks, vs = _cache(B, Hk, S, D, "per_token", seed=4)
    lens = torch.tensor([70, 31], dtype=torch.int32)
    g = torch.Generator().manual_seed(1)
    q1 = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    q4 = torch.randn(B, Hq, 4, D, generator=g).to(torch.bfloat16)
    assert torch.equal(oracle.window_attn(q1, k, v, ks, vs, lens, 70),
                       oracle.decode_attn(q1, k, v, ks, vs, lens))
    assert torch.equal(oracle.window_attn(q4, k, v, ks, vs, lens, 1000),
                       oracle.chunk_attn(q4, k, v, ks, vs, lens))


def test_window_of_one_returns_the_newest_value():
    B, Hq, Hk, D, S = 1, 4, 1, 64, 20
    k, v, ks, vs = _cache(B, Hk, S, D, "per_token", seed=5)
    lens = torch.tensor([17], dtype=torch.int32)
    q = torch.randn(B, Hq, 3, D).to(torch.bfloat16)
    out = oracle.window_attn(q, k, v, ks, vs, lens, 1)
    vd = oracle.dequant(v, vs).double()
    for i in range(3):
        for h in range(Hq):
            assert torch.equal(out[0, h, i], vd[0, 0, 17 - 3 + i])


@pytest.mark.parametrize("L,w", [(40, 8), (8, 8), (5, 8), (37, 16)])
def test_ring_store_decode_equals_window(L, w):
    """A sliding layer keeps its last w tokens in a ring of w rows (position
    g in row g % w): decode over the ring's min(L, w) rows, in ring order,
    equals the window attention over the full cache."""
    Hq, Hk, D = 4, 2, 64
    k, v, ks, vs = _cache(1, Hk, L, D, "per_token", seed=6)
    n = min(L, w)
    rk = torch.zeros(1, Hk, w, D, dtype=torch.uint8)
    rv = torch.zeros_like(rk)
    rks, rvs = torch.zeros(1, Hk, w, 1), torch.zeros(1, Hk, w, 1)
    for gpos in range(L - n, L):
        rk[:, :, gpos % w], rv[:, :, gpos % w] = k[:, :, gpos], v[:, :, gpos]
        rks[:, :, gpos % w], rvs[:, :, gpos % w] = ks[:, :, gpos], vs[:, :, gpos]
    q = torch.randn(1, Hq, D).to(torch.bfloat16)
    ring = oracle.decode_attn(q, rk, rv, rks, rvs, torch.tensor([n], dtype=torch.int32))
    full = oracle.window_attn(q, k, v, ks, vs, torch.tensor([L], dtype=torch.int32), w)
    assert torch.allclose(ring, full, atol=1e-13, rtol=1e-11)


def test_window_paged_equals_contiguous_and_length_rules():
    Hq, Hk, D, L = 4, 2, 64, 45
    k, v, ks, vs = _cache(1, Hk, L, D, "per_token", seed=7)
    pages = 3
    perm = torch.tensor([2, 0, 1], dtype=torch.int32)
    ak = torch.zeros(pages, Hk, 16, D, dtype=torch.uint8)
    av = torch.zeros_like(ak)
    aks, avs = torch.zeros(pages, Hk, 16, 1), torch.zeros(pages, Hk, 16, 1)
    for t in range(L):
        ph, sl = int(perm[t // 16]), t % 16
        ak[ph, :, sl], av[ph, :, sl] = k[0, :, t], v[0, :, t]
        aks[ph, :, sl], avs[ph, :, sl] = ks[0, :, t], vs[0, :, t]
    q = torch.randn(1, Hq, 3, D).to(torch.bfloat16)
    lens = torch.tensor([L], dtype=torch.int32)
    a = oracle.window_attn(q, k, v, ks, vs, lens, 9)
    b = oracle.window_attn(q, ak, av, aks, avs, lens, 9, page_size=16, table=perm.view(1, 3))
    assert torch.equal(a, b)
    out, err = oracle.window_attn(q, k, v, ks, vs, torch.tensor([2], dtype=torch.int32), 9,
                                  return_err=True)
    assert err == oracle.ORACLE_ERR_LEN and torch.all(out == 0)

"""Pins for the oracle's fp64 chunk attention (T new queries per sequence,
causal from the chunk's end; CPU only).

Anchors: an independent library routine (torch's float64
scaled_dot_product_attention with an explicit boolean mask built here), the
already pinned decode oracle on truncated caches (row i of a chunk is a
decode over the first L - T + i + 1 positions), a closed form (the first
query of a chunk that fills the cache sees one key), the length rules, and
contiguous vs paged placement.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

ORACLE_ERR_LEN = 4


def _cache(B, Hk, S, D, mode, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, Hk, S, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hk, S, D, generator=g).to(torch.bfloat16)
    kq, ks = oracle.quantize(k, mode)
    vq, vs = oracle.quantize(v, mode)
    return kq, ks, vq, vs


def _deq64(q, s, D):
    grp = D // s.shape[-1]
    exact = (q.numpy().astype(np.float64) - 128.0) * np.repeat(
        s.numpy().astype(np.float64), grp, axis=-1)
    return torch.from_numpy(exact.astype(np.float32).astype(np.float64))


def _q(B, Hq, T, D, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, Hq, T, D, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("mode,D", [("per_token", 64), ("group32", 64), ("per_token", 32)])
@pytest.mark.parametrize("G,T", [(1, 3), (4, 2), (2, 5)])
def test_matches_torch_sdpa_with_causal_mask(mode, D, G, T):
    B, Hk, S = 3, 2, 30
    Hq = Hk * G
    kq, ks, vq, vs = _cache(B, Hk, S, D, mode, seed=5 + G + T)
    lens = [T, 17, 30]
    q = _q(B, Hq, T, D, seed=9)
    sc = 1.0 / math.sqrt(D)
    out = oracle.chunk_attn(q, kq, vq, ks, vs, torch.tensor(lens, dtype=torch.int32), sc, mode)
    kd, vd = _deq64(kq, ks, D), _deq64(vq, vs, D)
    for b, L in enumerate(lens):
        kk = kd[b, :, :L].repeat_interleave(G, dim=0)[None]          # [1,Hq,L,D]
        vv = vd[b, :, :L].repeat_interleave(G, dim=0)[None]
        qq = q[b].double()[None]                                     # [1,Hq,T,D]
        # query i sits at position L - T + i and may see keys at positions <= it
        qpos = torch.arange(L - T, L).view(T, 1)
        kpos = torch.arange(L).view(1, L)
        allowed = kpos <= qpos
        ref = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=allowed, scale=sc)[0]
        assert torch.allclose(out[b], ref, rtol=1e-12, atol=1e-12), (b, mode, D, G, T)


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_row_i_is_decode_over_the_first_visible_positions(mode):
    B, Hk, G, S, D, T = 2, 2, 2, 40, 64, 4
    kq, ks, vq, vs = _cache(B, Hk, S, D, mode, seed=21)
    q = _q(B, Hk * G, T, D, seed=22)
    lens = torch.tensor([40, 9], dtype=torch.int32)
    out = oracle.chunk_attn(q, kq, vq, ks, vs, lens, None, mode)
    for i in range(T):
        trunc = lens - T + i + 1
        ref = oracle.decode_attn(q[:, :, i].contiguous(), kq, vq, ks, vs, trunc, None, mode)
        assert torch.equal(out[:, :, i], ref), i


def test_single_query_equals_decode():
    B, Hk, G, S, D = 3, 2, 4, 50, 64
    kq, ks, vq, vs = _cache(B, Hk, S, D, "per_token", seed=31)
    q = _q(B, Hk * G, 1, D, seed=32)
    lens = torch.tensor([1, 33, 50], dtype=torch.int32)
    out = oracle.chunk_attn(q, kq, vq, ks, vs, lens)
    ref = oracle.decode_attn(q[:, :, 0].contiguous(), kq, vq, ks, vs, lens)
    assert torch.equal(out[:, :, 0], ref)


def test_chunk_filling_the_cache_first_query_sees_one_key():
    B, Hk, G, S, D, T = 1, 1, 3, 6, 32, 6
    kq, ks, vq, vs = _cache(B, Hk, S, D, "per_token", seed=41)
    q = _q(B, Hk * G, T, D, seed=42)
    out = oracle.chunk_attn(q, kq, vq, ks, vs, torch.tensor([T], dtype=torch.int32))
    v0 = _deq64(vq, vs, D)[0, 0, 0]
    for h in range(G):
        assert torch.equal(out[0, h, 0], v0)             # softmax over one key is 1


def test_length_rules():
    B, Hk, S, D, T = 3, 1, 8, 32, 4
    kq, ks, vq, vs = _cache(B, Hk, S, D, "per_token", seed=51)
    q = _q(B, Hk, T, D, seed=52)
    out, err = oracle.chunk_attn(q, kq, vq, ks, vs, torch.tensor([0, 3, 8], dtype=torch.int32),
                                 return_err=True)
    assert err & ORACLE_ERR_LEN                          # 0 < L < T
    assert torch.count_nonzero(out[0]) == 0              # empty sequence: zero rows
    assert torch.count_nonzero(out[1]) == 0              # rejected length: zero rows
    assert torch.count_nonzero(out[2]) > 0
    _, err = oracle.chunk_attn(q, kq, vq, ks, vs, torch.tensor([0, 4, 8], dtype=torch.int32),
                               return_err=True)
    assert err == 0


def test_paged_placement_matches_contiguous():
    B, Hk, G, D, T, ps = 2, 2, 2, 64, 3, 16
    lens = [35, 16]
    S = max(lens)
    kq, ks, vq, vs = _cache(B, Hk, S, D, "group32", seed=61)
    q = _q(B, Hk * G, T, D, seed=62)
    sl = torch.tensor(lens, dtype=torch.int32)
    ref = oracle.chunk_attn(q, kq, vq, ks, vs, sl, None, "group32")
    need = [(L + ps - 1) // ps for L in lens]
    perm = torch.randperm(sum(need), generator=torch.Generator().manual_seed(63)).to(torch.int32)
    table = torch.full((B, max(need)), -1, dtype=torch.int32)
    ak = torch.zeros(sum(need), Hk, ps, D, dtype=torch.uint8)
    av = torch.zeros_like(ak)
    aks = torch.zeros(sum(need), Hk, ps, D // 32)
    avs = torch.zeros_like(aks)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
        for t in range(lens[b]):
            p, slot = int(table[b, t // ps]), t % ps
            ak[p, :, slot] = kq[b, :, t]
            av[p, :, slot] = vq[b, :, t]
            aks[p, :, slot] = ks[b, :, t]
            avs[p, :, slot] = vs[b, :, t]
    out = oracle.chunk_attn(q, ak, av, aks, avs, sl, None, "group32", page_size=ps, table=table)
    assert torch.equal(out, ref)

"""Pins for the oracle's fp64 decode attention (CPU only).

Anchors: an independent library routine (torch's float64
scaled_dot_product_attention on the CPU, after an independent dequantization
written here with float64 numpy), closed forms (one key, zero query,
identical keys, a dominant key), and invariances (token order, contiguous vs
paged placement, GQA head mapping, empty sequences).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _quantized_cache(B, Hk, S, D, mode, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn(B, Hk, S, D, generator=g) * sigma).to(torch.bfloat16)
    v = (torch.randn(B, Hk, S, D, generator=g) * sigma).to(torch.bfloat16)
    kq, ks = oracle.quantize(k, mode)
    vq, vs = oracle.quantize(v, mode)
    return kq, ks, vq, vs


def _deq64(q, s, D):
    """Independent dequant: (u8 - 128) * scale formed exactly in fp64 and rounded
    once to fp32 (the cache the attention reads is the fp32 dequantized one),
    returned as fp64."""
    grp = D // s.shape[-1]
    exact = (q.numpy().astype(np.float64) - 128.0) * np.repeat(
        s.numpy().astype(np.float64), grp, axis=-1)
    return exact.astype(np.float32).astype(np.float64)


def _sdpa_ref(q_bf16, kq, ks, vq, vs, seq_lens, attn_scale):
    B, Hq, D = q_bf16.shape
    Hk = kq.shape[1]
    out = torch.zeros(B, Hq, D, dtype=torch.float64)
    kd = torch.from_numpy(_deq64(kq, ks, D))
    vd = torch.from_numpy(_deq64(vq, vs, D))
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        kk = kd[b, :, :L].repeat_interleave(Hq // Hk, dim=0)[None]   # [1,Hq,L,D]
        vv = vd[b, :, :L].repeat_interleave(Hq // Hk, dim=0)[None]
        qq = q_bf16[b].double()[None, :, None, :]                   # [1,Hq,1,D]
        out[b] = F.scaled_dot_product_attention(qq, kk, vv, scale=attn_scale)[0, :, 0]
    return out


@pytest.mark.parametrize("mode,D", [("per_token", 64), ("group32", 64), ("per_token", 128),
                                    ("group32", 32)])
@pytest.mark.parametrize("G", [1, 4])
def test_matches_torch_sdpa_fp64(mode, D, G):
    B, Hk, S = 3, 2, 40
    Hq = Hk * G
    kq, ks, vq, vs = _quantized_cache(B, Hk, S, D, mode, seed=21 + D + G)
    g = torch.Generator().manual_seed(99)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    seq_lens = torch.tensor([40, 17, 1], dtype=torch.int32)
    sc = float(np.float32(1 / math.sqrt(D)))
    out = oracle.decode_attn(q, kq, vq, ks, vs, seq_lens, sc, mode)
    ref = _sdpa_ref(q, kq, ks, vq, vs, seq_lens, sc)
    assert torch.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_gqa_head_mapping_is_consecutive():
    """q head h reads kv head h // G (heads repeated consecutively)."""
    B, Hk, S, D, G = 1, 2, 8, 32, 3
    kq, ks, vq, vs = _quantized_cache(B, Hk, S, D, "per_token", seed=5)
    # make the two kv heads' values very different
    vq[0, 0] = 200
    vq[0, 1] = 50
    vs.fill_(1.0)
    q = torch.zeros(B, Hk * G, D, dtype=torch.bfloat16)
    out = oracle.decode_attn(q, kq, vq, ks, vs, torch.tensor([S], dtype=torch.int32))
    assert torch.all(out[0, :G] == 72.0) and torch.all(out[0, G:] == -78.0)


def test_single_key_returns_its_value():
    kq, ks, vq, vs = _quantized_cache(2, 1, 4, 64, "per_token", seed=8)
    q = torch.randn(2, 2, 64).to(torch.bfloat16)
    out = oracle.decode_attn(q, kq, vq, ks, vs, torch.tensor([1, 1], dtype=torch.int32))
    vhat = torch.from_numpy(_deq64(vq, vs, 64))[:, 0, 0]           # [2, D]
    assert torch.equal(out[:, 0], vhat) and torch.equal(out[:, 1], vhat)


def test_zero_query_gives_mean_and_identical_keys_give_mean():
    kq, ks, vq, vs = _quantized_cache(1, 1, 33, 64, "group32", seed=4)
    L = 33
    vmean = torch.from_numpy(_deq64(vq, vs, 64))[0, 0, :L].mean(0)
    q0 = torch.zeros(1, 1, 64, dtype=torch.bfloat16)
    out = oracle.decode_attn(q0, kq, vq, ks, vs, torch.tensor([L], dtype=torch.int32),
                             mode="group32")
    assert torch.allclose(out[0, 0], vmean, rtol=1e-13, atol=1e-13)
    kq2 = kq.clone()
    ks2 = ks.clone()
    kq2[0, 0, :] = kq[0, 0, 0]
    ks2[0, 0, :] = ks[0, 0, 0]
    q = torch.randn(1, 1, 64).to(torch.bfloat16)
    out2 = oracle.decode_attn(q, kq2, vq, ks2, vs, torch.tensor([L], dtype=torch.int32),
                              mode="group32")
    assert torch.allclose(out2[0, 0], vmean, rtol=1e-13, atol=1e-13)


def test_dominant_key_selects_its_value():
    kq, ks, vq, vs = _quantized_cache(1, 1, 20, 64, "per_token", seed=6)
    q = torch.ones(1, 1, 64, dtype=torch.bfloat16)
    kq[0, 0, 11] = 255          # k_hat = 127 * s, aligned with q
    ks[0, 0, 11] = 1.0
    out = oracle.decode_attn(q, kq, vq, ks, vs, torch.tensor([20], dtype=torch.int32),
                             attn_scale=1.0)
    vhat = torch.from_numpy(_deq64(vq, vs, 64))[0, 0, 11]
    assert torch.allclose(out[0, 0], vhat, rtol=0, atol=1e-12)


def test_token_permutation_invariance():
    kq, ks, vq, vs = _quantized_cache(1, 2, 50, 64, "per_token", seed=12)
    q = torch.randn(1, 4, 64).to(torch.bfloat16)
    sl = torch.tensor([50], dtype=torch.int32)
    out = oracle.decode_attn(q, kq, vq, ks, vs, sl)
    perm = torch.randperm(50, generator=torch.Generator().manual_seed(1))
    out_p = oracle.decode_attn(q, kq[:, :, perm].contiguous(), vq[:, :, perm].contiguous(),
                               ks[:, :, perm].contiguous(), vs[:, :, perm].contiguous(), sl)
    assert torch.allclose(out, out_p, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_paged_equals_contiguous(mode):
    B, Hk, D, ps = 3, 2, 64, 16
    lens = [37, 16, 1]
    S = max(lens)
    kq, ks, vq, vs = _quantized_cache(B, Hk, S, D, mode, seed=30)
    q = torch.randn(B, Hk * 4, D).to(torch.bfloat16)
    sl = torch.tensor(lens, dtype=torch.int32)
    ref = oracle.decode_attn(q, kq, vq, ks, vs, sl, mode=mode)
    need = [(L + ps - 1) // ps for L in lens]
    num_pages = sum(need) + 2
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(2)).to(torch.int32)
    max_pages = max(need)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    off = 0
    NG = ks.shape[-1]
    ka = torch.zeros(num_pages, Hk, ps, D, dtype=torch.uint8)
    va = torch.zeros_like(ka)
    ksa = torch.zeros(num_pages, Hk, ps, NG)
    vsa = torch.zeros_like(ksa)
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
        for t in range(lens[b]):
            p, s = int(table[b, t // ps]), t % ps
            ka[p, :, s] = kq[b, :, t]
            va[p, :, s] = vq[b, :, t]
            ksa[p, :, s] = ks[b, :, t]
            vsa[p, :, s] = vs[b, :, t]
    out = oracle.decode_attn(q, ka, va, ksa, vsa, sl, mode=mode, page_size=ps, table=table)
    assert torch.equal(out, ref)


def test_empty_sequence_and_bad_page_flag():
    kq, ks, vq, vs = _quantized_cache(2, 1, 16, 32, "per_token", seed=1)
    q = torch.randn(2, 1, 32).to(torch.bfloat16)
    out, err = oracle.decode_attn(q, kq, vq, ks, vs, torch.tensor([0, 16], dtype=torch.int32),
                                  return_err=True)
    assert err == 0 and torch.all(out[0] == 0)
    table = torch.tensor([[0], [5]], dtype=torch.int32)   # page 5 >= num_pages (2)
    out, err = oracle.decode_attn(q, kq, vq, ks, vs, torch.tensor([3, 3], dtype=torch.int32),
                                  page_size=16, table=table, return_err=True)
    assert err == oracle.ORACLE_ERR_PAGE and torch.all(out[1] == 0)

"""Pins of the oracle's other scale granularities and of the mixed cache
(abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs, QuantGranularity,
quantize_with_granularity, DynamicQuantConfig, OptimizedQuantizedKvCache):

* per-head calibration equals the pinned per-token quantiser applied to the
  whole block as one row; per-channel calibration equals it applied to each
  channel's column (bit-exact bytes and scales);
* grid data round-trips exactly; quantising with stored scales stays within
  half a step in range and clamps outside it;
* attention over per-head / per-channel caches and over the mixed cache
  against torch fp64 SDPA on values dequantised in the test;
* the page's own window bookkeeping tests (test_per_head_quantization,
  test_dynamic_quantization_window) and memory-savings bar;
* the mixed cache with no window is the pinned decode attention, and the
  tokens it quantises are the pinned per-token quantiser's bytes."""
import math

import pytest
import torch

import oracle


def _block(B, Hk, T, D, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, Hk, T, D, generator=g) * sigma).to(torch.bfloat16)


@pytest.mark.parametrize("T", [1, 5, 40])
def test_per_head_is_per_token_of_the_block(T):
    B, Hk, D = 2, 3, 64
    x = _block(B, Hk, T, D, seed=T)
    cache = torch.zeros(B, Hk, T, D, dtype=torch.uint8)
    sc = torch.zeros(B, Hk, 1)
    assert oracle.append_static(x, torch.zeros(B, dtype=torch.int32), cache, sc, "per_head") == 0
    q, s = oracle.quantize(x.reshape(B, Hk, 1, T * D), "per_token")
    assert torch.equal(cache.reshape(B, Hk, 1, T * D), q)
    assert torch.equal(sc.view(torch.int32), s.reshape(B, Hk, 1).view(torch.int32))


@pytest.mark.parametrize("T", [1, 7, 64])
def test_per_channel_is_per_token_of_each_column(T):
    B, Hk, D = 2, 2, 64
    x = _block(B, Hk, T, D, seed=10 + T)
    cache = torch.zeros(B, Hk, T, D, dtype=torch.uint8)
    sc = torch.zeros(B, Hk, D)
    assert oracle.append_static(x, torch.zeros(B, dtype=torch.int32), cache, sc,
                                "per_channel") == 0
    q, s = oracle.quantize(x.transpose(2, 3).contiguous(), "per_token")   # rows = channels
    assert torch.equal(cache, q.transpose(2, 3))
    assert torch.equal(sc.view(torch.int32), s.reshape(B, Hk, D).view(torch.int32))


@pytest.mark.parametrize("gran", ["per_head", "per_channel"])
def test_grid_roundtrip_exact(gran):
    """x = n / 2 with n in [-127, 127] and 63.5 present in every channel:
    scale 0.5 exactly, bytes n + 128 (after combs-models 0.2.2,
    kv_quant_roundtrip_exact_on_grid_values)."""
    B, Hk, T, D = 1, 2, 6, 32
    g = torch.Generator().manual_seed(4)
    n = torch.randint(-127, 128, (B, Hk, T, D), generator=g)
    n[:, :, 0, :] = 127
    x = (n.float() / 2).to(torch.bfloat16)
    cache = torch.zeros(B, Hk, T, D, dtype=torch.uint8)
    sc = torch.zeros(B, Hk, 1 if gran == "per_head" else D)
    oracle.append_static(x, torch.zeros(B, dtype=torch.int32), cache, sc, gran)
    assert torch.all(sc == 0.5)
    assert torch.equal(cache.long(), n + 128)


@pytest.mark.parametrize("gran", ["per_head", "per_channel"])
def test_stored_scales_half_step_and_clamp(gran):
    B, Hk, T, D = 1, 2, 9, 64
    x0 = _block(B, Hk, T, D, seed=5)
    cache = torch.zeros(B, Hk, 2 * T, D, dtype=torch.uint8)
    sc = torch.zeros(B, Hk, 1 if gran == "per_head" else D)
    oracle.append_static(x0, torch.zeros(B, dtype=torch.int32), cache, sc, gran)
    saved = sc.clone()
    x1 = _block(B, Hk, T, D, seed=6, sigma=1.5)          # partly beyond the calibrated range
    assert oracle.append_static(x1, torch.full((B,), T, dtype=torch.int32), cache, sc, gran,
                                calibrate=False) == 0
    assert torch.equal(sc, saved)                        # stored scales are only read
    s = sc if gran == "per_channel" else sc.expand(B, Hk, D)
    s = s.unsqueeze(2)
    xf = x1.float()
    deq = (cache[:, :, T:].float() - 128) * s
    inside = xf.abs() <= 127 * s
    # half a step, plus the rounding of the fp32 products on both sides
    bound = s.expand_as(xf) / 2 + 2 * torch.finfo(torch.float32).eps * xf.abs()
    assert torch.all((deq - xf).abs()[inside] <= bound[inside])
    # beyond the range the byte clamps: 255 (+127 s) above, 0 (-128 s) below
    hi, lo = xf > 127.5 * s, xf < -128.5 * s
    assert hi.any() and lo.any()
    assert torch.all(cache[:, :, T:][hi] == 255) and torch.all(cache[:, :, T:][lo] == 0)


@pytest.mark.parametrize("gran", ["per_head", "per_channel"])
@pytest.mark.parametrize("T,window", [(1, 0), (4, 0), (1, 7)])
def test_static_attention_vs_sdpa(gran, T, window):
    B, Hq, Hk, D, S = 2, 8, 2, 64, 50
    x, y = _block(B, Hk, S, D, seed=7), _block(B, Hk, S, D, seed=8)
    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
    v = torch.zeros_like(k)
    ns = 1 if gran == "per_head" else D
    ks, vs = torch.zeros(B, Hk, ns), torch.zeros(B, Hk, ns)
    z = torch.zeros(B, dtype=torch.int32)
    oracle.append_static(x, z, k, ks, gran)
    oracle.append_static(y, z, v, vs, gran)
    lens = torch.tensor([50, 21], dtype=torch.int32)
    q = _block(B, Hq, T, D, seed=9)
    sc = 1.0 / math.sqrt(D)
    got = oracle.static_attn(q if T > 1 else q[:, :, 0], k, v, ks, vs, lens, gran, window, sc)
    sk = ks.unsqueeze(2).expand(B, Hk, S, D) if gran == "per_channel" else ks.unsqueeze(3)
    sv = vs.unsqueeze(2).expand(B, Hk, S, D) if gran == "per_channel" else vs.unsqueeze(3)
    kd = ((k.float() - 128) * sk).double()
    vd = ((v.float() - 128) * sv).double()
    ref = torch.zeros(B, Hq, T, D, dtype=torch.float64)
    for b in range(B):
        L = int(lens[b])
        kp, qp = torch.arange(L).view(1, L), torch.arange(L - T, L).view(T, 1)
        bad = (kp > qp) | ((kp + window - 1 < qp) if window else torch.zeros_like(kp > qp))
        ref[b] = torch.nn.functional.scaled_dot_product_attention(
            q[b].double(), kd[b, :, :L].repeat_interleave(Hq // Hk, 0),
            vd[b, :, :L].repeat_interleave(Hq // Hk, 0),
            attn_mask=(~bad).unsqueeze(0).expand(Hq, T, L), scale=sc)
    assert torch.allclose(got.reshape(ref.shape), ref, atol=1e-12, rtol=1e-10)


class Mixed:
    """Oracle mixed cache (INT8 part + bf16 window ring) for one mode."""

    def __init__(self, B, Hk, S, D, W, mode, static_from=None):
        self.B, self.Hk, self.D, self.W, self.mode = B, Hk, D, W, mode
        self.k = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
        self.v = torch.zeros_like(self.k)
        if mode in ("per_token", "group32"):
            ng = 1 if mode == "per_token" else D // 32
            self.ks, self.vs = torch.zeros(B, Hk, S, ng), torch.zeros(B, Hk, S, ng)
        else:
            self.ks, self.vs = static_from
        self.rk = torch.zeros(B, Hk, max(W, 1), D, dtype=torch.bfloat16)
        self.rv = torch.zeros_like(self.rk)
        self.lens = torch.zeros(B, dtype=torch.int32)

    def append(self, xk, xv):
        e = oracle.append_mixed(xk, self.lens, self.k, self.ks, self.rk, self.mode, self.W)
        e |= oracle.append_mixed(xv, self.lens, self.v, self.vs, self.rv, self.mode, self.W)
        self.lens += xk.shape[2]
        return e

    def attn(self, q):
        return oracle.mixed_attn(q, self.k, self.v, self.ks, self.vs, self.rk, self.rv,
                                 self.lens, self.mode, window=self.W)


def test_page_window_bookkeeping():
    """test_per_head_quantization: window 4, 10 tokens -> 6 quantised, 4
    recent; test_dynamic_quantization_window: window 8, 5 tokens -> 0 and 5,
    5 more -> 2 and 8 (INT8 rows are the ones written)."""
    B, Hk, D = 1, 4, 64
    for W, steps, want in [(4, [10], [6]), (8, [5, 5], [0, 2])]:
        m = Mixed(B, Hk, 16, D, W, "per_token")
        m.k.fill_(0xEE)
        for i, (n, q) in enumerate(zip(steps, want)):
            assert m.append(_block(B, Hk, n, D, seed=n + i), _block(B, Hk, n, D, seed=99)) == 0
            L = int(m.lens[0])
            written = int((m.k[0, 0, :, 0] != 0xEE).sum())
            assert written == q == max(0, L - W)
            assert min(L, W) == L - q                       # recent length


def test_page_memory_savings_bar():
    """test_memory_savings: 1000 tokens, window 16, 8 kv heads x 128: the full
    bf16 cache over the mixed cache's bytes (INT8 values + fp32 scales +
    the bf16 window) is above 1.5."""
    L, W, Hk, D = 1000, 16, 8, 128
    full = L * Hk * D * 2 * 2
    mixed = 2 * ((L - W) * Hk * D + (L - W) * Hk * 4 + W * Hk * D * 2)
    assert full / mixed > 1.5


@pytest.mark.parametrize("mode", ["per_token", "group32", "per_head", "per_channel"])
def test_mixed_attention_vs_sdpa(mode):
    B, Hq, Hk, D, S, W = 2, 8, 2, 64, 60, 8
    static = None
    if mode in ("per_head", "per_channel"):
        ns = 1 if mode == "per_head" else D
        ks, vs = torch.zeros(B, Hk, ns), torch.zeros(B, Hk, ns)
        tmp = torch.zeros(B, Hk, 20, D, dtype=torch.uint8)
        z = torch.zeros(B, dtype=torch.int32)
        oracle.append_static(_block(B, Hk, 20, D, seed=1), z, tmp, ks, mode)    # calibration
        oracle.append_static(_block(B, Hk, 20, D, seed=2), z, tmp, vs, mode)
        static = (ks, vs)
    m = Mixed(B, Hk, S, D, W, mode, static)
    hist_k, hist_v = _block(B, Hk, 45, D, seed=3), _block(B, Hk, 45, D, seed=4)
    m.append(hist_k[:, :, :30], hist_v[:, :, :30])                    # a prefill
    for t in range(30, 45):                                           # decode steps
        m.append(hist_k[:, :, t:t + 1], hist_v[:, :, t:t + 1])
    q = _block(B, Hq, 1, D, seed=5)[:, :, 0]
    got = m.attn(q)
    L = 45
    Lq = L - W
    if mode in ("per_token", "group32"):
        kd = oracle.dequant(m.k[:, :, :Lq].contiguous(), m.ks[:, :, :Lq].contiguous(), mode)
        vd = oracle.dequant(m.v[:, :, :Lq].contiguous(), m.vs[:, :, :Lq].contiguous(), mode)
    else:
        sk = static[0].unsqueeze(2) if mode == "per_channel" else static[0].unsqueeze(3)
        sv = static[1].unsqueeze(2) if mode == "per_channel" else static[1].unsqueeze(3)
        kd = (m.k[:, :, :Lq].float() - 128) * sk
        vd = (m.v[:, :, :Lq].float() - 128) * sv
    kr = torch.stack([m.rk[:, :, g % W] for g in range(Lq, L)], 2).float()
    vr = torch.stack([m.rv[:, :, g % W] for g in range(Lq, L)], 2).float()
    kk = torch.cat([kd, kr], 2).double().repeat_interleave(Hq // Hk, 1)
    vv = torch.cat([vd, vr], 2).double().repeat_interleave(Hq // Hk, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().unsqueeze(2), kk, vv, scale=1.0 / math.sqrt(D))[:, :, 0]
    assert torch.allclose(got, ref, atol=1e-12, rtol=1e-10)
    # the window holds the newest tokens as they came
    for g in range(Lq, L):
        assert torch.equal(m.rk[:, :, g % W], hist_k[:, :, g])


def test_mixed_without_window_is_plain_decode_and_quantises_like_append():
    B, Hq, Hk, D, S = 2, 4, 2, 64, 40
    m = Mixed(B, Hk, S, D, 0, "per_token")
    xk, xv = _block(B, Hk, 33, D, seed=6), _block(B, Hk, 33, D, seed=7)
    m.append(xk[:, :, :20], xv[:, :, :20])
    m.append(xk[:, :, 20:], xv[:, :, 20:])
    k2 = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
    ks2 = torch.zeros(B, Hk, S, 1)
    oracle.append_contig(xk, torch.zeros(B, dtype=torch.int32), k2, ks2)
    assert torch.equal(m.k, k2) and torch.equal(m.ks, ks2)
    q = _block(B, Hq, 1, D, seed=8)[:, :, 0]
    ref = oracle.decode_attn(q, m.k, m.v, m.ks, m.vs, m.lens)
    assert torch.allclose(m.attn(q), ref, atol=1e-13, rtol=1e-12)


def test_mixed_window_covering_everything_is_bf16_attention():
    B, Hq, Hk, D, W = 1, 4, 1, 64, 64
    m = Mixed(B, Hk, 64, D, W, "per_token")
    xk, xv = _block(B, Hk, 50, D, seed=9), _block(B, Hk, 50, D, seed=10)
    m.append(xk, xv)
    assert torch.all(m.k == 0)                          # nothing quantised
    q = _block(B, Hq, 1, D, seed=11)[:, :, 0]
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().unsqueeze(2), xk.double().repeat_interleave(Hq, 1),
        xv.double().repeat_interleave(Hq, 1), scale=1.0 / math.sqrt(D))[:, :, 0]
    assert torch.allclose(m.attn(q), ref, atol=1e-12, rtol=1e-10)


@pytest.mark.parametrize("mode", ["per_token", "group32", "per_head", "per_channel"])
def test_mixed_int8_part_is_the_pinned_quantiser(mode):
    """Whatever the append pattern, the INT8 part holds exactly the bytes (and
    per-token scales) the pinned quantisers give the same tokens."""
    B, Hk, D, S, W = 2, 2, 64, 64, 5
    static = None
    if mode in ("per_head", "per_channel"):
        ns = 1 if mode == "per_head" else D
        ks, vs = torch.zeros(B, Hk, ns), torch.zeros(B, Hk, ns)
        tmp = torch.zeros(B, Hk, 8, D, dtype=torch.uint8)
        z = torch.zeros(B, dtype=torch.int32)
        oracle.append_static(_block(B, Hk, 8, D, seed=21), z, tmp, ks, mode)
        oracle.append_static(_block(B, Hk, 8, D, seed=22), z, tmp, vs, mode)
        static = (ks, vs)
    m = Mixed(B, Hk, S, D, W, mode, static)
    hk, hv = _block(B, Hk, 40, D, seed=23), _block(B, Hk, 40, D, seed=24)
    for a, b in [(0, 3), (3, 4), (4, 17), (17, 18), (18, 40)]:
        m.append(hk[:, :, a:b], hv[:, :, a:b])
    Lq = 40 - W
    ref = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
    z = torch.zeros(B, dtype=torch.int32)
    if mode in ("per_token", "group32"):
        rs = torch.zeros_like(m.ks)
        oracle.append_contig(hk[:, :, :Lq].contiguous(), z, ref, rs, mode)
        assert torch.equal(m.ks[:, :, :Lq], rs[:, :, :Lq])
    else:
        oracle.append_static(hk[:, :, :Lq].contiguous(), z, ref, static[0].clone(), mode,
                             calibrate=False)
    assert torch.equal(m.k[:, :, :Lq], ref[:, :, :Lq])
    assert torch.all(m.k[:, :, Lq:] == 0)

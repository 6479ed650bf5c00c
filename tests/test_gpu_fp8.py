"""GPU parity of the FP8 KV format (KVQ_FP8_E4M3 / KVQ_FP8_E5M2): appended
bytes bit-exact with the oracle's truncating encoders (contiguous and paged,
decode tokens and chunks, values across the whole range: subnormals, zeros
of both signs, saturation), dequant bit-exact with the oracle's decoders,
and decode / chunk / window attention on the FP8 cache within the fp64 bar
of the oracle (max-abs 2e-3, relative-L2 1e-3)."""
import pytest
import torch

import oracle
from kvq_testutil import assert_attn_close, bf16_randn, f32_scale, kvq

pytestmark = pytest.mark.gpu
FMTS = ["fp8_e4m3", "fp8_e5m2"]


def _wide_values(shape, seed):
    """bf16 values over many magnitudes: N(0,1) times 2^u, u uniform in [-20, 18],
    plus exact zeros of both signs."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * torch.pow(2.0, torch.randint(-20, 19, shape,
                                                                         generator=g).float())
    flat = x.view(-1)
    flat[::97] = 0.0
    flat[1::97] = -0.0
    return x.to(torch.bfloat16)


class Fp8Cache:
    def __init__(self, B, Hk, S, D, fmt, dev="cuda"):
        self.fmt = fmt
        self.k = torch.full((B, Hk, S, D), 0xCD, dtype=torch.uint8, device=dev)
        self.v = torch.full_like(self.k, 0xCD)
        self.ok = torch.full((B, Hk, S, D), 0xCD, dtype=torch.uint8)
        self.ov = torch.full_like(self.ok, 0xCD)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def append(self, kn, vn, pos):
        m = kvq()
        m.kvq_append(kn.cuda(), vn.cuda(), pos.cuda(), self.k, self.v, None, None, self.fmt,
                     err=self.err)
        return oracle.append_fp8(kn, pos, self.ok, self.fmt) | \
            oracle.append_fp8(vn, pos, self.ov, self.fmt)

    def bit_exact(self):
        torch.cuda.synchronize()
        return torch.equal(self.k.cpu(), self.ok) and torch.equal(self.v.cpu(), self.ov)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D,T", [(64, 1), (128, 1), (128, 33), (256, 5), (16, 3)])
def test_fp8_append_bit_exact(fmt, D, T):
    B, Hk, S = 3, 2, 80
    c = Fp8Cache(B, Hk, S, D, fmt)
    kn, vn = _wide_values((B, Hk, T, D), 1 + D + T), _wide_values((B, Hk, T, D), 2 + D + T)
    pos = torch.tensor([0, 7, S - T], dtype=torch.int32)
    assert c.append(kn, vn, pos) == 0
    assert c.bit_exact()
    # a range past the capacity is skipped and flagged on both sides
    bad = torch.tensor([S - T + 1, 0, 3], dtype=torch.int32)
    assert c.append(kn, vn, bad) == oracle.ORACLE_ERR_POS
    assert kvq().kvq_read_error(c.err) == 1
    assert c.bit_exact()


@pytest.mark.parametrize("fmt", FMTS)
def test_fp8_append_paged_bit_exact(fmt):
    m = kvq()
    Hk, D, T, npg = 2, 128, 21, 6
    table = torch.tensor([[4, 1, -1], [0, 5, 2]], dtype=torch.int32)
    k = torch.zeros(npg, Hk, 16, D, dtype=torch.uint8, device="cuda")
    v = torch.zeros_like(k)
    ok, ov = torch.zeros(npg, Hk, 16, D, dtype=torch.uint8), torch.zeros(npg, Hk, 16, D,
                                                                          dtype=torch.uint8)
    kn, vn = _wide_values((2, Hk, T, D), 5), _wide_values((2, Hk, T, D), 6)
    pos = torch.tensor([3, 20], dtype=torch.int32)
    m.kvq_append_paged(kn.cuda(), vn.cuda(), pos.cuda(), k, v, None, None, table.cuda(), 16, fmt)
    assert oracle.append_fp8(kn, pos, ok, fmt, 16, table) == 0
    assert oracle.append_fp8(vn, pos, ov, fmt, 16, table) == 0
    torch.cuda.synchronize()
    assert torch.equal(k.cpu(), ok) and torch.equal(v.cpu(), ov)


@pytest.mark.parametrize("fmt", FMTS)
def test_fp8_dequant_bit_exact(fmt):
    m = kvq()
    codes = torch.arange(256, dtype=torch.uint8).repeat(64).view(-1, 128)
    got = m.kvq_dequant(codes.cuda(), None, fmt).cpu()
    ref = oracle.fp8_decode(codes, fmt)
    nan = torch.isnan(ref)
    assert torch.equal(torch.isnan(got), nan)
    assert torch.equal(got[~nan].view(torch.int32) & 0x7fffffff,
                       ref[~nan].view(torch.int32) & 0x7fffffff)
    assert torch.equal(got[~nan], ref[~nan])


def _filled(B, Hk, D, fmt, lens, seed, sigma):
    S = max(max(lens), 1)
    c = Fp8Cache(B, Hk, S, D, fmt)
    L = max(lens)
    if L:
        assert c.append(bf16_randn((B, Hk, L, D), seed, sigma),
                        bf16_randn((B, Hk, L, D), seed + 1, sigma),
                        torch.zeros(B, dtype=torch.int32)) == 0
    return c


def _attn(c, q, sl, hint, window=0, **kw):
    m = kvq()
    D = q.shape[-1]
    if window:
        return m.kvq_window_attn(q.cuda(), c.k, c.v, None, None, sl.cuda(), hint, window,
                                 mode=c.fmt, attn_scale=f32_scale(D), err=c.err, **kw)
    call = m.kvq_decode_attn if q.dim() == 3 else m.kvq_chunk_attn
    return call(q.cuda(), c.k, c.v, None, None, sl.cuda(), hint, mode=c.fmt,
                attn_scale=f32_scale(D), err=c.err, **kw)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_fp8_decode_matches_oracle(fmt, D, G):
    B, Hk = 3, 2
    lens = [1, 129, 2500]
    c = _filled(B, Hk, D, fmt, lens, seed=G + D, sigma=2.0)
    q = bf16_randn((B, Hk * G, D), seed=G)
    sl = torch.tensor(lens, dtype=torch.int32)
    ref = oracle.fp8_attn(q, c.ok, c.ov, sl, fmt, 0, f32_scale(D))
    for ns in (0, 1, 5):
        assert_attn_close(_attn(c, q, sl, max(lens), num_splits=ns), ref,
                          f"{fmt} D={D} G={G} ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_fp8_many_units_chunks_windows(fmt):
    B, Hk, D = 24, 4, 128
    lens = [0, 1, 16, 17, 300, 1000, 3000, 5] * 3
    c = _filled(B, Hk, D, fmt, lens, seed=3, sigma=0.7)
    sl = torch.tensor(lens, dtype=torch.int32)
    q1 = bf16_randn((B, Hk * 4, D), seed=4)
    assert_attn_close(_attn(c, q1, sl, max(lens)),
                      oracle.fp8_attn(q1, c.ok, c.ov, sl, fmt, 0, f32_scale(D)), "many units")
    lens4 = [max(L, 4) for L in lens]
    sl4 = torch.tensor(lens4, dtype=torch.int32)
    q4 = bf16_randn((B, Hk * 2, 4, D), seed=5)
    assert_attn_close(_attn(c, q4, sl4, max(lens4)),
                      oracle.fp8_attn(q4, c.ok, c.ov, sl4, fmt, 0, f32_scale(D)), "chunk T=4")
    for w in (20, 333):
        assert_attn_close(_attn(c, q1, sl, max(lens), window=w),
                          oracle.fp8_attn(q1, c.ok, c.ov, sl, fmt, w, f32_scale(D)),
                          f"window {w}")


@pytest.mark.parametrize("fmt", FMTS)
def test_fp8_paged_decode(fmt):
    m = kvq()
    Hk, G, D = 2, 4, 128
    lens = [40, 700]
    need = [(L + 15) // 16 for L in lens]
    npg = sum(need)
    perm = torch.randperm(npg, generator=torch.Generator().manual_seed(2)).to(torch.int32)
    table = torch.full((2, max(need)), -1, dtype=torch.int32)
    table[0, :need[0]] = perm[:need[0]]
    table[1, :need[1]] = perm[need[0]:]
    k = torch.zeros(npg, Hk, 16, D, dtype=torch.uint8, device="cuda")
    v = torch.zeros_like(k)
    ok, ov = torch.zeros(npg, Hk, 16, D, dtype=torch.uint8), torch.zeros(npg, Hk, 16, D,
                                                                          dtype=torch.uint8)
    for b, L in enumerate(lens):
        kn, vn = bf16_randn((1, Hk, L, D), 10 + b), bf16_randn((1, Hk, L, D), 20 + b)
        z = torch.zeros(1, dtype=torch.int32)
        tb = table[b:b + 1].contiguous()
        m.kvq_append_paged(kn.cuda(), vn.cuda(), z.cuda(), k, v, None, None, tb.cuda(), 16, fmt)
        oracle.append_fp8(kn, z, ok, fmt, 16, tb)
        oracle.append_fp8(vn, z, ov, fmt, 16, tb)
    sl = torch.tensor(lens, dtype=torch.int32)
    q = bf16_randn((2, Hk * G, D), seed=30)
    out = m.kvq_decode_attn(q.cuda(), k, v, None, None, sl.cuda(), max(lens),
                            page_table=table.cuda(), page_size=16, mode=fmt,
                            attn_scale=f32_scale(D))
    torch.cuda.synchronize()
    assert torch.equal(k.cpu(), ok)
    assert_attn_close(out, oracle.fp8_attn(q, ok, ov, sl, fmt, 0, f32_scale(D), page_size=16,
                                           table=table), "paged")

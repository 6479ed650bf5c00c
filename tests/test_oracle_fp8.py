"""Pins of the oracle's FP8 KV format (llama-gguf 0.14.0,
src/model/kv_quantized.rs, quantize_fp8_e4m3 / quantize_fp8_e5m2 and the
dequantize pair): hand-worked bytes of the page's own test values
(tests/golden/fp8_codes.txt), the page's round-trip tolerances, the decoder
against torch's float8 dtypes (an independent library decoder) on all 256
codes, the encoder against a brute-force definition of truncation (the
largest magnitude code not above |x|), and attention over an FP8 cache
against torch fp64 SDPA over the torch-decoded values."""
import math

import pytest
import torch

import oracle
from conftest import read_golden

TORCH_FP8 = {"fp8_e4m3": torch.float8_e4m3fn, "fp8_e5m2": torch.float8_e5m2}
MAX_FINITE = {"fp8_e4m3": 448.0, "fp8_e5m2": 57344.0}


def _torch_decode(codes, fmt):
    return codes.to(torch.uint8).view(TORCH_FP8[fmt]).to(torch.float32)


def test_golden_codes():
    _, rows = read_golden("fp8_codes.txt")
    assert len(rows) >= 20
    for fmt, val, code, dec in rows:
        got = oracle.fp8_encode_f32(float(val), fmt)
        assert got == int(code, 16), (fmt, val, hex(got), code)
        d = oracle.fp8_decode(torch.tensor([got], dtype=torch.uint8), fmt).item()
        assert d == float(dec), (fmt, val, d, dec)


@pytest.mark.parametrize("fmt,vals,tol", [
    ("fp8_e4m3", [0.0, 1.0, -1.0, 0.5, 0.0136719, 448.0, 2.0 ** -6, 2.0 ** -9], 0.05),
    ("fp8_e5m2", [0.0, 1.0, -1.0, 0.5, 57344.0, 2.0 ** -14, 1.52588e-5], 0.1)])
def test_page_roundtrip_tolerances(fmt, vals, tol):
    """The page's test_fp8_e4m3_roundtrip / test_fp8_e5m2_roundtrip bars."""
    for v in vals:
        d = oracle.fp8_decode(torch.tensor([oracle.fp8_encode_f32(v, fmt)], dtype=torch.uint8),
                              fmt).item()
        if v == 0.0:
            assert d == 0.0
        elif abs(v) < 1e-5:
            assert abs(d) < 0.01
        else:
            assert abs(v - d) / abs(v) < tol, (v, d)


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "fp8_e5m2"])
def test_decoder_matches_torch_on_every_code(fmt):
    codes = torch.arange(256, dtype=torch.uint8)
    mine = oracle.fp8_decode(codes, fmt)
    ref = _torch_decode(codes, fmt)
    nan = torch.isnan(ref)
    assert torch.equal(torch.isnan(mine), nan)
    assert torch.equal(mine[~nan], ref[~nan])          # -0 == +0 compares equal


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "fp8_e5m2"])
def test_encoder_is_truncation(fmt):
    """For finite bf16 inputs: the code with the largest magnitude not above
    |x| among the finite codes, with x's sign (a zero of x's sign below the
    smallest subnormal); E4M3 saturates at 448, E5M2 gives inf from 2^16."""
    codes = torch.arange(128, dtype=torch.uint8)
    mags = _torch_decode(codes, fmt).double()
    finite = torch.isfinite(mags)
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-4, 0.01, 1.0, 30.0, 3e3, 3e4)])
    x = torch.cat([x, torch.tensor([2.0 ** -9, -2.0 ** -16, 447.9, 480.0, 511.0, 57344.0,
                                    60000.0, 65535.0, 65536.0, 131000.0])])
    xb = x.to(torch.bfloat16)
    got = oracle.fp8_encode(xb, fmt)
    xf = xb.double()
    for i in range(xf.numel()):
        v = float(xf[i])
        a = abs(v)
        sign = 0x80 if v < 0 else 0
        if fmt == "fp8_e5m2" and a >= 65536.0:
            want = sign | 0x7C
        elif a >= MAX_FINITE[fmt]:
            want = sign | int(torch.nonzero(mags == MAX_FINITE[fmt])[0])
        else:
            ok = torch.nonzero(finite & (mags <= a)).flatten()
            want = int(ok[mags[ok].argmax()])
            want = sign | want if (want != 0 or v != 0) else 0
        assert int(got[i]) == want, (fmt, v, hex(int(got[i])), hex(want))


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "fp8_e5m2"])
def test_encode_decode_fixed_points(fmt):
    """Every finite code is reproduced by encoding its own value (0x80, minus
    zero, encodes as 0x00)."""
    codes = torch.arange(256, dtype=torch.uint8)
    vals = oracle.fp8_decode(codes, fmt)
    for c in range(256):
        v = float(vals[c])
        if not math.isfinite(v):
            continue
        want = 0 if c == 0x80 else c
        assert oracle.fp8_encode_f32(v, fmt) == want, (fmt, hex(c), v)


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "fp8_e5m2"])
@pytest.mark.parametrize("T,window", [(1, 0), (3, 0), (1, 9), (4, 6)])
def test_fp8_attention_vs_sdpa(fmt, T, window):
    B, Hq, Hk, D, S = 2, 4, 2, 64, 40
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(B, Hk, S, D, generator=g) * 3).to(torch.bfloat16)
    y = (torch.randn(B, Hk, S, D, generator=g) * 3).to(torch.bfloat16)
    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
    v = torch.zeros_like(k)
    z = torch.zeros(B, dtype=torch.int32)
    assert oracle.append_fp8(x, z, k, fmt) == 0 and oracle.append_fp8(y, z, v, fmt) == 0
    assert torch.equal(k, oracle.fp8_encode(x, fmt))
    lens = torch.tensor([40, 17], dtype=torch.int32)
    q = torch.randn(B, Hq, T, D, generator=g).to(torch.bfloat16)
    sc = 1.0 / math.sqrt(D)
    got = oracle.fp8_attn(q if T > 1 else q[:, :, 0], k, v, lens, fmt, window, sc)
    kd, vd = _torch_decode(k, fmt).double(), _torch_decode(v, fmt).double()
    ref = torch.zeros(B, Hq, T, D, dtype=torch.float64)
    for b in range(B):
        L = int(lens[b])
        kp = torch.arange(L).view(1, L)
        qp = torch.arange(L - T, L).view(T, 1)
        bad = kp > qp
        if window:
            bad = bad | (kp + window - 1 < qp)
        ref[b] = torch.nn.functional.scaled_dot_product_attention(
            q[b].double(), kd[b, :, :L].repeat_interleave(Hq // Hk, 0),
            vd[b, :, :L].repeat_interleave(Hq // Hk, 0),
            attn_mask=(~bad).unsqueeze(0).expand(Hq, T, L), scale=sc)
    assert torch.allclose(got.reshape(ref.shape), ref, atol=1e-12, rtol=1e-10)


def test_fp8_paged_append_and_attention_equal_contiguous():
    fmt, Hk, D, L = "fp8_e4m3", 2, 64, 37
    x = torch.randn(1, Hk, L, D).to(torch.bfloat16)
    k = torch.zeros(1, Hk, L, D, dtype=torch.uint8)
    z1 = torch.zeros(1, dtype=torch.int32)
    oracle.append_fp8(x, z1, k, fmt)
    table = torch.tensor([[2, 0, 1]], dtype=torch.int32)
    ak = torch.zeros(3, Hk, 16, D, dtype=torch.uint8)
    assert oracle.append_fp8(x, z1, ak, fmt, page_size=16, table=table) == 0
    for t in range(L):
        assert torch.equal(ak[int(table[0, t // 16]), :, t % 16], k[0, :, t])
    q = torch.randn(1, 4, D).to(torch.bfloat16)
    lens = torch.tensor([L], dtype=torch.int32)
    assert torch.equal(oracle.fp8_attn(q, k, k, lens, fmt),
                       oracle.fp8_attn(q, ak, ak, lens, fmt, page_size=16, table=table))
    # a range beyond the capacity is skipped and flagged
    assert oracle.append_fp8(x[:, :, :1], torch.tensor([L], dtype=torch.int32), k, fmt) == \
        oracle.ORACLE_ERR_POS

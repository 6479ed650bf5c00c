"""GPU parity: kvq_append / kvq_append_paged / kvq_dequant against the oracle,
bit-exact (bytes and fp32 scale bits), including untouched canaries around
every write, error flags, and special values."""
import pytest
import torch

import oracle
from kvq_testutil import ContigCache, PagedCache, bf16_randn, kvq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("D", [32, 64, 128, 256])
@pytest.mark.parametrize("T", [1, 7, 64])
def test_append_contig_bit_exact(mode, D, T):
    B, Hk, S = 3, 2, 80
    c = ContigCache(B, Hk, S, D, mode)
    k = bf16_randn((B, Hk, T, D), seed=D + T, sigma=1.3)
    v = bf16_randn((B, Hk, T, D), seed=D + T + 1, sigma=0.7)
    pos = torch.tensor([0, 5, S - T], dtype=torch.int32)
    assert c.append(k, v, pos) == 0
    c.assert_bit_exact()
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("D", [16, 48, 80, 112])
def test_append_odd_head_dims_per_token(D):
    """head_dim that is a multiple of 16 but not a power of two (idle lanes)."""
    B, Hk, T, S = 2, 3, 5, 9
    c = ContigCache(B, Hk, S, D, "per_token")
    k = bf16_randn((B, Hk, T, D), seed=D)
    v = bf16_randn((B, Hk, T, D), seed=D + 1)
    assert c.append(k, v, torch.tensor([1, 4], dtype=torch.int32)) == 0
    c.assert_bit_exact()


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_append_special_values(mode):
    D, T = 64, 8
    k = bf16_randn((1, 1, T, D), seed=3)
    k[0, 0, 0] = 0.0                                   # zero row: eps floor
    k[0, 0, 1, :] = 0.25 * torch.arange(D).float().to(torch.bfloat16) - 8  # grid values
    k[0, 0, 1, 0] = 63.5                               # absmax -> scale exactly 0.5
    k[0, 0, 1, 32] = -63.5
    k[0, 0, 2] = torch.tensor(1e-39, dtype=torch.bfloat16)   # subnormal bf16
    k[0, 0, 3] = k[0, 0, 3] * 1e-9                     # tiny row below the floor
    k[0, 0, 4] = k[0, 0, 4] * 3e4                      # large
    k[0, 0, 5, ::3] = -k[0, 0, 5, ::3].abs() * 40      # negative outliers
    k[0, 0, 6] = torch.tensor([0.5, -0.5, 1.5, -1.5] * (D // 4), dtype=torch.bfloat16)
    v = -k.clone()
    c = ContigCache(1, 1, T, D, mode)
    assert c.append(k, v, torch.tensor([0], dtype=torch.int32)) == 0
    c.assert_bit_exact()
    # odd symmetry holds on the GPU too: u8(-x) = 256 - u8(x)
    torch.cuda.synchronize()
    assert torch.equal(c.v.cpu().to(torch.int32), 256 - c.k.cpu().to(torch.int32))


def test_append_overwrites_slot_and_keeps_neighbours():
    c = ContigCache(2, 2, 10, 64, "group32")
    for i in range(3):
        k = bf16_randn((2, 2, 1, 64), seed=10 + i)
        v = bf16_randn((2, 2, 1, 64), seed=20 + i)
        assert c.append(k, v, torch.tensor([4, 9], dtype=torch.int32)) == 0
    c.assert_bit_exact()


def test_append_position_overflow_is_flagged_and_skipped():
    c = ContigCache(3, 2, 12, 64, "per_token")
    k = bf16_randn((3, 2, 5, 64), seed=1)
    v = bf16_randn((3, 2, 5, 64), seed=2)
    pos = torch.tensor([0, 8, -1], dtype=torch.int32)   # rows 1 and 2 out of range
    assert c.append(k, v, pos) == oracle.ORACLE_ERR_POS
    c.assert_bit_exact()                                 # skipped rows untouched on both sides
    assert kvq().kvq_read_error(c.err) == kvq().DEVERR_POS
    assert kvq().kvq_read_error(c.err) == 0              # read clears the word


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_append_paged_bit_exact_across_page_boundaries(mode):
    B, Hk, D = 3, 2, 128
    table = torch.tensor([[7, 2, 9, 0], [4, 1, -1, -1], [3, 8, 6, 5]], dtype=torch.int32)
    c = PagedCache(10, Hk, D, mode, table)
    # prefill 20 tokens crossing the first page boundary, then decode-style appends
    k = bf16_randn((B, Hk, 20, D), seed=5)
    v = bf16_randn((B, Hk, 20, D), seed=6)
    assert c.append(k, v, torch.tensor([0, 3, 11], dtype=torch.int32)) == 0
    for step in range(3):
        k1 = bf16_randn((B, Hk, 1, D), seed=100 + step)
        v1 = bf16_randn((B, Hk, 1, D), seed=200 + step)
        assert c.append(k1, v1, torch.tensor([20 + step, 23 + step, 31 + step],
                                             dtype=torch.int32)) == 0
    c.assert_bit_exact()


def test_append_paged_bad_page_is_flagged():
    table = torch.tensor([[0, 12]], dtype=torch.int32)      # page 12 >= num_pages (4)
    c = PagedCache(4, 1, 64, "per_token", table)
    k = bf16_randn((1, 1, 4, 64), seed=1)
    v = bf16_randn((1, 1, 4, 64), seed=2)
    err = c.append(k, v, torch.tensor([14], dtype=torch.int32))   # tokens 14..17
    assert err == oracle.ORACLE_ERR_PAGE
    c.assert_bit_exact()                  # tokens 14, 15 written; 16, 17 skipped
    assert kvq().kvq_read_error(c.err) == kvq().DEVERR_PAGE
    # beyond max_pages * page_size
    err = c.append(k, v, torch.tensor([30], dtype=torch.int32))
    assert err == oracle.ORACLE_ERR_POS
    assert kvq().kvq_read_error(c.err) == kvq().DEVERR_POS
    c.assert_bit_exact()


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("rows", [1, 7, 1000, 4099])
def test_dequant_bit_exact(mode, rows):
    D = 128
    g = torch.Generator().manual_seed(rows)
    q = torch.randint(0, 256, (rows, D), generator=g, dtype=torch.uint8)
    n = 1 if mode == "per_token" else D // 32
    s = torch.rand(rows, n, generator=g) * 0.1 + 1e-6
    out = kvq().kvq_dequant(q.cuda(), s.cuda(), mode)
    ref = oracle.dequant(q, s, mode)
    assert torch.equal(out.cpu().view(torch.int32), ref.view(torch.int32))


def test_dequant_roundtrip_of_appended_cache():
    c = ContigCache(2, 4, 33, 64, "group32")
    k = bf16_randn((2, 4, 33, 64), seed=8)
    v = bf16_randn((2, 4, 33, 64), seed=9)
    assert c.append(k, v, torch.tensor([0, 0], dtype=torch.int32)) == 0
    out = kvq().kvq_dequant(c.k, c.ks, "group32")
    ref = oracle.dequant(c.ok, c.oks, "group32")
    assert torch.equal(out.cpu().view(torch.int32), ref.view(torch.int32))
    # half-step bound against the bf16 source
    bound = c.oks.repeat_interleave(32, dim=-1) * (0.5 + 2.0 ** -18 + 2.0 ** -17)
    assert torch.all((ref - k.float()).abs() <= bound)


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_append_ties_and_large_sweep_bit_exact(mode):
    """The quotient x / s is taken by a reciprocal multiply away from rounding
    ties and by the IEEE division near them: rows of exact ties (max 127, so
    s = 1 and x = k + 0.5), rows of values that are ties only up to bf16
    rounding, and a sweep of 2M values over many magnitudes, all bit-exact."""
    B, Hk, T, D = 2, 4, 2048, 128
    g = torch.Generator().manual_seed(77)
    x = torch.randn(B, Hk, T, D, generator=g) * torch.pow(
        2.0, torch.randint(-12, 12, (B, Hk, T, 1), generator=g).float())
    k = torch.randint(-127, 127, (B, Hk, 64, D), generator=g).float()
    x[:, :, :64] = k + 0.5                                   # exact ties (s = 1)
    x[:, :, :64, 0] = 127.0
    m = torch.rand(B, Hk, 64, 1, generator=g) * 10 + 0.1     # near-ties after bf16 rounding
    x[:, :, 64:128] = (k + 0.5) * m / 127.0
    x[:, :, 64:128, 0] = m[..., 0]
    xb = x.to(torch.bfloat16)
    c = ContigCache(B, Hk, T, D, mode)
    assert c.append(xb, -xb, torch.zeros(B, dtype=torch.int32)) == 0
    c.assert_bit_exact()

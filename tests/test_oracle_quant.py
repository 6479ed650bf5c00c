"""Pins for the oracle's quantize / dequantize / append (CPU only).

Each check is anchored outside the oracle itself: a worked example printed
on the pages (tests/golden), a closed form, an invariant of the definition,
or an fp64 route that reaches the same correctly rounded fp32 values by a
different arithmetic path (a quotient of two binary32 numbers rounded first
to binary64 and then to binary32 equals the directly rounded binary32
quotient, since 53 >= 2*24 + 2).
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def _row_with(x_vals, absmax=63.5, D=None):
    vals = [absmax] + list(x_vals)
    D = D or len(vals)
    vals += [0.0] * (D - len(vals))
    return torch.tensor([vals], dtype=torch.bfloat16)


def _round_half_away(r: np.ndarray) -> np.ndarray:
    return np.sign(r) * np.floor(np.abs(r) + 0.5)


def _f64_route(x_bf16: torch.Tensor, group: int):
    """Bytes and scales via binary64 arithmetic rounded once to binary32."""
    x = x_bf16.float().numpy().astype(np.float64)
    D = x.shape[-1]
    xg = x.reshape(-1, D // group, group)
    m = np.abs(xg).max(axis=-1)
    m = np.maximum(m, np.float64(np.float32(1e-8)))
    s = (m / 127.0).astype(np.float32)                      # correctly rounded m/127
    r = (xg / s.astype(np.float64)[..., None]).astype(np.float32).astype(np.float64)
    q = np.clip(_round_half_away(r) + 128, 0, 255).astype(np.uint8)
    return q.reshape(x.shape), s.reshape(x.shape[:-1] + (D // group,))


def test_ties_round_half_away_from_zero():
    kv, rows = read_golden("ties.txt")
    xs = [float(r[0]) for r in rows]
    expect = [int(r[1]) for r in rows]
    x = _row_with(xs, D=32)
    q, s = oracle.quantize(x)
    assert s.item() == 0.5
    assert q[0, 0].item() == 255
    got = q[0, 1:1 + len(xs)].tolist()
    assert got == expect


def test_grid_roundtrip_exact_per_group_and_per_token():
    kv, _ = read_golden("grid_roundtrip.txt")
    shape = [int(v) for v in kv["shape"].split(",")]
    n_el = int(np.prod(shape))
    i = np.arange(n_el)
    n = (i * int(kv["multiplier"])) % int(kv["modulus"]) - int(kv["offset"])
    x = n.astype(np.float32) * float(kv["step"])
    forced = float(kv["forced"])
    x_g = x.copy()
    x_g[::32] = forced
    n_g = n.copy()
    n_g[::32] = int(forced / float(kv["step"]))
    xt = torch.from_numpy(x_g).reshape(shape).to(torch.bfloat16)
    assert torch.equal(xt.float().reshape(-1), torch.from_numpy(x_g))   # exact in bf16
    for mode in ("group32", "per_token"):
        q, s = oracle.quantize(xt, mode)
        assert torch.all(s == float(kv["expected_scale"])), mode
        assert torch.equal(q.reshape(-1).to(torch.int64),
                           torch.from_numpy(n_g + int(kv["expected_byte_offset"])))
        back = oracle.dequant(q, s, mode)
        assert torch.equal(back.reshape(-1), torch.from_numpy(x_g)), mode


def test_roundtrip_bound_worked_example():
    kv, _ = read_golden("roundtrip_bound.txt")
    n = int(kv["n"])
    x = (np.arange(n, dtype=np.float32) - float(kv["center"])) / float(kv["denom"])
    shape = [int(v) for v in kv["shape"].split(",")]
    xt = torch.from_numpy(x).reshape(shape).to(torch.bfloat16)
    q, s = oracle.quantize(xt)
    back = oracle.dequant(q, s)
    assert (back - xt.float()).abs().max().item() < float(kv["bound"])


def test_half_step_bound_worked_example():
    kv, _ = read_golden("half_step.txt")
    shape = [int(v) for v in kv["shape"].split(",")]
    i = np.arange(int(np.prod(shape)))
    x = ((i * int(kv["multiplier"])) % int(kv["modulus"])).astype(np.float32) \
        / float(kv["denom"]) - float(kv["shift"])
    xt = torch.from_numpy(x).reshape(shape).to(torch.bfloat16)
    q, s = oracle.quantize(xt, "group32")
    back = oracle.dequant(q, s, "group32").reshape(-1, 32)
    xf = xt.float().reshape(-1, 32)
    absmax = xf.abs().max(dim=1, keepdim=True).values
    assert torch.all((xf - back).abs() <= absmax / 254.0 + float(kv["slack"]))


@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("sigma", [1.0, 1e-3, 37.0])
def test_matches_fp64_route_bit_exact(mode, sigma):
    g = torch.Generator().manual_seed(7)
    x = (torch.randn(64, 128, generator=g) * sigma).to(torch.bfloat16)
    x[3] = 0                                    # all-zero row: eps floor
    x[5, 17] = 40.0                             # outlier
    x[9] = x[9] * 1e-6                          # tiny row near the eps floor
    q, s = oracle.quantize(x, mode)
    q2, s2 = _f64_route(x, oracle.group_of(mode, 128))
    assert np.array_equal(s.numpy().view(np.uint32), s2.view(np.uint32))
    assert np.array_equal(q.numpy(), q2)


def test_dequant_matches_fp64_route():
    g = torch.Generator().manual_seed(11)
    q = torch.randint(0, 256, (50, 64), generator=g, dtype=torch.uint8)
    s = (torch.rand(50, 2, generator=g) * 3 + 1e-6).float()
    out = oracle.dequant(q, s, "group32")
    ref = ((q.numpy().astype(np.float64) - 128.0)
           * np.repeat(s.numpy().astype(np.float64), 32, axis=1)).astype(np.float32)
    assert np.array_equal(out.numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_invariants(mode):
    g = torch.Generator().manual_seed(3)
    x = torch.randn(200, 64, generator=g).to(torch.bfloat16)
    q, s = oracle.quantize(x, mode)
    grp = oracle.group_of(mode, 64)
    # bytes in [1, 255]
    assert int(q.min()) >= 1 and int(q.max()) <= 255
    # the absmax element of each group maps to an end of the range
    xg = x.float().reshape(200, -1, grp)
    qg = q.reshape(200, -1, grp).to(torch.int64)
    idx = xg.abs().argmax(dim=-1, keepdim=True)
    ends = qg.gather(-1, idx)
    assert torch.all((ends == 1) | (ends == 255))
    # odd symmetry: u8(-x) = 256 - u8(x), same scale
    qn, sn = oracle.quantize(-x, mode)
    assert torch.equal(sn, s)
    assert torch.equal(qn.to(torch.int64), 256 - q.to(torch.int64))
    # power-of-two scale invariance
    for k in (-3, 5):
        q2, s2 = oracle.quantize((x.float() * 2.0 ** k).to(torch.bfloat16), mode)
        assert torch.equal(q2, q)
        assert torch.equal(s2, s * 2.0 ** k)
    # half-step bound on every element: |x/s - q| <= 1/2 + the rounding of the
    # fp32 quotient (half an ulp of a value below 128, i.e. <= 2^-18), and the
    # product (q-128)*s adds one more fp32 rounding
    back = oracle.dequant(q, s, mode).reshape(200, -1, grp)
    bound = s.reshape(200, -1, 1) * (0.5 + 2.0 ** -18 + 128 * 2.0 ** -24)
    assert torch.all((back - xg).abs() <= bound)


def test_zero_vector_and_eps_floor():
    x = torch.zeros(2, 32, dtype=torch.bfloat16)
    x[1, 4] = 1e-9          # below the 1e-8 floor
    q, s = oracle.quantize(x)
    eps_scale = np.float32(1e-8) / np.float32(127.0)
    assert s[0].item() == float(eps_scale)
    assert s[1].item() == float(eps_scale)
    assert torch.all(q[0] == 128)
    # 1e-9 / (1e-8/127) = 12.7 -> 13
    assert q[1, 4].item() == 128 + 13


def test_group32_groups_are_independent():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(4, 128, generator=g).to(torch.bfloat16)
    q, s = oracle.quantize(x, "group32")
    y = x.clone()
    y[:, :32] *= 8
    q2, s2 = oracle.quantize(y, "group32")
    assert torch.equal(q2[:, 32:], q[:, 32:]) and torch.equal(s2[:, 1:], s[:, 1:])
    # a group's scale equals the per-token scale of that 32-slice alone
    for j in range(4):
        qj, sj = oracle.quantize(x[:, 32 * j:32 * j + 32].contiguous(), "per_token")
        assert torch.equal(sj[:, 0], s[:, j])
        assert torch.equal(qj, q[:, 32 * j:32 * j + 32])


def test_append_contig_places_rows_and_flags_overflow():
    g = torch.Generator().manual_seed(9)
    B, Hk, T, D, S = 3, 2, 5, 64, 12
    x = torch.randn(B, Hk, T, D, generator=g).to(torch.bfloat16)
    cache = torch.full((B, Hk, S, D), 7, dtype=torch.uint8)
    sc = torch.full((B, Hk, S, 2), -1.0)
    pos = torch.tensor([0, 7, 9], dtype=torch.int32)        # row 2 overflows (9+5>12)
    err = oracle.append_contig(x, pos, cache, sc, "group32")
    assert err == oracle.ORACLE_ERR_POS
    qx, sx = oracle.quantize(x, "group32")
    for b in range(2):
        p = int(pos[b])
        assert torch.equal(cache[b, :, p:p + T], qx[b])
        assert torch.equal(sc[b, :, p:p + T], sx[b])
        keep = torch.ones(S, dtype=torch.bool)
        keep[p:p + T] = False
        assert torch.all(cache[b, :, keep] == 7) and torch.all(sc[b, :, keep] == -1.0)
    assert torch.all(cache[2] == 7)


def test_append_paged_slot_arithmetic():
    g = torch.Generator().manual_seed(13)
    B, Hk, T, D, ps = 2, 3, 21, 32, 16
    x = torch.randn(B, Hk, T, D, generator=g).to(torch.bfloat16)
    pos = torch.tensor([5, 30], dtype=torch.int32)
    max_pages, num_pages = 4, 9
    table = torch.tensor([[8, 2, 6, -1], [0, 3, 7, 5]], dtype=torch.int32)
    arena = torch.zeros(num_pages, Hk, ps, D, dtype=torch.uint8)
    sc = torch.zeros(num_pages, Hk, ps, 1)
    err = oracle.append_paged(x, pos, arena, sc, table, ps)
    assert err == 0
    qx, sx = oracle.quantize(x)
    for b in range(B):
        for t in range(T):
            gpos = int(pos[b]) + t
            page = int(table[b, gpos // ps])     # hand lookup
            slot = gpos % ps
            assert torch.equal(arena[page, :, slot], qx[b, :, t])
            assert torch.equal(sc[page, :, slot], sx[b, :, t])
    # a -1 entry in the used range is skipped and flagged
    arena2 = torch.zeros_like(arena)
    err = oracle.append_paged(x[:1, :, :1], torch.tensor([50], dtype=torch.int32),
                              arena2, torch.zeros_like(sc), table[:1], ps)
    assert err == oracle.ORACLE_ERR_PAGE and int(arena2.sum()) == 0

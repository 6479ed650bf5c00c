"""GPU parity of the per-head / per-channel modes (KVQ_SCALE_PER_HEAD,
KVQ_SCALE_PER_CHANNEL): calibration (scales from one call's tokens) and
appends with stored scales bit-exact with the oracle, contiguous and paged;
dequant bit-exact with the pinned per-token dequant; decode, chunk and
window attention within the fp64 bar of the oracle."""
import pytest
import torch

import oracle
from kvq_testutil import assert_attn_close, bf16_randn, f32_scale, kvq

pytestmark = pytest.mark.gpu
GRANS = ["per_head", "per_channel"]


def _ns(gran, D):
    return 1 if gran == "per_head" else D


class StaticCache:
    """Contiguous per-head / per-channel INT8 cache, GPU and oracle twins."""

    def __init__(self, B, Hk, S, D, gran):
        self.gran = gran
        ns = _ns(gran, D)
        self.k = torch.full((B, Hk, S, D), 0xCD, dtype=torch.uint8, device="cuda")
        self.v = torch.full_like(self.k, 0xCD)
        self.ks = torch.full((B, Hk, ns), -7.0, device="cuda")
        self.vs = torch.full_like(self.ks, -7.0)
        self.ok = torch.full((B, Hk, S, D), 0xCD, dtype=torch.uint8)
        self.ov = torch.full_like(self.ok, 0xCD)
        self.oks = torch.full((B, Hk, ns), -7.0)
        self.ovs = torch.full_like(self.oks, -7.0)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def append(self, kn, vn, pos, calibrate):
        m = kvq()
        call = m.kvq_append_calibrate if calibrate else m.kvq_append
        call(kn.cuda(), vn.cuda(), pos.cuda(), self.k, self.v, self.ks, self.vs, self.gran,
             err=self.err)
        e = oracle.append_static(kn, pos, self.ok, self.oks, self.gran, calibrate)
        return e | oracle.append_static(vn, pos, self.ov, self.ovs, self.gran, calibrate)

    def assert_bit_exact(self):
        torch.cuda.synchronize()
        assert torch.equal(self.k.cpu(), self.ok) and torch.equal(self.v.cpu(), self.ov)
        assert torch.equal(self.ks.cpu().view(torch.int32), self.oks.view(torch.int32))
        assert torch.equal(self.vs.cpu().view(torch.int32), self.ovs.view(torch.int32))


@pytest.mark.parametrize("gran", GRANS)
@pytest.mark.parametrize("D,T", [(64, 1), (128, 7), (128, 300), (256, 33), (96, 5), (16, 40)])
def test_calibrate_then_append_bit_exact(gran, D, T):
    B, Hk, S = 3, 2, 2 * T + 5
    c = StaticCache(B, Hk, S, D, gran)
    z = torch.zeros(B, dtype=torch.int32)
    assert c.append(bf16_randn((B, Hk, T, D), D + T), bf16_randn((B, Hk, T, D), D + T + 1), z,
                    True) == 0
    c.assert_bit_exact()
    # later tokens with the stored scales, partly beyond the calibrated range
    pos = torch.full((B,), T, dtype=torch.int32)
    assert c.append(bf16_randn((B, Hk, T, D), 5, 1.7), bf16_randn((B, Hk, T, D), 6, 1.7), pos,
                    False) == 0
    c.assert_bit_exact()
    # a range past the capacity is skipped and flagged, the scales untouched
    bad = torch.tensor([S, 0, 0], dtype=torch.int32)
    assert c.append(bf16_randn((B, Hk, T, D), 7), bf16_randn((B, Hk, T, D), 8), bad, True) == \
        oracle.ORACLE_ERR_POS
    assert kvq().kvq_read_error(c.err) == 1
    c.assert_bit_exact()


@pytest.mark.parametrize("gran", GRANS)
def test_static_paged_append_and_dequant(gran):
    m = kvq()
    B, Hk, D, T = 2, 2, 128, 20
    c = StaticCache(B, Hk, T, D, gran)
    z = torch.zeros(B, dtype=torch.int32)
    c.append(bf16_randn((B, Hk, T, D), 1), bf16_randn((B, Hk, T, D), 2), z, True)
    table = torch.tensor([[3, 0], [1, 2]], dtype=torch.int32)
    ak = torch.zeros(4, Hk, 16, D, dtype=torch.uint8, device="cuda")
    av = torch.zeros_like(ak)
    kn, vn = bf16_randn((B, Hk, T, D), 3), bf16_randn((B, Hk, T, D), 4)
    m.kvq_append_paged(kn.cuda(), vn.cuda(), z.cuda(), ak, av, c.ks, c.vs, table.cuda(), 16,
                       gran)
    ref = torch.zeros(B, Hk, T, D, dtype=torch.uint8)
    oracle.append_static(kn, z, ref, c.oks.clone(), gran, calibrate=False)
    torch.cuda.synchronize()
    for b in range(B):
        for t in range(T):
            assert torch.equal(ak[int(table[b, t // 16]), :, t % 16].cpu(), ref[b, :, t])
    # dequant of one (sequence, kv head): its scales apply to every row; the
    # pinned per-token dequant of the transposed rows (per channel) or of the
    # rows with the head's scale repeated (per head)
    rows = c.k[0, 1].clone()                   # fresh, 16-byte aligned allocations
    sc = c.ks[0, 1].clone()
    got = m.kvq_dequant(rows, sc, gran).cpu()
    if gran == "per_channel":
        want = oracle.dequant(rows.cpu().t().contiguous(), sc.cpu().view(D, 1)).t()
    else:
        want = oracle.dequant(rows.cpu(), sc.cpu().expand(rows.shape[0], 1).contiguous())
    assert torch.equal(got, want)


def _filled(B, Hk, D, gran, lens, seed):
    S = max(lens)
    c = StaticCache(B, Hk, S, D, gran)
    c.append(bf16_randn((B, Hk, S, D), seed), bf16_randn((B, Hk, S, D), seed + 1),
             torch.zeros(B, dtype=torch.int32), True)
    return c


def _attn(c, q, sl, hint, window=0, **kw):
    m = kvq()
    D = q.shape[-1]
    if window:
        return m.kvq_window_attn(q.cuda(), c.k, c.v, c.ks, c.vs, sl.cuda(), hint, window,
                                 mode=c.gran, attn_scale=f32_scale(D), err=c.err, **kw)
    call = m.kvq_decode_attn if q.dim() == 3 else m.kvq_chunk_attn
    return call(q.cuda(), c.k, c.v, c.ks, c.vs, sl.cuda(), hint, mode=c.gran,
                attn_scale=f32_scale(D), err=c.err, **kw)


@pytest.mark.parametrize("gran", GRANS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_static_decode_matches_oracle(gran, D, G):
    B, Hk = 3, 2
    lens = [1, 200, 2100]
    c = _filled(B, Hk, D, gran, lens, seed=G * 3 + D)
    q = bf16_randn((B, Hk * G, D), seed=G)
    sl = torch.tensor(lens, dtype=torch.int32)
    ref = oracle.static_attn(q, c.ok, c.ov, c.oks, c.ovs, sl, gran, 0, f32_scale(D))
    for ns in (0, 1, 4):
        assert_attn_close(_attn(c, q, sl, max(lens), num_splits=ns), ref,
                          f"{gran} D={D} G={G} ns={ns}")


@pytest.mark.parametrize("gran", GRANS)
def test_static_many_units_chunk_window(gran):
    B, Hk, D = 20, 4, 128
    lens = [4, 17, 300, 1000, 2500] * 4
    c = _filled(B, Hk, D, gran, lens, seed=9)
    sl = torch.tensor(lens, dtype=torch.int32)
    q1 = bf16_randn((B, Hk * 4, D), seed=10)
    assert_attn_close(_attn(c, q1, sl, max(lens)),
                      oracle.static_attn(q1, c.ok, c.ov, c.oks, c.ovs, sl, gran, 0, f32_scale(D)),
                      "many units")
    q4 = bf16_randn((B, Hk * 2, 4, D), seed=11)
    assert_attn_close(_attn(c, q4, sl, max(lens)),
                      oracle.static_attn(q4, c.ok, c.ov, c.oks, c.ovs, sl, gran, 0, f32_scale(D)),
                      "chunk")
    assert_attn_close(_attn(c, q1, sl, max(lens), window=100),
                      oracle.static_attn(q1, c.ok, c.ov, c.oks, c.ovs, sl, gran, 100,
                                         f32_scale(D)), "window")

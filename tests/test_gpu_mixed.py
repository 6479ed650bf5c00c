"""GPU parity of the mixed cache (newest tokens bf16 in a ring, older ones
INT8): kvq_append_mixed bit-exact with the oracle's append (INT8 part bytes
and scales, the ring) over prefills and decode steps with ragged lengths,
and kvq_decode_attn_mixed within the fp64 bar of the oracle's mixed
attention, for the per-token, group-32, per-head and per-channel modes."""
import pytest
import torch

import oracle
from kvq_testutil import assert_attn_close, bf16_randn, f32_scale, kvq

pytestmark = pytest.mark.gpu
MODES = ["per_token", "group32", "per_head", "per_channel"]


class MixedPair:
    def __init__(self, B, Hk, S, D, W, mode, seed):
        m = kvq()
        self.B, self.Hk, self.S, self.D, self.W, self.mode = B, Hk, S, D, W, mode
        if mode in ("per_token", "group32"):
            ng = 1 if mode == "per_token" else D // 32
            sshape = (B, Hk, S, ng)
        else:
            sshape = (B, Hk, 1 if mode == "per_head" else D)
        self.k = torch.zeros(B, Hk, S, D, dtype=torch.uint8, device="cuda")
        self.v = torch.zeros_like(self.k)
        self.ks = torch.zeros(sshape, device="cuda")
        self.vs = torch.zeros_like(self.ks)
        self.rk = torch.zeros(B, Hk, W, D, dtype=torch.bfloat16, device="cuda")
        self.rv = torch.zeros_like(self.rk)
        self.ok, self.ov = self.k.cpu(), self.v.cpu()
        self.oks, self.ovs = self.ks.cpu(), self.vs.cpu()
        self.ork, self.orv = self.rk.cpu(), self.rv.cpu()
        self.lens = torch.zeros(B, dtype=torch.int32)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if mode in ("per_head", "per_channel"):            # calibrate the scales
            T = 24
            kc, vc = bf16_randn((B, Hk, T, D), seed), bf16_randn((B, Hk, T, D), seed + 1)
            tk = torch.zeros(B, Hk, T, D, dtype=torch.uint8, device="cuda")
            z = torch.zeros(B, dtype=torch.int32)
            m.kvq_append_calibrate(kc.cuda(), vc.cuda(), z.cuda(), tk, tk.clone(), self.ks,
                                   self.vs, mode)
            tko = tk.cpu()
            oracle.append_static(kc, z, tko, self.oks, mode)
            oracle.append_static(vc, z, tko.clone(), self.ovs, mode)

    def append(self, n_new, seed):
        """n_new[b] tokens for sequence b (one call per distinct count)."""
        m = kvq()
        for n in sorted(set(n_new)):
            if n == 0:
                continue
            rows = [b for b in range(self.B) if n_new[b] == n]
            # one call over all sequences that append n tokens: others get T = n
            # too in this batched layout, so call per sequence for ragged counts
            for b in rows:
                kn = bf16_randn((1, self.Hk, n, self.D), seed + 31 * b + n)
                vn = bf16_randn((1, self.Hk, n, self.D), seed + 77 * b + n)
                sl = slice(b, b + 1)
                lo = self.lens[sl].clone()
                sk = self.ks[sl] if self.mode in ("per_token", "group32") else self.ks[sl]
                m.kvq_append_mixed(kn.cuda(), vn.cuda(), lo.cuda(), self.k[sl], self.v[sl],
                                   sk, self.vs[sl], self.rk[sl], self.rv[sl], self.mode,
                                   err=self.err)
                okb, ovb = self.ok[sl], self.ov[sl]
                oksb, ovsb = self.oks[sl], self.ovs[sl]
                orkb, orvb = self.ork[sl], self.orv[sl]
                assert oracle.append_mixed(kn, lo, okb, oksb, orkb, self.mode) == 0
                assert oracle.append_mixed(vn, lo, ovb, ovsb, orvb, self.mode) == 0
                self.ok[sl], self.ov[sl], self.oks[sl], self.ovs[sl] = okb, ovb, oksb, ovsb
                self.ork[sl], self.orv[sl] = orkb, orvb
                self.lens[b] += n

    def assert_bit_exact(self):
        torch.cuda.synchronize()
        assert torch.equal(self.k.cpu(), self.ok) and torch.equal(self.v.cpu(), self.ov)
        assert torch.equal(self.ks.cpu().view(torch.int32), self.oks.view(torch.int32))
        assert torch.equal(self.vs.cpu().view(torch.int32), self.ovs.view(torch.int32))
        assert torch.equal(self.rk.cpu().view(torch.int16), self.ork.view(torch.int16))
        assert torch.equal(self.rv.cpu().view(torch.int16), self.orv.view(torch.int16))

    def check_decode(self, Hq, seed, **kw):
        m = kvq()
        q = bf16_randn((self.B, Hq, self.D), seed)
        hint = max(int(self.lens.max()), 1)
        out = m.kvq_decode_attn_mixed(q.cuda(), self.k, self.v, self.ks, self.vs, self.rk,
                                      self.rv, self.lens.cuda(), hint, mode=self.mode,
                                      attn_scale=f32_scale(self.D), err=self.err, **kw)
        ref = oracle.mixed_attn(q, self.ok, self.ov, self.oks, self.ovs, self.ork, self.orv,
                                self.lens, self.mode, f32_scale(self.D))
        assert_attn_close(out, ref, f"{self.mode} lens={self.lens.tolist()} {kw}")
        assert kvq().kvq_read_error(self.err) == 0


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("W", [8, 128])
def test_mixed_append_and_decode(mode, W):
    B, Hk, G, D, S = 3, 2, 4, 128, 1200
    c = MixedPair(B, Hk, S, D, W, mode, seed=W)
    c.append([300, 5, 140], seed=1)                 # prefills: longer, shorter than W
    c.assert_bit_exact()
    c.check_decode(Hk * G, seed=2)
    for step in range(3):                           # decode steps
        c.append([1, 1, 1], seed=10 + step)
        c.assert_bit_exact()
        c.check_decode(Hk * G, seed=20 + step, num_splits=0 if step else 3)
    c.append([700, 0, 9], seed=40)                  # a long chunk through the window
    c.assert_bit_exact()
    c.check_decode(Hk * G, seed=41)


@pytest.mark.parametrize("mode", ["per_token", "per_channel"])
def test_mixed_many_units(mode):
    """Many sequences (blocks of items per CTA), some still inside the window."""
    B, Hk, D, S, W = 24, 4, 128, 900, 64
    c = MixedPair(B, Hk, S, D, W, mode, seed=5)
    c.append([(37 * b) % 800 for b in range(B)], seed=6)
    c.assert_bit_exact()
    c.check_decode(Hk * 8, seed=7)
    c.check_decode(Hk * 2, seed=8, num_splits=5)


@pytest.mark.parametrize("D,G,W", [(128, 32, 2048), (96, 4, 200), (256, 8, 40)])
def test_mixed_wide_groups_long_windows_other_head_dims(D, G, W):
    """The window kernel takes a cluster of four CTAs per (sequence, q head):
    32 heads per kv head, the longest window (2048 tokens, 512 per CTA in
    several tiles), and head dims whose INT8 part runs on the CUDA-core split
    kernel."""
    B, Hk, S = 2, 2, 3000
    c = MixedPair(B, Hk, S, D, W, "per_token", seed=D + G)
    c.append([2500, 100], seed=3)
    c.assert_bit_exact()
    c.check_decode(Hk * G, seed=4)
    c.append([1, 1], seed=5)
    c.assert_bit_exact()
    c.check_decode(Hk * G, seed=6, num_splits=3)

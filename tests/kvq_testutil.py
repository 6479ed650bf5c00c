"""Helpers shared by the GPU parity tests: build the same INT8 cache twice,
once through the CUDA library and once through the CPU oracle, from the same
seeded bf16 inputs, and compare."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

ATOL = 2e-3       # max-abs bar against the fp64 oracle
RTOL_L2 = 1e-3    # relative-L2 bar against the fp64 oracle


def kvq():
    import decode_attention_kvq_b200 as m
    return m


def ng(mode, D):
    return 1 if mode == "per_token" else D // 32


def assert_attn_close(got: torch.Tensor, ref: torch.Tensor, what: str = ""):
    got = got.detach().cpu().double()
    ref = ref.double()
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    diff = (got - ref)
    max_abs = diff.abs().max().item() if diff.numel() else 0.0
    den = ref.norm().item()
    rel = diff.norm().item() / den if den > 0 else diff.norm().item()
    assert max_abs <= ATOL, f"{what}: max-abs {max_abs:.3e} > {ATOL}"
    assert rel <= RTOL_L2, f"{what}: rel-L2 {rel:.3e} > {RTOL_L2}"
    return max_abs, rel


class ContigCache:
    """Contiguous INT8 cache on the GPU plus its oracle twin on the CPU."""

    def __init__(self, B, Hk, S, D, mode, dev="cuda"):
        self.B, self.Hk, self.S, self.D, self.mode = B, Hk, S, D, mode
        n = ng(mode, D)
        self.k = torch.full((B, Hk, S, D), 0xCD, dtype=torch.uint8, device=dev)
        self.v = torch.full_like(self.k, 0xCD)
        self.ks = torch.full((B, Hk, S, n), -7.0, dtype=torch.float32, device=dev)
        self.vs = torch.full_like(self.ks, -7.0)
        self.ok = torch.full((B, Hk, S, D), 0xCD, dtype=torch.uint8)
        self.ov = torch.full_like(self.ok, 0xCD)
        self.oks = torch.full((B, Hk, S, n), -7.0, dtype=torch.float32)
        self.ovs = torch.full_like(self.oks, -7.0)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def append(self, k_new, v_new, pos):
        m = kvq()
        dev = self.k.device
        m.kvq_append(k_new.to(dev), v_new.to(dev), pos.to(dev), self.k, self.v, self.ks, self.vs,
                     self.mode, err=self.err)
        e1 = oracle.append_contig(k_new, pos, self.ok, self.oks, self.mode)
        e2 = oracle.append_contig(v_new, pos, self.ov, self.ovs, self.mode)
        return e1 | e2

    def assert_bit_exact(self):
        torch.cuda.synchronize()
        assert torch.equal(self.k.cpu(), self.ok), "K bytes differ"
        assert torch.equal(self.v.cpu(), self.ov), "V bytes differ"
        assert torch.equal(self.ks.cpu().view(torch.int32), self.oks.view(torch.int32)), "K scales"
        assert torch.equal(self.vs.cpu().view(torch.int32), self.ovs.view(torch.int32)), "V scales"

    def decode(self, q, seq_lens, hint, **kw):
        m = kvq()
        dev = self.k.device
        return m.kvq_decode_attn(q.to(dev), self.k, self.v, self.ks, self.vs, seq_lens.to(dev),
                                 hint, mode=self.mode, err=self.err, **kw)

    def oracle_decode(self, q, seq_lens, attn_scale):
        return oracle.decode_attn(q, self.ok, self.ov, self.oks, self.ovs, seq_lens,
                                  attn_scale, self.mode)

    def chunk(self, q, seq_lens, hint, **kw):
        m = kvq()
        dev = self.k.device
        return m.kvq_chunk_attn(q.to(dev), self.k, self.v, self.ks, self.vs, seq_lens.to(dev),
                                hint, mode=self.mode, err=self.err, **kw)

    def oracle_chunk(self, q, seq_lens, attn_scale):
        return oracle.chunk_attn(q, self.ok, self.ov, self.oks, self.ovs, seq_lens, attn_scale,
                                 self.mode)


class PagedCache:
    """Paged INT8 arena on the GPU plus its oracle twin."""

    def __init__(self, num_pages, Hk, D, mode, table, dev="cuda", page_size=16):
        self.Hk, self.D, self.mode, self.ps = Hk, D, mode, page_size
        n = ng(mode, D)
        shape = (num_pages, Hk, page_size, D)
        self.k = torch.full(shape, 0xCD, dtype=torch.uint8, device=dev)
        self.v = torch.full_like(self.k, 0xCD)
        self.ks = torch.full((num_pages, Hk, page_size, n), -7.0, device=dev)
        self.vs = torch.full_like(self.ks, -7.0)
        self.ok = torch.full(shape, 0xCD, dtype=torch.uint8)
        self.ov = torch.full_like(self.ok, 0xCD)
        self.oks = torch.full((num_pages, Hk, page_size, n), -7.0)
        self.ovs = torch.full_like(self.oks, -7.0)
        self.table_cpu = table.to(torch.int32).contiguous()
        self.table = self.table_cpu.to(dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)

    def append(self, k_new, v_new, pos, rows=None):
        """Append for all sequences, or for the batch rows listed in `rows`."""
        m = kvq()
        dev = self.k.device
        table = self.table_cpu if rows is None else self.table_cpu[rows].contiguous()
        m.kvq_append_paged(k_new.to(dev), v_new.to(dev), pos.to(dev), self.k, self.v, self.ks,
                           self.vs, table.to(dev), self.ps, self.mode, err=self.err)
        e1 = oracle.append_paged(k_new, pos, self.ok, self.oks, table, self.ps, self.mode)
        e2 = oracle.append_paged(v_new, pos, self.ov, self.ovs, table, self.ps, self.mode)
        return e1 | e2

    def assert_bit_exact(self):
        torch.cuda.synchronize()
        assert torch.equal(self.k.cpu(), self.ok), "K bytes differ"
        assert torch.equal(self.v.cpu(), self.ov), "V bytes differ"
        assert torch.equal(self.ks.cpu().view(torch.int32), self.oks.view(torch.int32)), "K scales"
        assert torch.equal(self.vs.cpu().view(torch.int32), self.ovs.view(torch.int32)), "V scales"

    def decode(self, q, seq_lens, hint, **kw):
        m = kvq()
        dev = self.k.device
        return m.kvq_decode_attn(q.to(dev), self.k, self.v, self.ks, self.vs, seq_lens.to(dev),
                                 hint, page_table=self.table, page_size=self.ps, mode=self.mode,
                                 err=self.err, **kw)

    def oracle_decode(self, q, seq_lens, attn_scale):
        return oracle.decode_attn(q, self.ok, self.ov, self.oks, self.ovs, seq_lens, attn_scale,
                                  self.mode, page_size=self.ps, table=self.table_cpu)

    def chunk(self, q, seq_lens, hint, **kw):
        m = kvq()
        dev = self.k.device
        return m.kvq_chunk_attn(q.to(dev), self.k, self.v, self.ks, self.vs, seq_lens.to(dev),
                                hint, page_table=self.table, page_size=self.ps, mode=self.mode,
                                err=self.err, **kw)

    def oracle_chunk(self, q, seq_lens, attn_scale):
        return oracle.chunk_attn(q, self.ok, self.ov, self.oks, self.ovs, seq_lens, attn_scale,
                                 self.mode, page_size=self.ps, table=self.table_cpu)


def f32_scale(D):
    """attn_scale as the fp32 value both sides use."""
    return float(np.float32(1.0 / math.sqrt(D)))


def bf16_randn(shape, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * sigma).to(torch.bfloat16)

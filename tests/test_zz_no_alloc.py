"""GPU test of kvq_decode_attn_noalloc, the decode entry point for callers
that cannot allocate device memory (it uses the library's own fixed split-K
scratch array instead of a caller workspace).

Collected last on purpose (file name), so that a run stopping at the first
failure has run every other test first.  It must pass alone in a fresh
process and after the other tests."""
import ctypes

import pytest
import torch

import synth
from kvq_testutil import (ContigCache, PagedCache, assert_attn_close, bf16_randn, f32_scale,
                          kvq)

pytestmark = pytest.mark.gpu


def _cache(B, Hk, L, D, seed):
    k = torch.randint(0, 256, (B, Hk, L, D), dtype=torch.uint8,
                      generator=torch.Generator().manual_seed(seed)).cuda()
    v = torch.randint(0, 256, (B, Hk, L, D), dtype=torch.uint8,
                      generator=torch.Generator().manual_seed(seed + 1)).cuda()
    g = torch.Generator().manual_seed(seed + 2)
    ks = (torch.rand(B, Hk, L, 1, generator=g) * 0.05 + 0.005).cuda()
    vs = (torch.rand(B, Hk, L, 1, generator=g) * 0.05 + 0.005).cuda()
    return k, v, ks, vs


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    m = kvq()
    B, Hq, Hk, D, L = 2, 32, 8, 128, 3000
    k, v, ks, vs = _cache(B, Hk, L, D, seed=3)
    seq = torch.tensor([3000, 1777], dtype=torch.int32).cuda()
    need = m.kvq_decode_workspace_bytes(B, Hq, Hk, D, L)
    assert 0 < need <= m.lib.kvq_noalloc_scratch_bytes()   # the scratch array is exercised
    for call in range(2):                                    # two calls in a row share the array
        q = bf16_randn((B, Hq, D), seed=40 + call).cuda()
        ref = m.kvq_decode_attn(q, k, v, ks, vs, seq, L)
        out = torch.full((B, Hq, D), float("nan"), device="cuda")
        cv = m.cache_view(k, v, ks, vs)
        st = m.lib.kvq_decode_attn_noalloc(
            q.data_ptr(), B, Hq, Hk, D, 0, ctypes.byref(cv), seq.data_ptr(), L,
            float(1.0 / D ** 0.5), out.data_ptr(), 0, None,
            torch.cuda.current_stream().cuda_stream)
        assert st == 0, m.lib.kvq_status_string(st)
        torch.cuda.synchronize()
        assert_attn_close(out, ref.cpu().double(), f"call {call}")


def test_noalloc_rejects_problems_larger_than_the_scratch():
    m = kvq()
    B, Hq, Hk, D, L = 64, 64, 8, 128, 64
    k, v, ks, vs = _cache(1, Hk, L, D, seed=9)
    q = bf16_randn((B, Hq, D), seed=1).cuda()
    seq = torch.full((B,), 16, dtype=torch.int32).cuda()
    out = torch.zeros(B, Hq, D, device="cuda")
    cv = m.cache_view(k, v, ks, vs)
    # 4096 requested splits of a long hint need far more than the fixed scratch
    assert m.kvq_decode_workspace_bytes(B, Hq, Hk, D, 1 << 20, 4096) > \
        m.lib.kvq_noalloc_scratch_bytes()
    st = m.lib.kvq_decode_attn_noalloc(q.data_ptr(), B, Hq, Hk, D, 0, ctypes.byref(cv),
                                       seq.data_ptr(), 1 << 20, 0.088, out.data_ptr(), 4096,
                                       None, torch.cuda.current_stream().cuda_stream)
    assert st == 5 and m.lib.kvq_status_string(st).decode() == "KVQ_ERR_SCRATCH_TOO_SMALL"
    torch.cuda.synchronize()
    assert torch.all(out == 0)                               # nothing was enqueued


def _noalloc(m, q, cache, seq, hint, mode, paged):
    """One kvq_decode_attn_noalloc call through the C ABI."""
    B, Hq, D = q.shape
    Hk = cache.k.shape[1]
    out = torch.full((B, Hq, D), float("nan"), device="cuda")
    cv = (m.cache_view(cache.k, cache.v, cache.ks, cache.vs, cache.table, 16) if paged else
          m.cache_view(cache.k, cache.v, cache.ks, cache.vs))
    st = m.lib.kvq_decode_attn_noalloc(
        q.data_ptr(), B, Hq, Hk, D, 0 if mode == "per_token" else 1, ctypes.byref(cv),
        seq.data_ptr(), hint, f32_scale(D), out.data_ptr(), 0, None,
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, m.lib.kvq_status_string(st)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_noalloc_matches_oracle_contiguous(mode):
    """The scratch-array path against the fp64 oracle and against the
    workspace entry point, two calls in a row, per-token and group-32."""
    m = kvq()
    B, Hq, Hk, D = 3, 32, 8, 128
    lens = [2900, 1500, 777]
    S = max(lens)
    c = ContigCache(B, Hk, S, D, mode)
    g = torch.Generator().manual_seed(71)
    kh = (torch.randn(B, Hk, S, D, generator=g)).to(torch.bfloat16)
    vh = (torch.randn(B, Hk, S, D, generator=g)).to(torch.bfloat16)
    assert c.append(kh, vh, torch.zeros(B, dtype=torch.int32)) == 0
    seq = torch.tensor(lens, dtype=torch.int32)
    assert m.kvq_decode_workspace_bytes(B, Hq, Hk, D, S) > 0
    for call in range(2):
        q = bf16_randn((B, Hq, D), seed=80 + call)
        out = _noalloc(m, q.cuda(), c, seq.cuda(), S, mode, paged=False)
        ref = c.oracle_decode(q, seq, f32_scale(D))
        assert_attn_close(out, ref, f"{mode} call {call} vs oracle")
        ws = c.decode(q, seq, S, attn_scale=f32_scale(D))
        assert_attn_close(out, ws.cpu().double(), f"{mode} call {call} vs workspace call")


def test_noalloc_matches_oracle_paged():
    """Paged arena through the scratch array, against the oracle."""
    m = kvq()
    B, Hq, Hk, D = 4, 32, 8, 128
    lens = [1200, 3001, 16, 640]
    table, npages = synth.page_table_for(lens, 16, torch.Generator().manual_seed(5))
    c = PagedCache(npages, Hk, D, "per_token", table)
    g = torch.Generator().manual_seed(72)
    for b, L in enumerate(lens):
        kh = torch.randn(1, Hk, L, D, generator=g).to(torch.bfloat16)
        vh = torch.randn(1, Hk, L, D, generator=g).to(torch.bfloat16)
        assert c.append(kh, vh, torch.zeros(1, dtype=torch.int32), rows=[b]) == 0
    seq = torch.tensor(lens, dtype=torch.int32)
    for call in range(2):
        q = bf16_randn((B, Hq, D), seed=90 + call)
        out = _noalloc(m, q.cuda(), c, seq.cuda(), max(lens), "per_token", paged=True)
        assert_attn_close(out, c.oracle_decode(q, seq, f32_scale(D)), f"paged call {call}")

"""The host pager driving the paged GPU path: tables and write positions come
from kvq_pager_* (append, popn rollback, release, page reuse), the INT8 arena
is written by kvq_append_paged and read by kvq_decode_attn, and every decode
is checked against the oracle run on the same table (bytes bit-exact,
attention within the fp64 bar)."""
import pytest
import torch

import oracle
from kvq_testutil import assert_attn_close, bf16_randn, f32_scale, kvq

pytestmark = pytest.mark.gpu


def test_pager_drives_paged_append_and_decode():
    m = kvq()
    B, Hq, Hk, D, npg, mp = 4, 16, 4, 128, 64, 24
    pager = m.Pager(npg, B, mp)
    dev = "cuda"
    shape = (npg, Hk, 16, D)
    k = torch.zeros(shape, dtype=torch.uint8, device=dev)
    v = torch.zeros_like(k)
    ks = torch.zeros(npg, Hk, 16, 1, device=dev)
    vs = torch.zeros_like(ks)
    ok, ov = torch.zeros(shape, dtype=torch.uint8), torch.zeros(shape, dtype=torch.uint8)
    oks, ovs = torch.zeros(npg, Hk, 16, 1), torch.zeros(npg, Hk, 16, 1)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    g = torch.Generator().manual_seed(11)
    seed = [100]

    def append(lens_new):
        """Append lens_new[b] tokens to each sequence (0 = none) as one call
        per distinct chunk length, through the pager's positions and table."""
        for b, n in enumerate(lens_new):
            if n == 0:
                continue
            pos = pager.append(b, n)
            kn = torch.randn(1, Hk, n, D, generator=g).to(torch.bfloat16)
            vn = torch.randn(1, Hk, n, D, generator=g).to(torch.bfloat16)
            tb = pager.table()[b:b + 1].clone()
            p = torch.tensor([pos], dtype=torch.int32)
            m.kvq_append_paged(kn.to(dev), vn.to(dev), p.to(dev), k, v, ks, vs, tb.to(dev), 16,
                               err=err)
            assert oracle.append_paged(kn, p, ok, oks, tb) == 0
            assert oracle.append_paged(vn, p, ov, ovs, tb) == 0

    def decode_and_check(what):
        seed[0] += 1
        q = bf16_randn((B, Hq, D), seed=seed[0])
        lens = pager.lens().clone()
        tb = pager.table().clone()
        hint = max(int(lens.max()), 1)
        out = m.kvq_decode_attn(q.to(dev), k, v, ks, vs, lens.to(dev), hint, page_table=tb.to(dev),
                                page_size=16, attn_scale=f32_scale(D), err=err)
        ref = oracle.decode_attn(q, ok, ov, oks, ovs, lens, f32_scale(D), page_size=16, table=tb)
        assert_attn_close(out, ref, what)
        assert m.kvq_read_error(err) == 0
        torch.cuda.synchronize()
        assert torch.equal(k.cpu(), ok) and torch.equal(v.cpu(), ov)
        assert torch.equal(ks.cpu(), oks) and torch.equal(vs.cpu(), ovs)

    append([300, 17, 64, 129])                       # prefill (ragged, page edges)
    decode_and_check("prefill")
    for step in range(3):                            # decode steps
        append([1, 1, 1, 1])
        decode_and_check(f"decode step {step}")
    assert pager.popn(0, 40) == 40                   # rollback: pages freed
    assert pager.popn(2, 3) == 3
    append([5, 0, 3, 0])                             # overwrite the rolled-back slots
    decode_and_check("after rollback")
    pager.release(1)                                 # sequence 1 finished: pages reused
    free_before = pager.num_free()
    append([0, 200, 0, 0])
    assert pager.num_free() == free_before - 13
    decode_and_check("after release and regrowth")

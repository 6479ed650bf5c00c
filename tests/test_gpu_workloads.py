"""GPU parity at the five workloads' full sizes, in the launch configuration
the benchmark times (automatic split plan): the cache is built through
kvq_append / kvq_append_paged (prefill, then the decode token), its bytes and
scales are compared bit-exactly with the oracle's own cache built from the
same bf16 inputs, and decode attention is compared with the oracle's fp64
attention over the oracle's cache on every output."""
import pytest
import torch

import synth
from kvq_testutil import ContigCache, PagedCache, assert_attn_close, f32_scale, kvq

pytestmark = pytest.mark.gpu


def _run_contig(wl, inp):
    B, Hk, D = wl.B, wl.Hk, wl.D
    Lmax = int(inp.cached.max())
    c = ContigCache(B, Hk, Lmax + 1, D, wl.mode)
    chunk = wl.prefill_chunk or Lmax
    for p0 in range(0, Lmax, chunk):
        T = min(chunk, Lmax - p0)
        k = inp.k_hist[:, :, p0:p0 + T].contiguous()
        v = inp.v_hist[:, :, p0:p0 + T].contiguous()
        assert c.append(k, v, torch.full((B,), p0, dtype=torch.int32)) == 0
    # the decode token goes to position cached[b]
    assert c.append(inp.k_new, inp.v_new, inp.cached) == 0
    return c


def _run_paged(wl, inp):
    B, Hk, D = wl.B, wl.Hk, wl.D
    c = PagedCache(inp.num_pages, Hk, D, wl.mode, inp.page_table)
    for b in range(B):
        L = int(inp.cached[b])
        k = inp.k_hist[b:b + 1, :, :L].contiguous()
        v = inp.v_hist[b:b + 1, :, :L].contiguous()
        assert c.append(k, v, torch.zeros(1, dtype=torch.int32), rows=[b]) == 0
    assert c.append(inp.k_new, inp.v_new, inp.cached) == 0
    return c


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_full_size(name):
    wl = synth.WORKLOADS[name]
    inp = synth.make_decode_inputs(wl)
    c = _run_paged(wl, inp) if wl.layout == "paged" else _run_contig(wl, inp)
    c.assert_bit_exact()
    hint = int(inp.seq_lens.max())
    sc = f32_scale(wl.D)
    out = c.decode(inp.q, inp.seq_lens, hint, attn_scale=sc)
    ref = c.oracle_decode(inp.q, inp.seq_lens, sc)
    max_abs, rel = assert_attn_close(out, ref, name)
    assert kvq().kvq_read_error(c.err) == 0
    print(f"{name}: max-abs {max_abs:.2e} rel-L2 {rel:.2e}")

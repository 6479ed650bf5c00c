"""GPU parity of the shapes the CUDA-core split kernel takes: head dims other
than 64 and 128 (every D % 16 == 0 up to 256), more than 16 (head, query)
rows per kv head outside the dense kernel's shapes, and batches above 1024
sequences.  Decode, paged decode, chunks, windows, the FP8 and per-head /
per-channel formats, the one-call decode step, and the separate combine
launch for D > 128, each against the oracle (bit-exact bytes, attention
within max-abs 2e-3 and relative-L2 1e-3)."""
import pytest
import torch

import oracle
from kvq_testutil import (ContigCache, PagedCache, assert_attn_close, bf16_randn, f32_scale,
                          kvq)

pytestmark = pytest.mark.gpu


def _contig(B, Hk, D, mode, lens, seed, extra=2):
    S = max(max(lens), 1) + extra
    c = ContigCache(B, Hk, S, D, mode)
    L = max(lens)
    if L:
        assert c.append(bf16_randn((B, Hk, L, D), seed), bf16_randn((B, Hk, L, D), seed + 1),
                        torch.zeros(B, dtype=torch.int32)) == 0
    return c


def _paged(B, Hk, D, mode, lens, seed, spare=3, fill=None):
    """Paged arena whose table covers lens; the first fill[b] (default lens[b])
    tokens of every sequence are appended."""
    fill = lens if fill is None else fill
    need = [(L + 15) // 16 for L in lens]
    gen = torch.Generator().manual_seed(seed)
    num_pages = sum(need) + spare
    perm = torch.randperm(num_pages, generator=gen).to(torch.int32)
    table = torch.full((B, max(max(need), 1)), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    c = PagedCache(num_pages, Hk, D, mode, table)
    for b, L in enumerate(fill):
        if L:
            assert c.append(bf16_randn((1, Hk, L, D), seed + 10 + b, 0.5),
                            bf16_randn((1, Hk, L, D), seed + 50 + b, 0.5),
                            torch.zeros(1, dtype=torch.int32), rows=[b]) == 0
    return c


def _modes(D):
    return ["per_token", "group32"] if D % 32 == 0 else ["per_token"]


CASES = [(D, mode) for D in (16, 32, 48, 96, 160, 256) for mode in _modes(D)]


@pytest.mark.parametrize("D,mode", CASES)
@pytest.mark.parametrize("G", [1, 4, 8])
def test_decode_other_head_dims(D, mode, G):
    B, Hk = 3, 2
    lens = [1, 130, 1100]
    c = _contig(B, Hk, D, mode, lens, seed=D + G)
    q = bf16_randn((B, Hk * G, D), seed=D * 3 + G)
    sl = torch.tensor(lens, dtype=torch.int32)
    ref = c.oracle_decode(q, sl, f32_scale(D))
    for ns in (0, 1, 3):
        assert_attn_close(c.decode(q, sl, max(lens), attn_scale=f32_scale(D), num_splits=ns),
                          ref, f"D={D} {mode} G={G} ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("D", [32, 96, 256])
@pytest.mark.parametrize("mode", ["per_token", "group32"])
def test_decode_paged_other_head_dims(D, mode):
    lens = [16, 47, 300]
    c = _paged(3, 2, D, mode, lens, seed=D)
    c.assert_bit_exact()
    q = bf16_randn((3, 8, D), seed=D + 1)
    sl = torch.tensor(lens, dtype=torch.int32)
    for ns in (0, 5):
        assert_attn_close(c.decode(q, sl, max(lens), attn_scale=f32_scale(D), num_splits=ns),
                          c.oracle_decode(q, sl, f32_scale(D)), f"paged D={D} ns={ns}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("D", [32, 96, 256])
@pytest.mark.parametrize("T", [2, 5])
def test_chunk_other_head_dims(D, T):
    B, Hk, G = 2, 2, 4                      # T = 5: 20 rows per kv head
    lens = [T + 3, 700]
    c = _contig(B, Hk, D, "per_token", lens, seed=D + T)
    q = bf16_randn((B, Hk * G, T, D), seed=D * T)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = c.chunk(q, sl, max(lens), attn_scale=f32_scale(D), num_splits=3)
    assert_attn_close(out, c.oracle_chunk(q, sl, f32_scale(D)), f"chunk D={D} T={T}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("D,mode", [(64, "per_token"), (64, "group32"), (128, "group32")])
def test_chunk_rows_beyond_sixteen_outside_the_dense_kernel(D, mode):
    """More than 16 rows per kv head in shapes the dense tensor-core kernel
    does not cover run on the CUDA-core split kernel."""
    B, Hk, G, T = 2, 2, 8, 6                # 48 rows per kv head
    lens = [T, 900]
    c = _contig(B, Hk, D, mode, lens, seed=7 + D)
    q = bf16_randn((B, Hk * G, T, D), seed=8 + D)
    sl = torch.tensor(lens, dtype=torch.int32)
    assert_attn_close(c.chunk(q, sl, max(lens), attn_scale=f32_scale(D)),
                      c.oracle_chunk(q, sl, f32_scale(D)), f"rows>16 D={D} {mode}")
    assert kvq().kvq_read_error(c.err) == 0


@pytest.mark.parametrize("D", [96, 256])
def test_window_other_head_dims(D):
    m = kvq()
    B, Hk, G = 2, 2, 4
    lens = [50, 1200]
    c = _contig(B, Hk, D, "per_token", lens, seed=D + 5)
    sl = torch.tensor(lens, dtype=torch.int32)
    q = bf16_randn((B, Hk * G, D), seed=D + 6)
    for w in (20, 333):
        out = m.kvq_window_attn(q.cuda(), c.k, c.v, c.ks, c.vs, sl.cuda(), max(lens), w,
                                attn_scale=f32_scale(D), err=c.err)
        assert_attn_close(out, oracle.window_attn(q, c.ok, c.ov, c.oks, c.ovs, sl, w,
                                                  f32_scale(D)), f"window D={D} w={w}")
    q4 = bf16_randn((B, Hk * G, 3, D), seed=D + 7)
    out = m.kvq_window_attn(q4.cuda(), c.k, c.v, c.ks, c.vs, sl.cuda(), max(lens), 64,
                            attn_scale=f32_scale(D), err=c.err)
    assert_attn_close(out, oracle.window_attn(q4, c.ok, c.ov, c.oks, c.ovs, sl, 64,
                                              f32_scale(D)), f"window chunk D={D}")
    assert m.kvq_read_error(c.err) == 0


@pytest.mark.parametrize("fmt", ["fp8_e4m3", "fp8_e5m2"])
@pytest.mark.parametrize("D", [96, 256])
def test_fp8_other_head_dims(fmt, D):
    m = kvq()
    B, Hk, G = 2, 2, 4
    lens = [1, 900]
    S = max(lens) + 1
    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8, device="cuda")
    v = torch.zeros_like(k)
    ok, ov = k.cpu(), v.cpu()
    kn = bf16_randn((B, Hk, max(lens), D), seed=D, sigma=2.0)
    vn = bf16_randn((B, Hk, max(lens), D), seed=D + 1, sigma=2.0)
    pos = torch.zeros(B, dtype=torch.int32)
    m.kvq_append(kn.cuda(), vn.cuda(), pos.cuda(), k, v, None, None, fmt)
    oracle.append_fp8(kn, pos, ok, fmt)
    oracle.append_fp8(vn, pos, ov, fmt)
    torch.cuda.synchronize()
    assert torch.equal(k.cpu(), ok) and torch.equal(v.cpu(), ov)
    q = bf16_randn((B, Hk * G, D), seed=D + 2)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = m.kvq_decode_attn(q.cuda(), k, v, None, None, sl.cuda(), max(lens), mode=fmt,
                            attn_scale=f32_scale(D))
    assert_attn_close(out, oracle.fp8_attn(q, ok, ov, sl, fmt, 0, f32_scale(D)), f"{fmt} D={D}")


@pytest.mark.parametrize("gran", ["per_head", "per_channel"])
@pytest.mark.parametrize("D", [96, 256])
def test_static_scales_other_head_dims(gran, D):
    m = kvq()
    B, Hk, G = 2, 2, 4
    lens = [1, 900]
    S = max(lens) + 1
    ns = 1 if gran == "per_head" else D
    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8, device="cuda")
    v = torch.zeros_like(k)
    ks = torch.zeros(B, Hk, ns, device="cuda")
    vs = torch.zeros_like(ks)
    ok, ov, oks, ovs = k.cpu(), v.cpu(), ks.cpu(), vs.cpu()
    kn = bf16_randn((B, Hk, max(lens), D), seed=D + 3)
    vn = bf16_randn((B, Hk, max(lens), D), seed=D + 4)
    pos = torch.zeros(B, dtype=torch.int32)
    m.kvq_append_calibrate(kn.cuda(), vn.cuda(), pos.cuda(), k, v, ks, vs, gran)
    oracle.append_static(kn, pos, ok, oks, gran, True)
    oracle.append_static(vn, pos, ov, ovs, gran, True)
    torch.cuda.synchronize()
    assert torch.equal(k.cpu(), ok) and torch.equal(ks.cpu().view(torch.int32),
                                                    oks.view(torch.int32))
    q = bf16_randn((B, Hk * G, D), seed=D + 5)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = m.kvq_decode_attn(q.cuda(), k, v, ks, vs, sl.cuda(), max(lens), mode=gran,
                            attn_scale=f32_scale(D))
    assert_attn_close(out, oracle.static_attn(q, ok, ov, oks, ovs, sl, gran, 0, f32_scale(D)),
                      f"{gran} D={D}")


@pytest.mark.parametrize("D", [32, 96, 256])
@pytest.mark.parametrize("mode", ["per_token", "group32"])
@pytest.mark.parametrize("paged", [False, True])
def test_append_decode_other_head_dims(D, mode, paged):
    """The one-call decode step on the CUDA-core kernel: the new token's bytes
    and scales bit-exact with the oracle's append, the output within the bar,
    and exactly the output of the two-call step."""
    m = kvq()
    B, Hk, G = 3, 2, 4
    lens = [1, 17, 400]
    hist = [L - 1 for L in lens]
    if paged:                           # the table covers the new token's page too
        c = _paged(B, Hk, D, mode, lens, seed=D + 9, fill=hist)
    else:
        c = _contig(B, Hk, D, mode, hist, seed=D + 9)
    k_new = bf16_randn((B, Hk, 1, D), seed=D + 11)
    v_new = bf16_randn((B, Hk, 1, D), seed=D + 12)
    q = bf16_randn((B, Hk * G, D), seed=D + 13)
    sl = torch.tensor(lens, dtype=torch.int32)
    extra = dict(page_table=c.table, page_size=16) if paged else {}
    kc, vc, ksc, vsc = c.k.clone(), c.v.clone(), c.ks.clone(), c.vs.clone()
    out = m.kvq_append_decode(q.cuda(), k_new.cuda(), v_new.cuda(), c.k, c.v, c.ks, c.vs,
                              sl.cuda(), max(lens), mode=mode, attn_scale=f32_scale(D),
                              err=c.err, **extra)
    pos = (sl - 1).to(torch.int32)
    if paged:
        oracle.append_paged(k_new, pos, c.ok, c.oks, c.table_cpu, 16, mode)
        oracle.append_paged(v_new, pos, c.ov, c.ovs, c.table_cpu, 16, mode)
    else:
        oracle.append_contig(k_new, pos, c.ok, c.oks, mode)
        oracle.append_contig(v_new, pos, c.ov, c.ovs, mode)
    c.assert_bit_exact()
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), f"fused D={D} {mode}")
    assert m.kvq_read_error(c.err) == 0
    # the two-call step on the saved cache
    if paged:
        m.kvq_append_paged(k_new.cuda(), v_new.cuda(), pos.cuda(), kc, vc, ksc, vsc, c.table, 16,
                           mode)
    else:
        m.kvq_append(k_new.cuda(), v_new.cuda(), pos.cuda(), kc, vc, ksc, vsc, mode)
    ref = m.kvq_decode_attn(q.cuda(), kc, vc, ksc, vsc, sl.cuda(), max(lens), mode=mode,
                            attn_scale=f32_scale(D), **extra)
    torch.cuda.synchronize()
    assert torch.equal(kc, c.k) and torch.equal(ksc.view(torch.int32), c.ks.view(torch.int32))
    assert torch.equal(out, ref)


def test_batch_above_1024_sequences():
    B, Hk, G, D = 1100, 2, 4, 128
    gen = torch.Generator().manual_seed(3)
    lens = torch.randint(0, 90, (B,), generator=gen).tolist()
    c = _contig(B, Hk, D, "per_token", lens, seed=41)
    q = bf16_randn((B, Hk * G, D), seed=42)
    sl = torch.tensor(lens, dtype=torch.int32)
    assert_attn_close(c.decode(q, sl, max(lens), attn_scale=f32_scale(D)),
                      c.oracle_decode(q, sl, f32_scale(D)), "B=1100")
    assert kvq().kvq_read_error(c.err) == 0


def test_d256_many_units_combine_in_two_halves():
    """Many split units at D = 256: the combine kernel folds the partials in
    two 128-column halves (scratch workspace full of junk on entry)."""
    m = kvq()
    B, Hk, G, D = 520, 8, 2, 256
    gen = torch.Generator().manual_seed(9)
    lens = torch.randint(129, 300, (B,), generator=gen).tolist()
    c = _contig(B, Hk, D, "per_token", lens, seed=51)
    q = bf16_randn((B, Hk * G, D), seed=52)
    sl = torch.tensor(lens, dtype=torch.int32)
    need = m.kvq_decode_workspace_bytes(B, Hk * G, Hk, D, max(lens))
    ws = torch.full((need,), 0x5A, dtype=torch.uint8, device="cuda")
    out = c.decode(q, sl, max(lens), attn_scale=f32_scale(D), workspace=ws)
    assert_attn_close(out, c.oracle_decode(q, sl, f32_scale(D)), "D=256 combine launch")

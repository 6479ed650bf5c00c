"""GPU parity of dense chunk attention (more than 16 (query, head) rows per
kv head: the tcgen05 kernel) against the oracle: full comparison on small
chunks (one and several 128-row tiles, ragged last tiles, chunks that fill
their cache, key ranges not a multiple of the 128-token tile), and, at the
long-context workload's full size (a 2048-token prefill chunk over 131072
cached tokens, GQA 8), sampled query rows against the oracle's decode
attention over the truncated cache (row i of a chunk attends to the first
L - T + i + 1 positions)."""
import pytest
import torch

import oracle
import synth
from kvq_testutil import ContigCache, assert_attn_close, bf16_randn, f32_scale, kvq

pytestmark = pytest.mark.gpu


def _contig(B, Hk, D, lens, seed, sigma=1.0):
    S = max(lens)
    c = ContigCache(B, Hk, S, D, "per_token")
    k = bf16_randn((B, Hk, S, D), seed, sigma)
    v = bf16_randn((B, Hk, S, D), seed + 1, sigma)
    assert c.append(k, v, torch.zeros(B, dtype=torch.int32)) == 0
    return c


@pytest.mark.parametrize("G,T,lens", [
    (8, 4, [4, 300]),            # 32 rows: one tile, a chunk that fills its cache
    (4, 33, [33, 129]),          # 132 rows: two tiles, the second one of 4 rows
    (1, 130, [130, 1000]),       # 130 rows, one head per kv head
    (8, 64, [64, 2049]),         # 512 rows: four full tiles
    (2, 200, [777, 256]),        # 400 rows, keys up to 777
])
def test_dense_chunk_matches_oracle(G, T, lens):
    B, Hk, D = len(lens), 2, 128
    c = _contig(B, Hk, D, lens, seed=G + T)
    q = bf16_randn((B, Hk * G, T, D), seed=T)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = c.chunk(q, sl, max(lens), attn_scale=f32_scale(D))
    assert_attn_close(out, c.oracle_chunk(q, sl, f32_scale(D)), f"G={G} T={T} lens={lens}")
    assert kvq().kvq_read_error(c.err) == 0


def test_dense_chunk_peaky_and_outliers():
    """Scores spread far apart (large |q|, outlier channels): the online max
    rises across tiles and the O rescale in tensor memory is exercised."""
    B, Hk, G, T, D = 1, 2, 8, 40, 128
    lens = [1500]
    c = _contig(B, Hk, D, lens, seed=5, sigma=3.0)
    q = bf16_randn((B, Hk * G, T, D), seed=6, sigma=4.0)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = c.chunk(q, sl, max(lens), attn_scale=f32_scale(D))
    assert_attn_close(out, c.oracle_chunk(q, sl, f32_scale(D)), "peaky")


def test_dense_chunk_length_rules():
    m = kvq()
    B, Hk, G, T, D = 3, 1, 8, 4, 128
    lens = [0, 2, 50]                     # empty: zero rows; shorter than the chunk: flagged
    c = _contig(B, Hk, D, [50, 50, 50], seed=7)
    q = bf16_randn((B, Hk * G, T, D), seed=8)
    sl = torch.tensor(lens, dtype=torch.int32)
    out = c.chunk(q, sl, 50, attn_scale=f32_scale(D))
    assert m.kvq_read_error(c.err) & 4
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[1]) == 0
    ref = c.oracle_chunk(q, sl, f32_scale(D))           # (rows of 0 and 2 are zero there too)
    assert_attn_close(out, ref, "all rows")


def test_dense_shapes_outside_the_tcgen05_kernel():
    """A dense chunk the tcgen05 kernel does not cover (group-32 scales) runs
    on the CUDA-core split kernel, within the bar of the oracle."""
    c = ContigCache(1, 1, 64, 128, "group32")
    kn = bf16_randn((1, 1, 64, 128), seed=10)
    vn = bf16_randn((1, 1, 64, 128), seed=11)
    assert c.append(kn, vn, torch.zeros(1, dtype=torch.int32)) == 0
    q = bf16_randn((1, 8, 4, 128), seed=9)          # 32 rows per kv head
    sl = torch.tensor([64], dtype=torch.int32)
    out = c.chunk(q, sl, 64, attn_scale=f32_scale(128))
    assert_attn_close(out, c.oracle_chunk(q, sl, f32_scale(128)), "dense group-32")
    assert kvq().kvq_read_error(c.err) == 0


def test_dense_chunk_long_context_full_size_sampled_rows():
    """The long-context workload: 131072 cached tokens + a 2048-token prefill
    chunk, Hq 64, Hk 8 (16384 rows per kv head, 128 tiles of 128 rows).
    Sampled queries (tile edges included) against the oracle's decode over the
    truncated cache."""
    m = kvq()
    wl = synth.WORKLOADS["long_context"]
    T = 2048
    inp = synth.make_decode_inputs(wl, qlen=T)
    B, Hk, D = wl.B, wl.Hk, wl.D
    L = int(inp.seq_lens[0])
    S = L
    dev = "cuda"
    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8, device=dev)
    v = torch.zeros_like(k)
    ks = torch.zeros(B, Hk, S, 1, device=dev)
    vs = torch.zeros_like(ks)
    for p0 in range(0, L - T, 8192):
        n = min(8192, L - T - p0)
        m.kvq_append(inp.k_hist[:, :, p0:p0 + n].contiguous().to(dev),
                     inp.v_hist[:, :, p0:p0 + n].contiguous().to(dev),
                     torch.full((B,), p0, dtype=torch.int32, device=dev), k, v, ks, vs)
    m.kvq_append(inp.k_new.to(dev), inp.v_new.to(dev),
                 torch.full((B,), L - T, dtype=torch.int32, device=dev), k, v, ks, vs)
    sl = inp.seq_lens.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out = m.kvq_chunk_attn(inp.q.to(dev), k, v, ks, vs, sl, L, attn_scale=f32_scale(D), err=err)
    assert m.kvq_read_error(err) == 0
    kc, vc, ksc, vsc = k.cpu(), v.cpu(), ks.cpu(), vs.cpu()
    for i in (0, 1, 15, 16, 17, 1000, T - 2, T - 1):
        qi = inp.q[:, :, i].contiguous()                      # [B, Hq, D]
        ref = oracle.decode_attn(qi, kc, vc, ksc, vsc, torch.tensor([L - T + i + 1],
                                                                    dtype=torch.int32),
                                 f32_scale(D))
        assert_attn_close(out[:, :, i], ref, f"query {i}")

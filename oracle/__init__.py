"""CPU oracle for INT8 KV-cache append, dequantization, decode attention and
chunk attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline / reference leg may import this package.  It is
a thin ctypes binding over ``kvq_oracle.c`` (plain scalar C: fp32 IEEE
quantisation, fp64 attention) and shares nothing with the CUDA library.

Parity pins: every routine here is pinned by ``tests/test_oracle_*.py``
(worked examples from the pages, closed forms, invariants and an
independent library routine for attention).
"""
from __future__ import annotations

import ctypes
import math

import torch

from . import _build

_lib = None

ORACLE_ERR_POS = 1
ORACLE_ERR_PAGE = 2
ORACLE_ERR_LEN = 4


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        lib.oracle_quantize_rows.argtypes = [P, I64, I, I, P, P]
        lib.oracle_quantize_rows.restype = None
        lib.oracle_dequant_rows.argtypes = [P, P, I64, I, I, P]
        lib.oracle_dequant_rows.restype = None
        lib.oracle_append_contig.argtypes = [P, I, I, I, I, I, P, P, P, I]
        lib.oracle_append_contig.restype = I
        lib.oracle_append_paged.argtypes = [P, I, I, I, I, I, P, P, P, P, I, I, I]
        lib.oracle_append_paged.restype = I
        lib.oracle_decode_attn.argtypes = [P, I, I, I, I, I, P, P, P, P, I, I, P, I, I, P,
                                           ctypes.c_double, P]
        lib.oracle_decode_attn.restype = I
        lib.oracle_chunk_attn.argtypes = [P, I, I, I, I, I, I, P, P, P, P, I, I, P, I, I, P,
                                          ctypes.c_double, P]
        lib.oracle_chunk_attn.restype = I
        lib.oracle_window_attn.argtypes = [P, I, I, I, I, I, I, P, P, P, P, I, I, P, I, I, P, I,
                                           ctypes.c_double, P]
        lib.oracle_window_attn.restype = I
        lib.oracle_fp8_encode.argtypes = [ctypes.c_float, I]
        lib.oracle_fp8_encode.restype = ctypes.c_uint8
        lib.oracle_fp8_decode.argtypes = [ctypes.c_uint8, I]
        lib.oracle_fp8_decode.restype = ctypes.c_float
        lib.oracle_fp8_encode_rows.argtypes = [P, I64, I, P]
        lib.oracle_fp8_encode_rows.restype = None
        lib.oracle_append_fp8.argtypes = [P, I, I, I, I, I, P, P, I, I, P, I, I]
        lib.oracle_append_fp8.restype = I
        lib.oracle_fp8_attn.argtypes = [P, I, I, I, I, I, I, P, P, I, I, P, I, I, P, I,
                                        ctypes.c_double, P]
        lib.oracle_fp8_attn.restype = I
        lib.oracle_append_static.argtypes = [P, I, I, I, I, I, I, P, P, P, I]
        lib.oracle_append_static.restype = I
        lib.oracle_static_attn.argtypes = [P, I, I, I, I, I, I, P, P, P, P, I, P, I,
                                           ctypes.c_double, P]
        lib.oracle_static_attn.restype = I
        lib.oracle_append_mixed.argtypes = [P, I, I, I, I, I, P, P, P, P, I, I]
        lib.oracle_append_mixed.restype = I
        lib.oracle_mixed_attn.argtypes = [P, I, I, I, I, I, P, P, P, P, P, P, I, I, P,
                                          ctypes.c_double, P]
        lib.oracle_mixed_attn.restype = I
        lib.oracle_cache_bytes.argtypes = [I64] * 6
        lib.oracle_cache_bytes.restype = I64
        lib.oracle_fp32_cache_bytes.argtypes = [I64] * 4
        lib.oracle_fp32_cache_bytes.restype = I64
        _lib = lib
    return _lib


def _cpu(t: torch.Tensor, dtype) -> torch.Tensor:
    assert t.device.type == "cpu", "oracle works on CPU tensors"
    assert t.dtype == dtype, (t.dtype, dtype)
    return t.contiguous()


def _bits16(x: torch.Tensor) -> torch.Tensor:
    return _cpu(x, torch.bfloat16).view(torch.int16)


def group_of(mode: str, D: int) -> int:
    if mode == "per_token":
        return D
    if mode == "group32":
        return 32
    raise ValueError(mode)


def quantize(x: torch.Tensor, mode: str = "per_token"):
    """x bf16 [..., D] -> (u8 [..., D], fp32 scales [..., NG])."""
    D = x.shape[-1]
    grp = group_of(mode, D)
    xb = _bits16(x)
    rows = xb.numel() // D if D else 0
    q = torch.empty(x.shape, dtype=torch.uint8)
    s = torch.empty(*x.shape[:-1], D // grp, dtype=torch.float32)
    _load().oracle_quantize_rows(xb.data_ptr(), rows, D, grp, q.data_ptr(), s.data_ptr())
    return q, s


def dequant(q: torch.Tensor, scale: torch.Tensor, mode: str = "per_token") -> torch.Tensor:
    D = q.shape[-1]
    grp = group_of(mode, D)
    qc = _cpu(q, torch.uint8)
    sc = _cpu(scale, torch.float32)
    rows = qc.numel() // D if D else 0
    out = torch.empty(q.shape, dtype=torch.float32)
    _load().oracle_dequant_rows(qc.data_ptr(), sc.data_ptr(), rows, D, grp, out.data_ptr())
    return out


def append_contig(x_new, pos, cache, scale, mode="per_token") -> int:
    """Quantize x_new bf16 [B,Hk,T,D] into cache u8 [B,Hk,max_seq,D] at pos[b]."""
    B, Hk, T, D = x_new.shape
    grp = group_of(mode, D)
    assert cache.is_contiguous() and scale.is_contiguous()
    xb = _bits16(x_new)
    p = _cpu(pos, torch.int32)
    return _load().oracle_append_contig(xb.data_ptr(), B, Hk, T, D, grp, p.data_ptr(),
                                        cache.data_ptr(), scale.data_ptr(), cache.shape[2])


def append_paged(x_new, pos, arena, scale, table, page_size=16, mode="per_token") -> int:
    B, Hk, T, D = x_new.shape
    grp = group_of(mode, D)
    assert arena.is_contiguous() and scale.is_contiguous()
    xb = _bits16(x_new)
    p = _cpu(pos, torch.int32)
    tb = _cpu(table, torch.int32)
    return _load().oracle_append_paged(xb.data_ptr(), B, Hk, T, D, grp, p.data_ptr(),
                                       arena.data_ptr(), scale.data_ptr(), tb.data_ptr(),
                                       tb.shape[1], arena.shape[0], page_size)


def decode_attn(q, k, v, k_scale, v_scale, seq_lens, attn_scale=None, mode="per_token",
                Hk=None, page_size=0, table=None, return_err=False):
    """fp64 decode attention over the dequantized INT8 cache.

    q bf16 [B,Hq,D]; contiguous: k/v u8 [B,Hk,max_seq,D]; paged (page_size>0):
    arenas u8 [num_pages,Hk,page_size,D] plus table int32 [B,max_pages].
    Returns fp64 [B,Hq,D].
    """
    B, Hq, D = q.shape
    grp = group_of(mode, D)
    Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    qb = _bits16(q)
    kc, vc = _cpu(k, torch.uint8), _cpu(v, torch.uint8)
    ks, vs = _cpu(k_scale, torch.float32), _cpu(v_scale, torch.float32)
    sl = _cpu(seq_lens, torch.int32)
    out = torch.empty(B, Hq, D, dtype=torch.float64)
    if page_size > 0:
        tb = _cpu(table, torch.int32)
        err = _load().oracle_decode_attn(qb.data_ptr(), B, Hq, Hk, D, grp, kc.data_ptr(),
                                         vc.data_ptr(), ks.data_ptr(), vs.data_ptr(), 0,
                                         page_size, tb.data_ptr(), tb.shape[1], kc.shape[0],
                                         sl.data_ptr(), float(attn_scale), out.data_ptr())
    else:
        err = _load().oracle_decode_attn(qb.data_ptr(), B, Hq, Hk, D, grp, kc.data_ptr(),
                                         vc.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                                         kc.shape[2], 0, None, 0, 0, sl.data_ptr(),
                                         float(attn_scale), out.data_ptr())
    return (out, err) if return_err else out


def chunk_attn(q, k, v, k_scale, v_scale, seq_lens, attn_scale=None, mode="per_token",
               page_size=0, table=None, return_err=False):
    """fp64 attention of T chunk queries per (sequence, q head), causal from
    the chunk's end: query i of a sequence of length L (the chunk included)
    attends to positions 0 .. L - T + i.

    q bf16 [B,Hq,T,D]; cache arguments as for decode_attn.  Returns fp64
    [B,Hq,T,D].
    """
    B, Hq, T, D = q.shape
    grp = group_of(mode, D)
    Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    qb = _bits16(q)
    kc, vc = _cpu(k, torch.uint8), _cpu(v, torch.uint8)
    ks, vs = _cpu(k_scale, torch.float32), _cpu(v_scale, torch.float32)
    sl = _cpu(seq_lens, torch.int32)
    out = torch.empty(B, Hq, T, D, dtype=torch.float64)
    if page_size > 0:
        tb = _cpu(table, torch.int32)
        err = _load().oracle_chunk_attn(qb.data_ptr(), B, Hq, Hk, T, D, grp, kc.data_ptr(),
                                        vc.data_ptr(), ks.data_ptr(), vs.data_ptr(), 0,
                                        page_size, tb.data_ptr(), tb.shape[1], kc.shape[0],
                                        sl.data_ptr(), float(attn_scale), out.data_ptr())
    else:
        err = _load().oracle_chunk_attn(qb.data_ptr(), B, Hq, Hk, T, D, grp, kc.data_ptr(),
                                        vc.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                                        kc.shape[2], 0, None, 0, 0, sl.data_ptr(),
                                        float(attn_scale), out.data_ptr())
    return (out, err) if return_err else out


def window_attn(q, k, v, k_scale, v_scale, seq_lens, window, attn_scale=None,
                mode="per_token", page_size=0, table=None, return_err=False):
    """fp64 sliding-window attention: query i of a sequence of length L (the
    chunk's T tokens included) sits at position p = L - T + i and attends to
    positions max(0, p - window + 1) .. p.  q bf16 [B,Hq,D] (a decode step,
    T = 1) or [B,Hq,T,D]; cache arguments as for decode_attn.  Returns fp64
    with q's shape."""
    if q.dim() == 3:
        B, Hq, D = q.shape
        T = 1
    else:
        B, Hq, T, D = q.shape
    grp = group_of(mode, D)
    Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    qb = _bits16(q)
    kc, vc = _cpu(k, torch.uint8), _cpu(v, torch.uint8)
    ks, vs = _cpu(k_scale, torch.float32), _cpu(v_scale, torch.float32)
    sl = _cpu(seq_lens, torch.int32)
    out = torch.empty(*q.shape, dtype=torch.float64)
    if page_size > 0:
        tb = _cpu(table, torch.int32)
        err = _load().oracle_window_attn(qb.data_ptr(), B, Hq, Hk, T, D, grp, kc.data_ptr(),
                                         vc.data_ptr(), ks.data_ptr(), vs.data_ptr(), 0,
                                         page_size, tb.data_ptr(), tb.shape[1], kc.shape[0],
                                         sl.data_ptr(), int(window), float(attn_scale),
                                         out.data_ptr())
    else:
        err = _load().oracle_window_attn(qb.data_ptr(), B, Hq, Hk, T, D, grp, kc.data_ptr(),
                                         vc.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                                         kc.shape[2], 0, None, 0, 0, sl.data_ptr(), int(window),
                                         float(attn_scale), out.data_ptr())
    return (out, err) if return_err else out


FP8_FORMATS = {"fp8_e4m3": 0, "fp8_e5m2": 1}


def fp8_encode(x: torch.Tensor, fmt: str) -> torch.Tensor:
    """bf16 values -> FP8 bytes (the page's truncating encoders, with the
    readings stated in kvq_oracle.c)."""
    xb = _bits16(x)
    out = torch.empty(x.shape, dtype=torch.uint8)
    _load().oracle_fp8_encode_rows(xb.data_ptr(), xb.numel(), FP8_FORMATS[fmt], out.data_ptr())
    return out


def fp8_encode_f32(value: float, fmt: str) -> int:
    """One fp32 value -> its FP8 byte."""
    return int(_load().oracle_fp8_encode(float(value), FP8_FORMATS[fmt]))


def fp8_decode(c: torch.Tensor, fmt: str) -> torch.Tensor:
    """FP8 bytes -> their exact fp32 values (pure-Python loop: small inputs)."""
    f = _load().oracle_fp8_decode
    code = FP8_FORMATS[fmt]
    flat = _cpu(c, torch.uint8).reshape(-1).tolist()
    return torch.tensor([f(int(b), code) for b in flat], dtype=torch.float32).reshape(c.shape)


def append_fp8(x_new, pos, dst, fmt, page_size=0, table=None) -> int:
    """Encode x_new bf16 [B,Hk,T,D] into an FP8 cache: contiguous
    [B,Hk,max_seq,D] at pos[b], or a paged arena [num_pages,Hk,page_size,D]
    with table [B,max_pages]."""
    B, Hk, T, D = x_new.shape
    assert dst.is_contiguous()
    xb = _bits16(x_new)
    p = _cpu(pos, torch.int32)
    if page_size > 0:
        tb = _cpu(table, torch.int32)
        return _load().oracle_append_fp8(xb.data_ptr(), B, Hk, T, D, FP8_FORMATS[fmt],
                                         p.data_ptr(), dst.data_ptr(), 0, page_size,
                                         tb.data_ptr(), tb.shape[1], dst.shape[0])
    return _load().oracle_append_fp8(xb.data_ptr(), B, Hk, T, D, FP8_FORMATS[fmt], p.data_ptr(),
                                     dst.data_ptr(), dst.shape[2], 0, None, 0, 0)


def fp8_attn(q, k, v, seq_lens, fmt, window=0, attn_scale=None, page_size=0, table=None,
             return_err=False):
    """fp64 attention over an FP8 cache: q bf16 [B,Hq,D] (decode) or
    [B,Hq,T,D] (causal chunk); window > 0 adds the sliding-window rule.
    Returns fp64 with q's shape."""
    if q.dim() == 3:
        B, Hq, D = q.shape
        T = 1
    else:
        B, Hq, T, D = q.shape
    Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    qb = _bits16(q)
    kc, vc = _cpu(k, torch.uint8), _cpu(v, torch.uint8)
    sl = _cpu(seq_lens, torch.int32)
    out = torch.empty(*q.shape, dtype=torch.float64)
    f = FP8_FORMATS[fmt]
    if page_size > 0:
        tb = _cpu(table, torch.int32)
        err = _load().oracle_fp8_attn(qb.data_ptr(), B, Hq, Hk, T, D, f, kc.data_ptr(),
                                      vc.data_ptr(), 0, page_size, tb.data_ptr(), tb.shape[1],
                                      kc.shape[0], sl.data_ptr(), int(window), float(attn_scale),
                                      out.data_ptr())
    else:
        err = _load().oracle_fp8_attn(qb.data_ptr(), B, Hq, Hk, T, D, f, kc.data_ptr(),
                                      vc.data_ptr(), kc.shape[2], 0, None, 0, 0, sl.data_ptr(),
                                      int(window), float(attn_scale), out.data_ptr())
    return (out, err) if return_err else out


STATIC_GRAN = {"per_head": 1, "per_channel": 2}
MIXED_MODES = {"per_token": 0, "group32": 1, "per_head": 3, "per_channel": 4}


def append_static(x_new, pos, cache, scales, gran, calibrate=True) -> int:
    """Per-head / per-channel quantisation of x_new bf16 [B,Hk,T,D] into the
    contiguous cache at pos[b]; scales fp32 [B,Hk,1] or [B,Hk,D] are set from
    this call's tokens (calibrate) or read."""
    B, Hk, T, D = x_new.shape
    assert cache.is_contiguous() and scales.is_contiguous() and scales.dtype == torch.float32
    xb = _bits16(x_new)
    p = _cpu(pos, torch.int32)
    return _load().oracle_append_static(xb.data_ptr(), B, Hk, T, D, STATIC_GRAN[gran],
                                        int(bool(calibrate)), p.data_ptr(), cache.data_ptr(),
                                        scales.data_ptr(), cache.shape[2])


def static_attn(q, k, v, k_scales, v_scales, seq_lens, gran, window=0, attn_scale=None,
                return_err=False):
    """fp64 attention over a per-head / per-channel INT8 cache: q bf16 [B,Hq,D]
    (decode) or [B,Hq,T,D] (causal chunk), optional sliding window."""
    if q.dim() == 3:
        B, Hq, D = q.shape
        T = 1
    else:
        B, Hq, T, D = q.shape
    Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    qb = _bits16(q)
    kc, vc = _cpu(k, torch.uint8), _cpu(v, torch.uint8)
    ks, vs = _cpu(k_scales, torch.float32), _cpu(v_scales, torch.float32)
    sl = _cpu(seq_lens, torch.int32)
    out = torch.empty(*q.shape, dtype=torch.float64)
    err = _load().oracle_static_attn(qb.data_ptr(), B, Hq, Hk, T, D, STATIC_GRAN[gran],
                                     kc.data_ptr(), vc.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                                     kc.shape[2], sl.data_ptr(), int(window), float(attn_scale),
                                     out.data_ptr())
    return (out, err) if return_err else out


def append_mixed(x_new, lens_old, cache, scales, ring, mode="per_token", window=None) -> int:
    """Append to a mixed cache: x_new bf16 [B,Hk,T,D] joins the bf16 window
    ring [B,Hk,W,D]; tokens older than the window's W are quantised into the
    INT8 part cache [B,Hk,max_seq,D] with the mode's scales."""
    B, Hk, T, D = x_new.shape
    W = ring.shape[2] if window is None else int(window)
    assert ring.dtype == torch.bfloat16 and ring.is_contiguous() and cache.is_contiguous()
    xb = _bits16(x_new)
    lo = _cpu(lens_old, torch.int32)
    return _load().oracle_append_mixed(xb.data_ptr(), B, Hk, T, D, MIXED_MODES[mode],
                                       lo.data_ptr(), cache.data_ptr(), scales.data_ptr(),
                                       ring.view(torch.int16).data_ptr(), W, cache.shape[2])


def mixed_attn(q, k, v, k_scales, v_scales, rk, rv, seq_lens, mode="per_token",
               attn_scale=None, window=None, return_err=False):
    """fp64 decode attention over a mixed cache (INT8 part + bf16 window ring)."""
    B, Hq, D = q.shape
    Hk = k.shape[1]
    W = rk.shape[2] if window is None else int(window)
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    qb = _bits16(q)
    kc, vc = _cpu(k, torch.uint8), _cpu(v, torch.uint8)
    ks, vs = _cpu(k_scales, torch.float32), _cpu(v_scales, torch.float32)
    rkb, rvb = _bits16(rk), _bits16(rv)
    sl = _cpu(seq_lens, torch.int32)
    out = torch.empty(B, Hq, D, dtype=torch.float64)
    err = _load().oracle_mixed_attn(qb.data_ptr(), B, Hq, Hk, D, MIXED_MODES[mode],
                                    kc.data_ptr(), vc.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                                    rkb.data_ptr(), rvb.data_ptr(), W, kc.shape[2],
                                    sl.data_ptr(), float(attn_scale), out.data_ptr())
    return (out, err) if return_err else out


def cache_bytes(layers, Hk, seq, D, group, scale_bytes=4) -> int:
    return int(_load().oracle_cache_bytes(layers, Hk, seq, D, group, scale_bytes))


def fp32_cache_bytes(layers, Hk, seq, D) -> int:
    return int(_load().oracle_fp32_cache_bytes(layers, Hk, seq, D))


# ------------------------------------------------- all-core baseline build
_omp_lib = None


def _load_omp():
    global _omp_lib
    if _omp_lib is None:
        lib = ctypes.CDLL(_build.build_omp())
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.oracle_attn_units.argtypes = [P, I, I, I, I, I, I, P, P, P, P, I, I, P, I, I, P,
                                          ctypes.c_double, P, I]
        lib.oracle_attn_units.restype = I
        _omp_lib = lib
    return _omp_lib


def unit_tables(table: torch.Tensor, Hk: int, num_pages: int) -> torch.Tensor:
    """Per-(sequence, kv head) page ids of a paged arena seen as one-head
    pages: page p of head hk becomes p * Hk + hk (entries outside the arena
    stay -1).  int32 [B * Hk, max_pages]."""
    t = _cpu(table, torch.int32).to(torch.int64)
    ok = (t >= 0) & (t < num_pages)
    hk = torch.arange(Hk, dtype=torch.int64).view(1, Hk, 1)
    u = torch.where(ok.unsqueeze(1), t.unsqueeze(1) * Hk + hk, torch.full_like(hk, -1))
    return u.reshape(-1, t.shape[1]).to(torch.int32).contiguous()


def attn_units(q, k, v, k_scale, v_scale, seq_lens, attn_scale, mode="per_token",
               page_size=0, utables=None, num_pages=0, threads=1):
    """The oracle's decode (q [B,Hq,D]) or chunk (q [B,Hq,T,D]) attention run
    as one pinned-oracle call per (sequence, kv head) unit on `threads` host
    threads (baseline timing only; results equal decode_attn / chunk_attn).
    Paged caches take utables from unit_tables()."""
    if q.dim() == 3:
        B, Hq, D = q.shape
        T = 1
    else:
        B, Hq, T, D = q.shape
    grp = group_of(mode, D)
    Hk = k.shape[1]
    qb = _bits16(q)
    kc, vc = _cpu(k, torch.uint8), _cpu(v, torch.uint8)
    ks, vs = _cpu(k_scale, torch.float32), _cpu(v_scale, torch.float32)
    sl = _cpu(seq_lens, torch.int32)
    out = torch.empty(*q.shape, dtype=torch.float64)
    if page_size > 0:
        tb = _cpu(utables, torch.int32)
        err = _load_omp().oracle_attn_units(
            qb.data_ptr(), B, Hq, Hk, T, D, grp, kc.data_ptr(), vc.data_ptr(), ks.data_ptr(),
            vs.data_ptr(), 0, page_size, tb.data_ptr(), tb.shape[1], num_pages, sl.data_ptr(),
            float(attn_scale), out.data_ptr(), int(threads))
    else:
        err = _load_omp().oracle_attn_units(
            qb.data_ptr(), B, Hq, Hk, T, D, grp, kc.data_ptr(), vc.data_ptr(), ks.data_ptr(),
            vs.data_ptr(), kc.shape[2], 0, None, 0, 0, sl.data_ptr(), float(attn_scale),
            out.data_ptr(), int(threads))
    return out, err

"""Thin Python binding over libkvq (include/kvq.h): INT8 KV-cache append and
decode attention on B200 (sm_100a).

Every function here only checks tensor arguments and marshals raw device
pointers into the C ABI; all computation runs in the library's CUDA kernels.
Importing this package fails loudly if libkvq.so has not been built
(``python decode_attention_kvq_b200/build.py``); there is no CPU fallback.

Functions take torch CUDA tensors (PyTorch supplies device memory and
streams) and enqueue on the current CUDA stream unless ``stream`` is given.

A decode step on a contiguous cache (B sequences, Hk kv heads, head_dim D):

    k = torch.zeros(B, Hk, S, D, dtype=torch.uint8, device="cuda"); v = torch.zeros_like(k)
    ks = torch.zeros(B, Hk, S, 1, device="cuda"); vs = torch.zeros_like(ks)   # D // 32 for group32
    kvq_append(k_new, v_new, pos, k, v, ks, vs)        # bf16 [B, Hk, T, D] at pos[b]
    out = kvq_decode_attn(q, k, v, ks, vs, seq_lens, max_len)   # q bf16 [B, Hq, D]
    out = kvq_chunk_attn(qc, k, v, ks, vs, seq_lens, max_len)   # qc bf16 [B, Hq, T, D]

``seq_lens`` (int32 [B], on the device) counts the cached tokens including
the ones just appended; ``max_len`` is a host upper bound of it.
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from ._lib import KvqError, lib, LIB_PATH, check  # noqa: F401

PER_TOKEN = 0
GROUP32 = 1
FP8_E4M3 = 2
FP8_E5M2 = 3
PER_HEAD = 4
PER_CHANNEL = 5
DEVERR_POS = 1
DEVERR_PAGE = 2
DEVERR_LEN = 4

_MODES = {"per_token": PER_TOKEN, "group32": GROUP32, "fp8_e4m3": FP8_E4M3,
          "fp8_e5m2": FP8_E5M2, "per_head": PER_HEAD, "per_channel": PER_CHANNEL}
_MODES.update({v: v for v in list(_MODES.values())})


class CacheView(ctypes.Structure):
    """Mirror of ``kvq_cache_view``."""
    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("page_size", ctypes.c_int32),
        ("max_seq", ctypes.c_int32),
        ("page_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
    ]


def _mode(mode) -> int:
    try:
        return _MODES[mode]
    except KeyError:
        raise ValueError(f"unknown scale mode {mode!r}") from None


def _ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, ref: torch.Tensor) -> int:
    if stream is None:
        # the current stream of the tensor's device, as a raw handle (the
        # Stream object that torch.cuda.current_stream builds costs more
        # than the rest of a call)
        if _raw_stream is not None:
            return _raw_stream(ref.device.index)
        return torch.cuda.current_stream(ref.device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def num_groups(mode, D: int) -> int:
    """Scales per (token, kv head): 1 per token, D / 32 for group-32, 0 for FP8
    and for the per-head / per-channel modes (whose scales are per (sequence,
    kv head): see static_scales)."""
    m = _mode(mode)
    return 1 if m == PER_TOKEN else (D // 32 if m == GROUP32 else 0)


def static_scales(mode, D: int) -> int:
    """Scales per (sequence, kv head) of the per-head (1) / per-channel (D) modes."""
    m = _mode(mode)
    return 1 if m == PER_HEAD else (D if m == PER_CHANNEL else 0)


def kvq_append(k_new, v_new, pos, k_cache, v_cache, k_scale, v_scale, mode="per_token",
               err=None, stream=None):
    """Quantise k_new/v_new bf16 [B,Hk,T,D] into the contiguous cache at pos[b].

    k_cache/v_cache u8 [B,Hk,max_seq,D]; k_scale/v_scale fp32 [B,Hk,max_seq,NG]
    (None in the FP8 modes); pos int32 [B]; err optional int32 [1] device
    error word.
    """
    B, Hk, T, D = k_new.shape
    check(lib.kvq_append(
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        B, Hk, T, D, _mode(mode), _ptr(pos, torch.int32, "pos"),
        _ptr(k_cache, torch.uint8, "k_cache"), _ptr(v_cache, torch.uint8, "v_cache"),
        _ptr(k_scale, torch.float32, "k_scale"), _ptr(v_scale, torch.float32, "v_scale"),
        k_cache.shape[2], _ptr(err, torch.int32, "err"), _stream(stream, k_new)), "kvq_append")


def kvq_append_calibrate(k_new, v_new, pos, k_cache, v_cache, k_scale, v_scale,
                         mode="per_head", err=None, stream=None):
    """Per-head / per-channel quantisation of k_new/v_new bf16 [B,Hk,T,D] into
    the contiguous cache at pos[b], with the scales (fp32 [B,Hk,1] or
    [B,Hk,D]) first computed from these tokens."""
    B, Hk, T, D = k_new.shape
    check(lib.kvq_append_calibrate(
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        B, Hk, T, D, _mode(mode), _ptr(pos, torch.int32, "pos"),
        _ptr(k_cache, torch.uint8, "k_cache"), _ptr(v_cache, torch.uint8, "v_cache"),
        _ptr(k_scale, torch.float32, "k_scale"), _ptr(v_scale, torch.float32, "v_scale"),
        k_cache.shape[2], _ptr(err, torch.int32, "err"), _stream(stream, k_new)),
        "kvq_append_calibrate")


def kvq_append_paged(k_new, v_new, pos, k_arena, v_arena, k_scale, v_scale, page_table,
                     page_size=16, mode="per_token", err=None, stream=None):
    """Quantise k_new/v_new bf16 [B,Hk,T,D] into the paged arena.

    k_arena/v_arena u8 [num_pages,Hk,page_size,D]; scales fp32
    [num_pages,Hk,page_size,NG]; page_table int32 [B,max_pages].
    """
    B, Hk, T, D = k_new.shape
    check(lib.kvq_append_paged(
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        B, Hk, T, D, _mode(mode), _ptr(pos, torch.int32, "pos"),
        _ptr(k_arena, torch.uint8, "k_arena"), _ptr(v_arena, torch.uint8, "v_arena"),
        _ptr(k_scale, torch.float32, "k_scale"), _ptr(v_scale, torch.float32, "v_scale"),
        _ptr(page_table, torch.int32, "page_table"), page_table.shape[1], k_arena.shape[0],
        page_size, _ptr(err, torch.int32, "err"), _stream(stream, k_new)), "kvq_append_paged")


def cache_view(k, v, k_scale, v_scale, page_table=None, page_size=0) -> CacheView:
    """Build a kvq_cache_view over contiguous caches or paged arenas."""
    cv = CacheView()
    cv.k = _ptr(k, torch.uint8, "k")
    cv.v = _ptr(v, torch.uint8, "v")
    cv.k_scale = _ptr(k_scale, torch.float32, "k_scale")
    cv.v_scale = _ptr(v_scale, torch.float32, "v_scale")
    if page_size:
        cv.page_size = page_size
        cv.max_seq = 0
        cv.page_table = _ptr(page_table, torch.int32, "page_table")
        cv.max_pages = page_table.shape[1]
        cv.num_pages = k.shape[0]
    else:
        cv.page_size = 0
        cv.max_seq = k.shape[2]
        cv.page_table = 0
        cv.max_pages = 0
        cv.num_pages = 0
    return cv


def new_workspace(nbytes, device) -> torch.Tensor:
    """A split-K workspace of nbytes bytes (its contents are scratch)."""
    return torch.empty(int(nbytes), dtype=torch.uint8, device=device)


def kvq_decode_workspace_bytes(B, Hq, Hk, D, max_seq_len_hint, num_splits=0) -> int:
    return int(lib.kvq_decode_workspace_bytes(B, Hq, Hk, D, max_seq_len_hint, num_splits))


def kvq_decode_plan(B, Hk, max_seq_len_hint, num_splits=0, num_sms=0):
    """(chunk tokens per split, splits of the longest sequence)."""
    chunk, splits = ctypes.c_int(0), ctypes.c_int(0)
    check(lib.kvq_decode_plan(B, Hk, max_seq_len_hint, num_splits, num_sms,
                              ctypes.byref(chunk), ctypes.byref(splits)), "kvq_decode_plan")
    return chunk.value, splits.value


def kvq_decode_attn(q, k, v, k_scale, v_scale, seq_lens, max_seq_len_hint, *, Hk=None,
                    page_table=None, page_size=0, attn_scale=None, mode="per_token",
                    out=None, workspace=None, num_splits=0, err=None, stream=None,
                    view: Optional[CacheView] = None):
    """Decode attention of q bf16 [B,Hq,D] over the INT8 cache; returns fp32 [B,Hq,D].

    Contiguous cache: k/v u8 [B,Hk,max_seq,D].  Paged: arenas
    [num_pages,Hk,16,D] with page_table int32 [B,max_pages] and page_size=16.
    seq_lens int32 [B] counts the cached tokens including the newest one.
    """
    B, Hq, D = q.shape
    if Hk is None:
        Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    if view is None:
        view = cache_view(k, v, k_scale, v_scale, page_table, page_size)
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    if workspace is None:               # (a given workspace's size is checked by the call)
        need = kvq_decode_workspace_bytes(B, Hq, Hk, D, max_seq_len_hint, num_splits)
        if need > 0:
            workspace = new_workspace(need, q.device)
    ws_ptr = _ptr(workspace, None, "workspace") if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    check(lib.kvq_decode_attn(
        _ptr(q, torch.bfloat16, "q"), B, Hq, Hk, D, _mode(mode), ctypes.byref(view),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(max_seq_len_hint), float(attn_scale),
        _ptr(out, torch.float32, "out"), ws_ptr, ws_bytes, int(num_splits),
        _ptr(err, torch.int32, "err"), _stream(stream, q)), "kvq_decode_attn")
    return out


def kvq_append_decode(q, k_new, v_new, k, v, k_scale, v_scale, seq_lens, max_seq_len_hint, *,
                      Hk=None, page_table=None, page_size=0, attn_scale=None,
                      mode="per_token", out=None, workspace=None, num_splits=0, err=None,
                      stream=None, view: Optional[CacheView] = None):
    """One decode step in one call: k_new / v_new bf16 [B,Hk,1,D] are quantised
    into position seq_lens[b] - 1 of the cache (written in place), then q bf16
    [B,Hq,D] attends to positions 0 .. seq_lens[b] - 1; returns fp32 [B,Hq,D].
    seq_lens counts the tokens INCLUDING the new one.  Cache arguments as for
    kvq_decode_attn (per_token or group32 mode)."""
    B, Hq, D = q.shape
    if Hk is None:
        Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    if view is None:
        view = cache_view(k, v, k_scale, v_scale, page_table, page_size)
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    if workspace is None:               # (a given workspace's size is checked by the call)
        need = kvq_decode_workspace_bytes(B, Hq, Hk, D, max_seq_len_hint, num_splits)
        if need > 0:
            workspace = new_workspace(need, q.device)
    ws_ptr = _ptr(workspace, None, "workspace") if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    check(lib.kvq_append_decode(
        _ptr(q, torch.bfloat16, "q"), _ptr(k_new, torch.bfloat16, "k_new"),
        _ptr(v_new, torch.bfloat16, "v_new"), B, Hq, Hk, D, _mode(mode), ctypes.byref(view),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(max_seq_len_hint), float(attn_scale),
        _ptr(out, torch.float32, "out"), ws_ptr, ws_bytes, int(num_splits),
        _ptr(err, torch.int32, "err"), _stream(stream, q)), "kvq_append_decode")
    return out


def kvq_chunk_attn(q, k, v, k_scale, v_scale, seq_lens, max_seq_len_hint, *, Hk=None,
                   page_table=None, page_size=0, attn_scale=None, mode="per_token",
                   out=None, workspace=None, num_splits=0, err=None, stream=None,
                   view: Optional[CacheView] = None):
    """Attention of a chunk of T queries per (sequence, q head), causal from
    the chunk's end; returns fp32 [B,Hq,T,D].

    q bf16 [B,Hq,T,D]; seq_lens int32 [B] counts the cached tokens including
    the chunk's T.  Cache arguments as for kvq_decode_attn.
    """
    B, Hq, T, D = q.shape
    if Hk is None:
        Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    if view is None:
        view = cache_view(k, v, k_scale, v_scale, page_table, page_size)
    if out is None:
        out = torch.empty(B, Hq, T, D, dtype=torch.float32, device=q.device)
    if workspace is None:               # (a given workspace's size is checked by the call)
        need = kvq_chunk_workspace_bytes(B, Hq, Hk, T, D, max_seq_len_hint, num_splits)
        if need > 0:
            workspace = new_workspace(need, q.device)
    ws_ptr = _ptr(workspace, None, "workspace") if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    check(lib.kvq_chunk_attn(
        _ptr(q, torch.bfloat16, "q"), B, Hq, Hk, T, D, _mode(mode), ctypes.byref(view),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(max_seq_len_hint), float(attn_scale),
        _ptr(out, torch.float32, "out"), ws_ptr, ws_bytes, int(num_splits),
        _ptr(err, torch.int32, "err"), _stream(stream, q)), "kvq_chunk_attn")
    return out


def kvq_chunk_workspace_bytes(B, Hq, Hk, T, D, max_seq_len_hint, num_splits=0) -> int:
    return int(lib.kvq_chunk_workspace_bytes(B, Hq, Hk, T, D, int(max_seq_len_hint),
                                             int(num_splits)))


def kvq_window_attn(q, k, v, k_scale, v_scale, seq_lens, max_seq_len_hint, window, *,
                    Hk=None, page_table=None, page_size=0, attn_scale=None, mode="per_token",
                    out=None, workspace=None, num_splits=0, err=None, stream=None,
                    view: Optional[CacheView] = None):
    """Sliding-window attention: q bf16 [B,Hq,D] (a decode step) or
    [B,Hq,T,D]; query i at position L - T + i sees the positions
    max(0, p - window + 1) .. p.  Returns fp32 of q's shape."""
    if q.dim() == 3:
        B, Hq, D = q.shape
        T = 1
    else:
        B, Hq, T, D = q.shape
    if Hk is None:
        Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    if view is None:
        view = cache_view(k, v, k_scale, v_scale, page_table, page_size)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if workspace is None:
        need = int(lib.kvq_window_workspace_bytes(B, Hq, Hk, T, D, int(max_seq_len_hint),
                                                  int(window), int(num_splits)))
        if need > 0:
            workspace = new_workspace(need, q.device)
    ws_ptr = _ptr(workspace, None, "workspace") if workspace is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    check(lib.kvq_window_attn(
        _ptr(q, torch.bfloat16, "q"), B, Hq, Hk, T, D, _mode(mode), ctypes.byref(view),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(max_seq_len_hint), int(window),
        float(attn_scale), _ptr(out, torch.float32, "out"), ws_ptr, ws_bytes, int(num_splits),
        _ptr(err, torch.int32, "err"), _stream(stream, q)), "kvq_window_attn")
    return out


def kvq_append_mixed(k_new, v_new, lens_old, k_cache, v_cache, k_scale, v_scale, k_ring,
                     v_ring, mode="per_token", err=None, stream=None):
    """Mixed cache append: k_new/v_new bf16 [B,Hk,T,D] join the bf16 window
    rings [B,Hk,W,D]; tokens leaving the window are quantised into the INT8
    part (k_cache [B,Hk,max_seq,D] and its scales).  lens_old int32 [B]."""
    B, Hk, T, D = k_new.shape
    check(lib.kvq_append_mixed(
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(v_new, torch.bfloat16, "v_new"),
        B, Hk, T, D, _mode(mode), _ptr(lens_old, torch.int32, "lens_old"),
        _ptr(k_cache, torch.uint8, "k_cache"), _ptr(v_cache, torch.uint8, "v_cache"),
        _ptr(k_scale, torch.float32, "k_scale"), _ptr(v_scale, torch.float32, "v_scale"),
        k_cache.shape[2], _ptr(k_ring, torch.bfloat16, "k_ring"),
        _ptr(v_ring, torch.bfloat16, "v_ring"), k_ring.shape[2], _ptr(err, torch.int32, "err"),
        _stream(stream, k_new)), "kvq_append_mixed")


def kvq_decode_attn_mixed(q, k, v, k_scale, v_scale, k_ring, v_ring, seq_lens, max_seq_len_hint,
                          *, mode="per_token", attn_scale=None, out=None, workspace=None,
                          num_splits=0, err=None, stream=None, page_table=None, page_size=0):
    """Decode attention over a mixed cache (INT8 part + bf16 window rings
    [B,Hk,W,D]); seq_lens counts every token.  Returns fp32 [B,Hq,D]."""
    B, Hq, D = q.shape
    Hk = k.shape[1]
    W = k_ring.shape[2]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    view = cache_view(k, v, k_scale, v_scale, page_table, page_size)
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    if workspace is None:
        need = int(lib.kvq_mixed_workspace_bytes(B, Hq, Hk, D, int(max_seq_len_hint), W,
                                                 int(num_splits)))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    check(lib.kvq_decode_attn_mixed(
        _ptr(q, torch.bfloat16, "q"), B, Hq, Hk, D, _mode(mode), ctypes.byref(view),
        _ptr(k_ring, torch.bfloat16, "k_ring"), _ptr(v_ring, torch.bfloat16, "v_ring"), W,
        _ptr(seq_lens, torch.int32, "seq_lens"), int(max_seq_len_hint), float(attn_scale),
        _ptr(out, torch.float32, "out"), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), int(num_splits),
        _ptr(err, torch.int32, "err"), _stream(stream, q)), "kvq_decode_attn_mixed")
    return out


def kvq_decode_attn_noalloc(q, k, v, k_scale, v_scale, seq_lens, max_seq_len_hint, *,
                            Hk=None, page_table=None, page_size=0, attn_scale=None,
                            mode="per_token", out=None, num_splits=0, err=None, stream=None,
                            view: Optional[CacheView] = None):
    """kvq_decode_attn without a caller workspace: the split-K scratch is the
    library's own fixed array (for callers that cannot allocate device memory;
    see include/kvq.h).  `out` must be given by callers that cannot allocate."""
    B, Hq, D = q.shape
    if Hk is None:
        Hk = k.shape[1]
    if attn_scale is None:
        attn_scale = 1.0 / math.sqrt(D)
    if view is None:
        view = cache_view(k, v, k_scale, v_scale, page_table, page_size)
    if out is None:
        out = torch.empty(B, Hq, D, dtype=torch.float32, device=q.device)
    check(lib.kvq_decode_attn_noalloc(
        _ptr(q, torch.bfloat16, "q"), B, Hq, Hk, D, _mode(mode), ctypes.byref(view),
        _ptr(seq_lens, torch.int32, "seq_lens"), int(max_seq_len_hint), float(attn_scale),
        _ptr(out, torch.float32, "out"), int(num_splits), _ptr(err, torch.int32, "err"),
        _stream(stream, q)), "kvq_decode_attn_noalloc")
    return out


def kvq_dequant(q, scale, mode="per_token", out=None, stream=None):
    """fp32 (byte - 128) * scale for q u8 [..., D], scale fp32 [..., NG]."""
    D = q.shape[-1]
    rows = q.numel() // D if D else 0
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    check(lib.kvq_dequant(_ptr(q, torch.uint8, "q"), _ptr(scale, torch.float32, "scale"),
                          rows, D, _mode(mode), _ptr(out, torch.float32, "out"),
                          _stream(stream, q)), "kvq_dequant")
    return out


def kvq_read_error(err, stream=None) -> int:
    """Synchronise, return and clear the device error bits."""
    bits = ctypes.c_int32(0)
    st = lib.kvq_read_error(_ptr(err, torch.int32, "err"), ctypes.byref(bits),
                            _stream(stream, err))
    if st not in (0, 4):
        check(st, "kvq_read_error")
    return bits.value


def kvq_cache_bytes(layers, Hk, seq, D, mode="per_token") -> int:
    return int(lib.kvq_cache_bytes(layers, Hk, seq, D, _mode(mode)))


def kvq_version() -> str:
    return lib.kvq_version().decode()


class Pager:
    """Host bookkeeping of a paged arena (kvq_pager_* in include/kvq.h): the
    free-page allocator, one page table and length per sequence, append,
    rollback (popn), release and reset, and the rollback rule of
    sliding-window layers.  The pager's memory is a host buffer this object
    owns; ``table()`` / ``lens()`` are int32 host tensors over it, to be
    copied to the device for kvq_append_paged and the attention calls."""

    def __init__(self, num_pages: int, max_seqs: int, max_pages: int, page_size: int = 16,
                 windows=()):
        wins = (ctypes.c_int32 * max(len(windows), 1))(*[int(w) for w in windows])
        nbytes = int(lib.kvq_pager_bytes(num_pages, max_seqs, max_pages, len(windows)))
        if nbytes == 0:
            raise ValueError("bad pager sizes")
        # 16-byte aligned host buffer (torch's CPU allocator aligns to 64 bytes)
        self._mem = torch.empty(nbytes, dtype=torch.uint8)
        handle = ctypes.c_void_p()
        check(lib.kvq_pager_init(self._mem.data_ptr(), nbytes, num_pages, page_size, max_seqs,
                                 max_pages, wins if windows else None, len(windows),
                                 ctypes.byref(handle)), "kvq_pager_init")
        self._h = handle
        self.num_pages, self.max_seqs, self.max_pages = num_pages, max_seqs, max_pages
        self.page_size = page_size
        tp = lib.kvq_pager_table(self._h)
        lp = lib.kvq_pager_lens(self._h)
        base = self._mem.data_ptr()
        # the table and the lengths live inside the pager's buffer
        self._table = self._mem[tp - base:tp - base + 4 * max_seqs * max_pages].view(
            torch.int32).view(max_seqs, max_pages)
        self._lens = self._mem[lp - base:lp - base + 4 * max_seqs].view(torch.int32)

    def append(self, seq: int, n: int) -> int:
        """Grow sequence seq by n tokens; returns the first write position."""
        pos = ctypes.c_int64(0)
        check(lib.kvq_pager_append(self._h, seq, n, ctypes.byref(pos)), "kvq_pager_append")
        return pos.value

    def popn(self, seq: int, n: int) -> int:
        return int(lib.kvq_pager_popn(self._h, seq, n))

    def release(self, seq: int) -> None:
        check(lib.kvq_pager_release(self._h, seq), "kvq_pager_release")

    def reset(self) -> None:
        lib.kvq_pager_reset(self._h)

    def num_free(self) -> int:
        return int(lib.kvq_pager_free_pages(self._h))

    def pages_used(self, seq: int) -> int:
        return int(lib.kvq_pager_pages_used(self._h, seq))

    def seq_len(self, seq: int) -> int:
        return int(lib.kvq_pager_seq_len(self._h, seq))

    def table(self) -> torch.Tensor:
        """int32 [max_seqs, max_pages] host view (-1 = no page)."""
        return self._table

    def lens(self) -> torch.Tensor:
        """int32 [max_seqs] host view of the lengths."""
        return self._lens

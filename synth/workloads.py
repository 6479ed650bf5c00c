"""Workload definitions and seeded generators.

The five workloads follow the decode shapes of the INT8 KV-cache pages:
a tiny GQA decode, a Llama-3-8B-shaped layer, a batched decode with
group-32 scales, a paged decode (page size 16 as in the combs-models
``kv.rs`` page, ``CacheConfig``) and a 131072-token long-context decode with
a 2048-token prefill chunk.

Reading of open points (stated once here, repeated in the design notes):
* "uniform in [a, b]" lengths are integers drawn inclusively.
* "p% channels scaled xF": ``round(p * Hk * D)`` distinct (kv-head, dim)
  pairs chosen by the seeded generator; K and V of every token in those
  channels are multiplied by F (in fp32, then rounded to bf16).
* The page table is a seeded random permutation of a shared arena of
  ``sum_b ceil(seq_len_b / 16)`` pages, handed to sequences in order and
  padded with -1.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hk: int
    D: int
    mode: str               # "per_token" | "group32" | "fp8_e4m3" | "fp8_e5m2" | "per_channel" ...
    layout: str             # "contiguous" | "paged"
    len_lo: int             # cached length before the decode append (inclusive range)
    len_hi: int
    sigma: float
    outlier_frac: float = 0.0
    outlier_factor: float = 1.0
    prefill_chunk: int = 0  # tokens per append call when building the cache
    seed: int = 0
    window: int = 0         # sliding-window attention over the last `window` positions (0: none)
    recent: int = 0         # mixed cache: the newest `recent` tokens kept bf16 (0: none)

    @property
    def G(self) -> int:
        return self.Hq // self.Hk

    @property
    def NG(self) -> int:
        """Scales per (token, kv head)."""
        return {"per_token": 1, "group32": self.D // 32}.get(self.mode, 0)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 4, 1, 64, "per_token", "contiguous", 256, 256, 1.0,
                     seed=1001),
    "llama3_8b_layer": Workload("llama3_8b_layer", 1, 32, 8, 128, "per_token", "contiguous",
                                4096, 4096, 1.0, 0.01, 10.0, seed=1002),
    "batched_group32": Workload("batched_group32", 16, 32, 8, 128, "group32", "contiguous",
                                1024, 8192, 1.0, seed=1003),
    "paged": Workload("paged", 32, 32, 8, 128, "per_token", "paged", 512, 16384, 0.5,
                      seed=1004),
    "long_context": Workload("long_context", 1, 64, 8, 128, "per_token", "contiguous",
                             131072, 131072, 1.0, 0.02, 20.0, prefill_chunk=2048, seed=1005),
}


# The same shapes and data with the other cache formats and attention forms
# (measurement lines for them; the five workloads above are the parity and
# headline cases).
EXTRA_WORKLOADS = {
    "long_context_fp8_e4m3": dataclasses.replace(WORKLOADS["long_context"],
                                                 name="long_context_fp8_e4m3", mode="fp8_e4m3"),
    "long_context_per_channel": dataclasses.replace(WORKLOADS["long_context"],
                                                    name="long_context_per_channel",
                                                    mode="per_channel"),
    "long_context_window4096": dataclasses.replace(WORKLOADS["long_context"],
                                                   name="long_context_window4096", window=4096),
    "llama3_8b_layer_mixed128": dataclasses.replace(WORKLOADS["llama3_8b_layer"],
                                                    name="llama3_8b_layer_mixed128", recent=128),
}
ALL_WORKLOADS = {**WORKLOADS, **EXTRA_WORKLOADS}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def bf16_normal(shape, sigma: float, gen: torch.Generator) -> torch.Tensor:
    """N(0, sigma^2) drawn in fp32 on the CPU and rounded to bf16."""
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(torch.bfloat16)


def lengths_uniform(B: int, lo: int, hi: int, gen: torch.Generator) -> torch.Tensor:
    """Integer lengths uniform on [lo, hi] inclusive, int32 [B]."""
    if lo == hi:
        return torch.full((B,), lo, dtype=torch.int32)
    return torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)


def outlier_channels(Hk: int, D: int, frac: float, gen: torch.Generator) -> torch.Tensor:
    """round(frac*Hk*D) distinct flat (kv_head*D + dim) channel ids, int64."""
    n = int(round(frac * Hk * D))
    if n <= 0:
        return torch.zeros(0, dtype=torch.int64)
    return torch.randperm(Hk * D, generator=gen)[:n].sort().values


def apply_outliers(x_bf16: torch.Tensor, channels: torch.Tensor, factor: float) -> torch.Tensor:
    """Multiply the listed (kv_head, dim) channels of x [..., Hk, T, D] by factor."""
    if channels.numel() == 0:
        return x_bf16
    Hk, D = x_bf16.shape[-3], x_bf16.shape[-1]
    x = x_bf16.float()
    h = channels // D
    d = channels % D
    x[..., h, :, d] *= factor
    return x.to(torch.bfloat16)


def num_pages_for(seq_len: int, page_size: int = 16) -> int:
    return (int(seq_len) + page_size - 1) // page_size


def page_table_for(seq_lens, page_size: int, gen: torch.Generator,
                   max_pages: Optional[int] = None, extra_pages: int = 0):
    """Random-permutation page table over a shared arena.

    Returns (table int32 [B, max_pages] padded with -1, num_pages).
    """
    seq_lens = [int(s) for s in seq_lens]
    need = [num_pages_for(s, page_size) for s in seq_lens]
    total = sum(need) + int(extra_pages)
    if max_pages is None:
        max_pages = max(need) if need else 1
    max_pages = max(int(max_pages), 1)
    perm = torch.randperm(max(total, 1), generator=gen).to(torch.int32)
    table = torch.full((len(seq_lens), max_pages), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, max(total, 1)


@dataclasses.dataclass
class DecodeInputs:
    """Everything one decode step of a workload needs, on the CPU.

    k_hist/v_hist: bf16 [B, Hk, Lmax, D] history tokens (token t of sequence b
    is valid for t < cached[b]); k_new/v_new: bf16 [B, Hk, 1, D]; q: bf16
    [B, Hq, D]; cached: int32 [B] lengths before the append; seq_lens =
    cached + 1.
    """
    wl: Workload
    k_hist: torch.Tensor
    v_hist: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    q: torch.Tensor
    cached: torch.Tensor
    seq_lens: torch.Tensor
    page_table: Optional[torch.Tensor] = None
    num_pages: int = 0


def make_decode_inputs(wl: Workload, *, B: Optional[int] = None, len_lo: Optional[int] = None,
                       len_hi: Optional[int] = None, seed: Optional[int] = None,
                       page_size: int = 16, qlen: int = 1) -> DecodeInputs:
    """Seeded decode-step inputs for a workload (optionally shrunk).  qlen > 1:
    a chunk of qlen new tokens (k_new/v_new [B, Hk, qlen, D]) and qlen queries
    per head (q [B, Hq, qlen, D]); qlen = 1 draws exactly the decode inputs."""
    B = wl.B if B is None else B
    lo = wl.len_lo if len_lo is None else len_lo
    hi = wl.len_hi if len_hi is None else len_hi
    g = _gen(wl.seed if seed is None else seed)
    cached = lengths_uniform(B, lo, hi, g)
    Lmax = int(cached.max().item()) if B > 0 else 0
    chans = outlier_channels(wl.Hk, wl.D, wl.outlier_frac, g)
    k_hist = apply_outliers(bf16_normal((B, wl.Hk, Lmax, wl.D), wl.sigma, g), chans, wl.outlier_factor)
    v_hist = apply_outliers(bf16_normal((B, wl.Hk, Lmax, wl.D), wl.sigma, g), chans, wl.outlier_factor)
    k_new = apply_outliers(bf16_normal((B, wl.Hk, qlen, wl.D), wl.sigma, g), chans, wl.outlier_factor)
    v_new = apply_outliers(bf16_normal((B, wl.Hk, qlen, wl.D), wl.sigma, g), chans, wl.outlier_factor)
    q = bf16_normal((B, wl.Hq, wl.D) if qlen == 1 else (B, wl.Hq, qlen, wl.D), 1.0, g)
    seq_lens = (cached + qlen).to(torch.int32)
    table, npages = (None, 0)
    if wl.layout == "paged":
        table, npages = page_table_for(seq_lens.tolist(), page_size, g)
    return DecodeInputs(wl, k_hist, v_hist, k_new, v_new, q, cached, seq_lens, table, npages)

#!/usr/bin/env python
"""Benchmark of the INT8 KV-cache decode hot path on B200.

One step = one pass of the whole hot path over one batch: for every layer of
the workload, quantise-on-append the new token's K/V into the INT8 cache
(kvq_append / kvq_append_paged), then decode attention on the INT8 cache
(kvq_decode_attn: split kernel + combine).  The default workload is one
Llama-3-8B-shaped decode (B=1, Hq=32, Hk=8, D=128, 4096 cached tokens + 1)
repeated over 32 independent layer caches (277 MB, larger than the 126 MB L2,
so consecutive reads of a layer never hit in L2).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
        [--workload llama3_8b_layer|tiny|batched_group32|paged|long_context] [--qlen T]
--qlen T > 1 times chunk steps instead: every layer appends a chunk of T new
tokens and runs kvq_chunk_attn with T queries per head (causal from the
chunk's end).
Multi-GPU: launched by torch.distributed.run, one rank per GPU; every rank
runs its own replica of the workload (weak scaling, no data-path collective);
the job time is the max over ranks.

The line's headline fields time exactly K steps of the chosen workload.
Its "per_config" object then times every workload on its own (median over
at least 10 repeats, enough of them to span a quarter of a second), each
with its roofline, append rate, end-to-end rate and clock record.  The CPU
baseline is the oracle on this host: all cores (OpenMP over independent
(sequence, kv head) units) and one core.

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "decode-attn INT8-KV GB/s & fraction of HBM peak; tokens/s per layer; append GB/s"
DEFAULT_WORKLOAD = "llama3_8b_layer"
QLEN = 1                                  # queries per (sequence, q head) per step (--qlen)
LAYERS = {"llama3_8b_layer": 32}


# ------------------------------------------------------------------ helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _ng(wl):
    """Scales per (token, kv head) of the workload's cache format."""
    return {"per_token": 1, "group32": wl.D // 32}.get(wl.mode, 0)


def _static_ns(wl):
    """Scales per (sequence, kv head): per-head 1, per-channel D, else 0."""
    return {"per_head": 1, "per_channel": wl.D}.get(wl.mode, 0)


def measured_tensor_peak():
    """Dense bf16 TFLOP/s on this machine's B200s (burst), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def chunk_flops(wl, seq_lens, T):
    """Useful flops of one chunk-attention call: every (query, head) row times
    the keys it sees (L - T + i + 1 for query i), 2 D for Q.K^T and 2 D for P.V."""
    pairs = sum(T * (L - T) + T * (T + 1) // 2 for L in seq_lens)
    return pairs * wl.Hq * wl.D * 2 * 2


def decode_bytes(wl, seq_lens, page_size=0):
    """Algorithmic bytes of one decode call: the attended K/V bytes + their
    scales (per token, or per (sequence, kv head)), the bf16 window of a mixed
    cache, Q, output, page-table entries."""
    ng = _ng(wl)
    kv = 0
    for L in seq_lens:
        n8 = L
        if wl.window:
            n8 = min(L, wl.window + QLEN - 1)
        if wl.recent:
            n8 = max(L - wl.recent, 0)
            kv += wl.Hk * (L - n8) * 2 * wl.D * 2           # bf16 window
        kv += wl.Hk * n8 * (2 * wl.D + 2 * 4 * ng) + wl.Hk * 2 * 4 * _static_ns(wl)
    qo = wl.B * wl.Hq * wl.D * (2 + 4) * QLEN
    pt = sum((L + 15) // 16 * 4 for L in seq_lens) if page_size else 0
    return kv + qo + pt


def append_bytes(wl, T):
    ng = _ng(wl)
    rd = T * wl.B * wl.Hk * wl.D * 2 * 2
    wr = T * wl.B * wl.Hk * (2 * wl.D + 2 * 4 * ng)
    if wl.recent:                  # the token leaving the window is read back, the new one written
        rd += T * wl.B * wl.Hk * wl.D * 2 * 2
        wr += T * wl.B * wl.Hk * wl.D * 2 * 2
    return rd + wr


class ClockSampler:
    """Samples SM clock, power and throttle reasons through NVML (the library
    nvidia-smi reads) in a background thread while the timed region runs."""

    HW_SLOW = 0x8
    HW_THERMAL = 0x40
    SW_THERMAL = 0x20
    SW_POWER = 0x4

    def __init__(self, device_index: int, period_s: float = 0.002, enabled: bool = True):
        self.samples = []
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        if not enabled:
            return
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = str(e)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((mhz, reasons))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        if self._thread:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"]}
        mhz = statistics.median(s[0] for s in self.samples)
        bits = 0
        for _, r in self.samples:
            bits |= r
        names = []
        for bit, name in [(self.HW_SLOW, "hw_slowdown"), (self.HW_THERMAL, "hw_thermal_slowdown"),
                          (self.SW_THERMAL, "sw_thermal_slowdown"),
                          (self.SW_POWER, "sw_power_cap")]:
            if bits & bit:
                names.append(name)
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


def physical_gpu_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if local < len(parts) and parts[local].isdigit():
            return int(parts[local])
    return local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def decode_traffic_record():
    """DRAM bytes per decode launch from a committed ncu summary, valid only if
    the decode kernel source still has the hash recorded with it."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("decode_sources_sha256") != decode_sources_hash():
        return None
    return rec


def decode_sources_hash():
    """sha256 over the decode kernels' sources (split kernel, combine, PTX helpers)."""
    h = hashlib.sha256()
    for name in ("kvq_decode_tc.cu", "kvq_decode.cu", "kvq_ptx.cuh", "kvq_internal.cuh"):
        with open(os.path.join(ROOT, "decode_attention_kvq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# ---------------------------------------------------------------- workload
class Layer:
    """One layer's KV cache on the GPU with its decode-step inputs: INT8 with
    per-token / group-32 / per-channel scales, or FP8; contiguous or paged;
    optionally a mixed cache (bf16 window ring) or sliding-window attention."""

    def __init__(self, kvq, wl, inp, dev, keep_host=False):
        self.wl = wl
        B, Hk, D = wl.B, wl.Hk, wl.D
        ng = _ng(wl)
        ns = _static_ns(wl)
        self.paged = wl.layout == "paged"
        cached = inp.cached
        self.seq_lens_list = [int(x) for x in inp.seq_lens]
        self.hint = max(self.seq_lens_list)

        def scales(lead):
            if ns:                      # per (sequence, kv head)
                return torch.zeros(B, Hk, ns, device=dev)
            if ng == 0:                 # FP8: none
                return None
            return torch.zeros(*lead, ng, device=dev)

        if self.paged:
            shape = (inp.num_pages, Hk, 16, D)
            self.table = inp.page_table.to(dev)
            self.k = torch.zeros(shape, dtype=torch.uint8, device=dev)
            self.v = torch.zeros_like(self.k)
            self.ks, self.vs = scales((inp.num_pages, Hk, 16)), scales((inp.num_pages, Hk, 16))
            for b in range(B):
                L = int(cached[b])
                kv_k = inp.k_hist[b:b + 1, :, :L].contiguous().to(dev)
                kv_v = inp.v_hist[b:b + 1, :, :L].contiguous().to(dev)
                kvq.kvq_append_paged(kv_k, kv_v, torch.zeros(1, dtype=torch.int32, device=dev),
                                     self.k, self.v, self.ks, self.vs,
                                     self.table[b:b + 1].contiguous(), 16, wl.mode)
        else:
            S = self.hint
            self.table = None
            self.k = torch.zeros(B, Hk, S, D, dtype=torch.uint8, device=dev)
            self.v = torch.zeros_like(self.k)
            self.ks, self.vs = scales((B, Hk, S)), scales((B, Hk, S))
            Lmax = int(cached.max())
            if wl.recent:               # mixed cache: the history through the window
                self.rk = torch.zeros(B, Hk, wl.recent, D, dtype=torch.bfloat16, device=dev)
                self.rv = torch.zeros_like(self.rk)
                lens = torch.zeros(B, dtype=torch.int32, device=dev)
                for p0 in range(0, Lmax, 8192):
                    T = min(8192, Lmax - p0)
                    kvq.kvq_append_mixed(inp.k_hist[:, :, p0:p0 + T].contiguous().to(dev),
                                         inp.v_hist[:, :, p0:p0 + T].contiguous().to(dev),
                                         lens, self.k, self.v, self.ks, self.vs, self.rk,
                                         self.rv, wl.mode)
                    lens += T
            else:
                chunk = 8192
                for p0 in range(0, Lmax, chunk):
                    T = min(chunk, Lmax - p0)
                    args = (inp.k_hist[:, :, p0:p0 + T].contiguous().to(dev),
                            inp.v_hist[:, :, p0:p0 + T].contiguous().to(dev),
                            torch.full((B,), p0, dtype=torch.int32, device=dev),
                            self.k, self.v, self.ks, self.vs, wl.mode)
                    if ns and p0 == 0:  # per-channel: the first chunk sets the scales
                        kvq.kvq_append_calibrate(*args)
                    else:
                        kvq.kvq_append(*args)
        self.k_new = inp.k_new.to(dev)
        self.v_new = inp.v_new.to(dev)
        self.q = inp.q.to(dev)
        self.pos = cached.to(dev)
        self.seq_lens = inp.seq_lens.to(dev)
        self.qlen = QLEN
        self.out = torch.empty((B, wl.Hq, D) if QLEN == 1 else (B, wl.Hq, QLEN, D), device=dev)
        self.view = kvq.cache_view(self.k, self.v, self.ks, self.vs, self.table,
                                   16 if self.paged else 0)
        if keep_host:
            self.host = inp
        # prefill chunk re-append (long-context workload): rewrite the last chunk
        # (a chunk step's own tokens are the chunk: no separate re-append then)
        self.chunk_T = wl.prefill_chunk if (not wl.recent and QLEN == 1) else 0
        if self.chunk_T:
            p0 = int(cached[0]) - self.chunk_T
            self.chunk_k = inp.k_hist[:, :, p0:p0 + self.chunk_T].contiguous().to(dev)
            self.chunk_v = inp.v_hist[:, :, p0:p0 + self.chunk_T].contiguous().to(dev)
            self.chunk_pos = torch.full((B,), p0, dtype=torch.int32, device=dev)

    def workspace_bytes(self, kvq):
        wl, hint = self.wl, self.hint
        if wl.recent:
            return int(kvq.lib.kvq_mixed_workspace_bytes(wl.B, wl.Hq, wl.Hk, wl.D, hint,
                                                         wl.recent, 0))
        if wl.window:
            return int(kvq.lib.kvq_window_workspace_bytes(wl.B, wl.Hq, wl.Hk, QLEN, wl.D, hint,
                                                          wl.window, 0))
        if QLEN == 1:
            return kvq.kvq_decode_workspace_bytes(wl.B, wl.Hq, wl.Hk, wl.D, hint)
        return kvq.kvq_chunk_workspace_bytes(wl.B, wl.Hq, wl.Hk, QLEN, wl.D, hint)

    def append(self, kvq, k_new=None, v_new=None, stream=None):
        k_new = self.k_new if k_new is None else k_new
        v_new = self.v_new if v_new is None else v_new
        if self.wl.recent:
            # the step's token joins the window; the one leaving it is quantised
            kvq.kvq_append_mixed(k_new, v_new, self.pos, self.k, self.v, self.ks, self.vs,
                                 self.rk, self.rv, self.wl.mode, stream=stream)
            return
        if self.chunk_T:
            kvq.kvq_append(self.chunk_k, self.chunk_v, self.chunk_pos, self.k, self.v, self.ks,
                           self.vs, self.wl.mode, stream=stream)
        if self.paged:
            kvq.kvq_append_paged(k_new, v_new, self.pos, self.k, self.v, self.ks,
                                 self.vs, self.table, 16, self.wl.mode, stream=stream)
        else:
            kvq.kvq_append(k_new, v_new, self.pos, self.k, self.v, self.ks, self.vs,
                           self.wl.mode, stream=stream)

    @property
    def fusable(self):
        """The step can run as one kvq_append_decode call (INT8 per-token or
        group-32 decode without a window or a bf16 recent window)."""
        wl = self.wl
        return (self.qlen == 1 and not wl.window and not wl.recent and
                wl.mode in ("per_token", "group32"))

    def step_fused(self, kvq, workspace, k_new=None, v_new=None, q=None, out=None, stream=None):
        """The decode step through the one-call entry point: the new token is
        quantised inside the decode kernel (the prefill-chunk re-append of the
        long-context workload stays its own call)."""
        k_new = self.k_new if k_new is None else k_new
        v_new = self.v_new if v_new is None else v_new
        q = self.q if q is None else q
        out = self.out if out is None else out
        if self.chunk_T:
            kvq.kvq_append(self.chunk_k, self.chunk_v, self.chunk_pos, self.k, self.v, self.ks,
                           self.vs, self.wl.mode, stream=stream)
        kvq.kvq_append_decode(q, k_new, v_new, self.k, self.v, self.ks, self.vs, self.seq_lens,
                              self.hint, page_table=self.table,
                              page_size=16 if self.paged else 0, view=self.view,
                              mode=self.wl.mode, out=out, workspace=workspace, stream=stream)

    def decode(self, kvq, workspace, q=None, out=None, stream=None):
        q = self.q if q is None else q
        out = self.out if out is None else out
        wl = self.wl
        common = dict(mode=wl.mode, out=out, workspace=workspace, stream=stream)
        if wl.recent:
            kvq.kvq_decode_attn_mixed(q, self.k, self.v, self.ks, self.vs, self.rk, self.rv,
                                      self.seq_lens, self.hint, **common)
        elif wl.window:
            kvq.kvq_window_attn(q, self.k, self.v, self.ks, self.vs, self.seq_lens, self.hint,
                                wl.window, page_table=self.table,
                                page_size=16 if self.paged else 0, view=self.view, **common)
        else:
            call = kvq.kvq_decode_attn if self.qlen == 1 else kvq.kvq_chunk_attn
            call(q, self.k, self.v, self.ks, self.vs, self.seq_lens, self.hint,
                 page_table=self.table, page_size=16 if self.paged else 0, view=self.view,
                 **common)


def build_layers(kvq, wl, n_layers, dev, keep_host=False):
    layers = []
    for i in range(n_layers):
        inp = synth.make_decode_inputs(wl, seed=wl.seed + 7919 * i, qlen=QLEN)
        layers.append(Layer(kvq, wl, inp, dev, keep_host=keep_host and i == 0))
        del inp
    torch.cuda.synchronize(dev)
    return layers


# -------------------------------------------------------------- cpu oracle
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


class OracleLayer:
    """One layer of the workload held by the CPU oracle: the history is
    quantised once at set-up; a step quantises the decode token into the
    cache and runs fp64 decode attention, either single-threaded (the pinned
    oracle as it stands) or as one pinned-oracle call per (sequence, kv head)
    on `threads` host threads (the oracle's all-core baseline build)."""

    def __init__(self, wl, seed):
        import oracle  # test infrastructure: used only by the CPU baseline legs
        self.oracle = oracle
        self.wl = wl
        inp = synth.make_decode_inputs(wl, seed=seed, qlen=QLEN)
        self.inp = inp
        B, Hk, D = wl.B, wl.Hk, wl.D
        ng = 1 if wl.mode == "per_token" else D // 32
        self.paged = wl.layout == "paged"
        z1 = torch.zeros(1, dtype=torch.int32)
        if self.paged:
            shape = (inp.num_pages, Hk, 16, D)
            self.k = torch.zeros(shape, dtype=torch.uint8)
            self.v = torch.zeros_like(self.k)
            self.ks = torch.zeros(inp.num_pages, Hk, 16, ng)
            self.vs = torch.zeros_like(self.ks)
            for b in range(B):
                L = int(inp.cached[b])
                tb = inp.page_table[b:b + 1].contiguous()
                oracle.append_paged(inp.k_hist[b:b + 1, :, :L].contiguous(), z1, self.k, self.ks,
                                    tb, 16, wl.mode)
                oracle.append_paged(inp.v_hist[b:b + 1, :, :L].contiguous(), z1, self.v, self.vs,
                                    tb, 16, wl.mode)
            self.utables = oracle.unit_tables(inp.page_table, Hk, inp.num_pages)
        else:
            S = int(inp.seq_lens.max())
            self.k = torch.zeros(B, Hk, S, D, dtype=torch.uint8)
            self.v = torch.zeros_like(self.k)
            self.ks = torch.zeros(B, Hk, S, ng)
            self.vs = torch.zeros_like(self.ks)
            Lm = int(inp.cached.max())
            zb = torch.zeros(B, dtype=torch.int32)
            oracle.append_contig(inp.k_hist[:, :, :Lm].contiguous(), zb, self.k, self.ks, wl.mode)
            oracle.append_contig(inp.v_hist[:, :, :Lm].contiguous(), zb, self.v, self.vs, wl.mode)
            self.utables = None
        self.scale = float(torch.tensor(1.0 / math.sqrt(D), dtype=torch.float32))
        self.nbytes = decode_bytes(wl, [int(x) for x in inp.seq_lens], 16 if self.paged else 0)
        self.inp.k_hist = self.inp.v_hist = None

    def step(self, threads: int = 1) -> float:
        o, wl, inp = self.oracle, self.wl, self.inp
        t0 = time.perf_counter()
        if self.paged:
            o.append_paged(inp.k_new, inp.cached, self.k, self.ks, inp.page_table, 16, wl.mode)
            o.append_paged(inp.v_new, inp.cached, self.v, self.vs, inp.page_table, 16, wl.mode)
        else:
            o.append_contig(inp.k_new, inp.cached, self.k, self.ks, wl.mode)
            o.append_contig(inp.v_new, inp.cached, self.v, self.vs, wl.mode)
        if threads <= 1:
            attn = o.decode_attn if QLEN == 1 else o.chunk_attn
            if self.paged:
                attn(inp.q, self.k, self.v, self.ks, self.vs, inp.seq_lens, self.scale, wl.mode,
                     page_size=16, table=inp.page_table)
            else:
                attn(inp.q, self.k, self.v, self.ks, self.vs, inp.seq_lens, self.scale, wl.mode)
        else:
            o.attn_units(inp.q, self.k, self.v, self.ks, self.vs, inp.seq_lens, self.scale,
                         wl.mode, page_size=16 if self.paged else 0, utables=self.utables,
                         num_pages=inp.num_pages, threads=threads)
        return time.perf_counter() - t0


def oracle_sample(wl, n_steps_max, budget_s, threads=1, n_distinct=4):
    """Time the oracle on a bounded sample of the workload: layer steps cycled
    over a few distinct layers until the time budget or the step cap is hit.
    Returns (GB/s, sample description)."""
    layers = [OracleLayer(wl, wl.seed + 7919 * i) for i in range(n_distinct)]
    done, elapsed, nbytes = 0, 0.0, 0
    while done < n_steps_max and (elapsed < budget_s or done == 0):
        ly = layers[done % n_distinct]
        elapsed += ly.step(threads)
        nbytes += ly.nbytes
        done += 1
    how = ("single-threaded C oracle" if threads <= 1 else
           f"C oracle, one call per (sequence, kv head) unit on {threads} OpenMP threads")
    desc = (f"{done} layer steps of {wl.name} (append {QLEN} token(s) + fp64 attention) "
            f"over {n_distinct} distinct layers, {how}, {elapsed:.2f} s timed")
    return nbytes / elapsed / 1e9, desc


def cpu_baseline(wl, args):
    """The oracle timed on this host: all cores (OpenMP over independent
    (sequence, kv head) units, the headline value) and one core."""
    threads = os.cpu_count() or 1
    gbs_all, desc_all = oracle_sample(wl, args.cpu_layers, args.cpu_budget_s, threads=threads)
    gbs_one, desc_one = oracle_sample(wl, args.cpu_layers, args.cpu_budget_s, threads=1)
    return {"value": round(gbs_all, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": desc_all, "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "single_thread": {"value": round(gbs_one, 4), "unit": "GB/s", "cores": 1,
                              "sample": desc_one}}


# ------------------------------------------------------------------- arms
def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    # each step is a bounded sample of the workload: one layer step of the
    # oracle, on all host cores, on a layer prepared once
    threads = os.cpu_count() or 1
    ly = OracleLayer(wl, wl.seed)
    per_step = []
    for i in range(args.warmup + args.steps):
        el = ly.step(threads)
        if i >= args.warmup:
            per_step.append((ly.nbytes / el / 1e9, el))
    desc = (f"1 layer step of {wl.name} per step (append {QLEN} token(s) + fp64 attention), "
            f"C oracle, one call per (sequence, kv head) unit on {threads} OpenMP threads")
    value = statistics.median(g for g, _ in per_step)
    ms = 1000.0 * statistics.median(e for _, e in per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hk": wl.Hk, "D": wl.D,
                   "seq_len": wl.len_hi + QLEN, "scale_mode": wl.mode, "layout": wl.layout,
                   "q_len": QLEN, "sample": "1 layer step per step"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": desc, "cpu_model": cpu_model(),
                         "host_cpus": os.cpu_count()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


NOMINAL_HBM_GBS = 8000.0                  # B200 HBM3e, nominal


class GpuWorkload:
    """One workload resident on the GPU: its layer caches, the decode
    workspace and the step's two phases captured as CUDA graphs (every
    layer's append, then every layer's decode attention)."""

    def __init__(self, kvq, wl, dev, n_layers):
        self.kvq, self.wl, self.dev = kvq, wl, dev
        self.layers = build_layers(kvq, wl, n_layers, dev)
        self.n_layers = n_layers
        L0 = self.layers[0]
        self.hint = L0.hint
        ws_bytes = L0.workspace_bytes(kvq)
        self.workspace = kvq.new_workspace(max(ws_bytes, 16), dev)
        self.chunk, self.splits = kvq.kvq_decode_plan(wl.B, wl.Hk, L0.hint)
        # append (+ prefill-chunk append) + split kernel (+ combine kernel when a
        # sequence spans several chunks: then the call has a workspace)
        self.launches_per_layer = ((1 + (1 if L0.chunk_T else 0)) + 1 +
                                   (1 if ws_bytes > 0 else 0))
        self.stream = torch.cuda.Stream(dev)
        with torch.cuda.stream(self.stream):       # warm the library once eagerly
            for ly in self.layers:
                ly.append(kvq)
                ly.decode(kvq, self.workspace)
        torch.cuda.synchronize(dev)
        self.g_append, self.g_decode = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_append, stream=self.stream):
            for ly in self.layers:
                ly.append(kvq)
        with torch.cuda.graph(self.g_decode, stream=self.stream):
            for ly in self.layers:
                ly.decode(kvq, self.workspace)
        # the same step through the one-call entry point, where it applies
        self.g_fused = None
        if L0.fusable:
            with torch.cuda.stream(self.stream):
                for ly in self.layers:
                    ly.step_fused(kvq, self.workspace)
            torch.cuda.synchronize(dev)
            self.g_fused = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_fused, stream=self.stream):
                for ly in self.layers:
                    ly.step_fused(kvq, self.workspace)
        torch.cuda.synchronize(dev)
        self.dec_b = sum(decode_bytes(wl, ly.seq_lens_list, 16 if ly.paged else 0)
                         for ly in self.layers)
        self.app_b = n_layers * (append_bytes(wl, QLEN) +
                                 (append_bytes(wl, L0.chunk_T) if L0.chunk_T else 0))

    def warm(self, W):
        with torch.cuda.stream(self.stream):
            for _ in range(W):
                self.g_append.replay()
                self.g_decode.replay()
        torch.cuda.synchronize(self.dev)

    def timed(self, reps, sampler):
        """reps steps, each bracketed by CUDA events on the launching stream:
        returns per-step (append s, decode s) and the whole region's seconds."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
        with sampler:
            with torch.cuda.stream(self.stream):
                for i in range(reps):
                    ev[i][0].record(self.stream)
                    self.g_append.replay()
                    ev[i][1].record(self.stream)
                    self.g_decode.replay()
                    ev[i][2].record(self.stream)
            torch.cuda.synchronize(self.dev)
        per = [(e[0].elapsed_time(e[1]) / 1e3, e[1].elapsed_time(e[2]) / 1e3) for e in ev]
        return per, ev[0][0].elapsed_time(ev[-1][2]) / 1e3

    def timed_fused(self, reps, sampler):
        """reps one-call steps (g_fused), each bracketed by CUDA events on the
        launching stream: per-step seconds."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        with torch.cuda.stream(self.stream):
            for _ in range(3):
                self.g_fused.replay()
        with sampler:
            with torch.cuda.stream(self.stream):
                for i in range(reps):
                    ev[i][0].record(self.stream)
                    self.g_fused.replay()
                    ev[i][1].record(self.stream)
            torch.cuda.synchronize(self.dev)
        return [e[0].elapsed_time(e[1]) / 1e3 for e in ev]

    def fused_entry(self, reps, world, dev):
        """The one-call step: per-layer time, tokens/s per layer and the bytes it
        moves (decode + append) against the HBM roofline; median over reps."""
        if self.g_fused is None:
            return None
        sampler = ClockSampler(physical_gpu_index(dev.index))
        per = self.timed_fused(reps, sampler)
        t = reduce_max(statistics.median(per), dev)
        pl = t / self.n_layers
        moved = (self.dec_b + self.app_b) / self.n_layers
        achieved = moved / pl / 1e9
        peak, _ = measured_peaks()
        return {"call": "kvq_append_decode (new token quantised inside the decode kernel)",
                "repeats": reps, "statistic": "median over repeats",
                "us_per_layer": round(pl * 1e6, 3),
                "tokens_per_s_per_layer": round(world * self.wl.B * QLEN / pl, 1),
                "bytes_per_layer": int(moved), "gbs": round(world * achieved, 2),
                "frac": round(achieved / peak, 4), "clocks": sampler.summary()}

    def close(self):
        del self.g_append, self.g_decode, self.g_fused
        self.layers = None
        self.workspace = None
        torch.cuda.synchronize(self.dev)
        torch.cuda.empty_cache()


def roofline(wl, achieved):
    peak, peak_kind = measured_peaks()
    traffic = decode_traffic_record()
    tv = None
    if traffic:
        tv = (traffic.get("workloads", {}).get(wl.name, {}) or {}).get("traffic_bytes_per_launch")
    return {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": tv,
            "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
            "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
            "nominal_peak": NOMINAL_HBM_GBS}


def per_config_entry(kvq, wl, dev, K, W, world, gw=None):
    """One workload measured on its own: median over repeats (at least 10,
    and enough to cover a quarter of a second so the clock sampler sees the
    region), each repeat one step of every layer."""
    n_layers = LAYERS.get(wl.name, 1)
    own = gw is None
    if own:
        gw = GpuWorkload(kvq, wl, dev, n_layers)
    gw.warm(W)
    probe, t_probe = gw.timed(3, ClockSampler(-1, enabled=False))
    reps = max(10, K, min(2000, int(math.ceil(0.25 / max(t_probe / 3, 1e-6)))))
    barrier(dev)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(physical_gpu_index(dev.index))
    per, _ = gw.timed(reps, sampler)
    barrier(dev)
    t_app = statistics.median(a for a, _ in per)
    t_dec = statistics.median(d for _, d in per)
    t_app = reduce_max(t_app, dev)
    t_dec = reduce_max(t_dec, dev)
    dec_mean = sum(d for _, d in per) / reps
    pl_dec = t_dec / gw.n_layers
    pl_app = t_app / gw.n_layers
    achieved = gw.dec_b / gw.n_layers / pl_dec / 1e9
    e2e = run_e2e(kvq, wl, gw.layers, gw.workspace, dev, min(K, 20), W, world)
    fused = gw.fused_entry(reps, world, dev)
    entry = {
        "config": {"B": wl.B, "Hq": wl.Hq, "Hk": wl.Hk, "D": wl.D, "seq_len": gw.hint,
                   "scale_mode": wl.mode, "layout": wl.layout, "layers_per_step": gw.n_layers,
                   "split_chunk": gw.chunk, "splits": gw.splits,
                   "prefill_chunk": wl.prefill_chunk,
                   "l2": ("inputs larger than L2 (%.0f MB per step)" % ((gw.dec_b + gw.app_b) / 1e6)
                          if gw.dec_b + gw.app_b > 126e6 else
                          "inputs L2-resident (%.2f MB per step): a latency figure"
                          % ((gw.dec_b + gw.app_b) / 1e6))},
        "repeats": reps, "statistic": "median over repeats",
        "decode_us_per_layer": round(pl_dec * 1e6, 3),
        "decode_us_per_layer_mean": round(dec_mean / gw.n_layers * 1e6, 3),
        "decode_us_per_layer_min": round(min(d for _, d in per) / gw.n_layers * 1e6, 3),
        "append_us_per_layer": round(pl_app * 1e6, 3),
        "decode_gbs": round(world * achieved, 2),
        "roofline": roofline(wl, achieved),
        "append_gbs": round(world * gw.app_b / t_app / 1e9, 2),
        "tokens_per_s_per_layer": round(world * wl.B * QLEN /
                                        min(pl_app + pl_dec,
                                            fused["us_per_layer"] * 1e-6 if fused else 1e9), 1),
        "tokens_per_s_per_layer_two_calls": round(world * wl.B * QLEN / (pl_app + pl_dec), 1),
        "algorithmic_bytes_per_decode_call": int(gw.dec_b / gw.n_layers),
        "fused_step": fused,
        "e2e": e2e,
        "clocks": sampler.summary(),
    }
    if own:
        gw.close()
    return entry


def prefill_entry(kvq, wl, dev, K, W, world, T):
    """A prefill step of the workload's shape: append a T-token chunk per
    (sequence, kv head), then T queries per head attend causally (the dense
    chunk kernel when (Hq / Hk) * T > 16).  Tensor-bound: useful flops over the
    measured bf16 peak; median over repeats."""
    global QLEN
    saved = QLEN
    QLEN = T
    try:
        gw = GpuWorkload(kvq, wl, dev, 1)
        gw.warm(max(W, 3))
        _, t_probe = gw.timed(2, ClockSampler(-1, enabled=False))
        reps = max(10, min(200, int(math.ceil(0.25 / max(t_probe / 2, 1e-6)))))
        sampler = ClockSampler(physical_gpu_index(dev.index))
        per, _ = gw.timed(reps, sampler)
        t_app = reduce_max(statistics.median(a for a, _ in per), dev)
        t_att = reduce_max(statistics.median(d for _, d in per), dev)
        L0 = gw.layers[0]
        flops = chunk_flops(wl, L0.seq_lens_list, T)
        peak, kind = measured_tensor_peak()
        achieved = flops / t_att / 1e12
        entry = {
            "config": {"B": wl.B, "Hq": wl.Hq, "Hk": wl.Hk, "D": wl.D, "q_len": T,
                       "seq_len": L0.hint, "scale_mode": wl.mode, "layout": wl.layout},
            "repeats": reps, "statistic": "median over repeats",
            "attention_ms": round(t_att * 1e3, 4), "append_us": round(t_app * 1e6, 3),
            "append_gbs": round(world * append_bytes(wl, T) / t_app / 1e9, 2),
            "tokens_per_s": round(world * wl.B * T / (t_app + t_att), 1),
            "useful_flops": int(flops),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                         "peak_source": f"{kind} dense bf16 (MEASURED_PEAKS.json bf16_tflops)",
                         "kernel_ceiling_frac": round(2 / 3, 4)},
            "clocks": sampler.summary(),
        }
        gw.close()
        return entry
    finally:
        QLEN = saved


def run_kvq(args, wl):
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    import decode_attention_kvq_b200 as kvq  # fails loudly if libkvq.so is missing

    n_layers = args.layers or LAYERS.get(wl.name, 1)
    gw = GpuWorkload(kvq, wl, dev, n_layers)

    # ---- the headline: exactly K steps after W warm-up steps
    K, W = args.steps, args.warmup
    gw.warm(W)
    barrier(dev)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(physical_gpu_index(local))
    per, t_total = gw.timed(K, sampler)
    barrier(dev)
    t_append = sum(a for a, _ in per)
    t_decode = sum(d for _, d in per)
    t_total_max = reduce_max(t_total, dev)
    t_decode_max = reduce_max(t_decode, dev)
    t_append_max = reduce_max(t_append, dev)

    value = world * gw.dec_b * K / t_decode_max / 1e9
    per_layer_decode = t_decode_max / (K * n_layers)
    per_layer_append = t_append_max / (K * n_layers)
    tokens_per_s_per_layer = wl.B * QLEN / (per_layer_append + per_layer_decode)
    append_gbs = gw.app_b * K / t_append_max / 1e9
    decode_call_bytes = gw.dec_b / n_layers
    achieved = decode_call_bytes / per_layer_decode / 1e9
    rl = roofline(wl, achieved)
    rl["kernel"] = "kvq_decode_attn call (split + combine kernels, per layer)"
    rl["algorithmic_bytes_per_launch"] = int(decode_call_bytes)

    # ---- end to end through the public API from pinned host buffers
    e2e = run_e2e(kvq, wl, gw.layers, gw.workspace, dev, K, W, world)
    # ---- the same step as one call per layer (new token quantised inside the
    # decode kernel), K more steps
    fused = gw.fused_entry(max(K, 10), world, dev)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(1e3 * t_total_max / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
        "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hk": wl.Hk, "D": wl.D,
                   "seq_len": gw.hint, "q_len": QLEN, "scale_mode": wl.mode,
                   "layout": wl.layout,
                   "layers_per_step": n_layers, "parallelism": f"replicas x{world}",
                   "l2": ("inputs larger than L2 (%.0f MB per step)"
                          % ((gw.dec_b + gw.app_b) / 1e6)),
                   "split_chunk": gw.chunk, "splits": gw.splits},
        "tokens_per_s_per_layer": round(world * max(tokens_per_s_per_layer,
                                                    fused["tokens_per_s_per_layer"] / world
                                                    if fused else 0.0), 1),
        "tokens_per_s_per_layer_two_calls": round(world * tokens_per_s_per_layer, 1),
        "fused_step": fused,
        "append_gbs": round(append_gbs, 2),
        "decode_us_per_layer": round(per_layer_decode * 1e6, 3),
        "append_us_per_layer": round(per_layer_append * 1e6, 3),
        "roofline": rl,
        "gpu_launches": gw.launches_per_layer * n_layers * K,
        "clocks": sampler.summary(),
        "e2e": e2e,
    }
    # ---- every workload on its own (medians over repeats); the headline's
    # caches and graphs are reused for its own entry
    if QLEN == 1 and not args.no_per_config and args.layers == 0:
        pc = {}
        for name, w in synth.ALL_WORKLOADS.items():
            pc[name] = per_config_entry(kvq, w, dev, K, W, world,
                                        gw=gw if name == wl.name else None)
        pc["long_context_prefill2048"] = prefill_entry(kvq, synth.WORKLOADS["long_context"], dev,
                                                       K, W, world, 2048)
        line["per_config"] = pc
    gw.close()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_e2e(kvq, wl, layers, workspace, dev, K, W, world):
    """Same metric through the public Python API with host buffers: each step
    copies every layer's q / k_new / v_new from pinned host memory (one packed
    copy for the step), runs the decode step eagerly for every layer (one
    kvq_append_decode call where the cache format allows, else kvq_append +
    kvq_decode_attn), and copies all the outputs back (one packed copy)."""
    n = len(layers)
    # the step's inputs, packed layer after layer: q, k_new, v_new (bf16)
    parts = [t for ly in layers for t in (ly.q, ly.k_new, ly.v_new)]
    h_in = torch.cat([t.reshape(-1).cpu() for t in parts]).pin_memory()
    d_in = torch.empty_like(h_in, device=dev)
    views, off = [], 0
    for t in parts:
        views.append(d_in[off:off + t.numel()].view(t.shape))
        off += t.numel()
    outs = [ly.out for ly in layers]
    d_out = torch.empty(sum(t.numel() for t in outs), dtype=torch.float32, device=dev)
    h_out = torch.empty(d_out.numel(), dtype=torch.float32).pin_memory()
    out_views, off = [], 0
    for t in outs:
        out_views.append(d_out[off:off + t.numel()].view(t.shape))
        off += t.numel()
    h2d = h_in.numel() * h_in.element_size()
    d2h = h_out.numel() * h_out.element_size()
    stream = torch.cuda.Stream(dev)

    def step():
        with torch.cuda.stream(stream):
            d_in.copy_(h_in, non_blocking=True)
            for i, ly in enumerate(layers):
                q, k_new, v_new = views[3 * i:3 * i + 3]
                if ly.fusable:
                    ly.step_fused(kvq, workspace, k_new, v_new, q=q, out=out_views[i],
                                  stream=stream)
                else:
                    ly.append(kvq, k_new, v_new, stream=stream)
                    ly.decode(kvq, workspace, q=q, out=out_views[i], stream=stream)
            h_out.copy_(d_out, non_blocking=True)

    def timed(run):
        # (a graph replays on the current stream: the launching stream here)
        with torch.cuda.stream(stream):
            for _ in range(max(W, 1)):
                run()
        torch.cuda.synchronize(dev)
        barrier(dev)
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(K):
                run()
            stop.record(stream)
        stop.synchronize()
        torch.cuda.synchronize(dev)
        return reduce_max(start.elapsed_time(stop) / 1e3, dev)

    t = timed(step)
    dec_b = sum(decode_bytes(wl, ly.seq_lens_list, 16 if ly.paged else 0) for ly in layers)
    out = {"value": round(world * dec_b * K / t / 1e9, 3), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "ms_per_step": round(1e3 * t / K, 4), "layers_per_step": n,
           "how": "eager calls through the Python API, one per layer"}
    # the same step captured once as a CUDA graph (the pinned-host copies in
    # and out are nodes of it) and replayed: the calls' host cost drops out
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    torch.cuda.synchronize(dev)
    tg = timed(g.replay)
    out["graph"] = {"value": round(world * dec_b * K / tg / 1e9, 3), "unit": "GB/s",
                    "ms_per_step": round(1e3 * tg / K, 4),
                    "how": "the step (copies in, every layer's call, copy out) replayed "
                           "from one captured CUDA graph"}
    del g
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    ap.add_argument("--workload", choices=list(synth.ALL_WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--layers", type=int, default=0, help="layer caches per step (0: default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload")
    ap.add_argument("--cpu-budget-s", type=float, default=10.0,
                    help="seconds of oracle work per CPU-baseline leg")
    ap.add_argument("--cpu-layers", type=int, default=1500)
    ap.add_argument("--qlen", type=int, default=1,
                    help="queries per head per step: > 1 runs chunk attention steps")
    args = ap.parse_args(argv)
    global QLEN
    if args.qlen < 1:
        ap.error("--qlen must be at least 1")
    QLEN = args.qlen
    args.warmup = max(args.warmup, 3)     # timing rule: at least 3 untimed warm-up steps
    wl = synth.ALL_WORKLOADS[args.workload]
    if args.impl == "reference":
        if args.workload not in synth.WORKLOADS:
            ap.error("the reference arm runs the five parity workloads")
        return run_reference(args, wl)
    return run_kvq(args, wl)


if __name__ == "__main__":
    sys.exit(main())

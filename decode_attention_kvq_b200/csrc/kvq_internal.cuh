// kvq_internal.cuh -- declarations shared by the CUDA translation units of
// libkvq (launchers, parameter blocks, small device helpers).  Not part of
// the public ABI; the public declarations live in include/kvq.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// bf16 bits -> fp32 (exact widening: bf16 is the top half of binary32).
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h16) {
    return __uint_as_float(h16 << 16);
}

__device__ __forceinline__ void raise_flag(int32_t* d_err, uint32_t bits) {
    if (d_err) atomicOr(reinterpret_cast<int*>(d_err), static_cast<int>(bits));
}

// ------------------------------------------------- INT8 quantiser (append)
// Method (abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
// CudaQuantizedKvCache::quantize_tensor): s = max(max |x|, 1e-8) / 127 and
// byte = clamp(round_half_away(x / s) + 128, 0, 255), both divisions IEEE
// round-to-nearest fp32.  Every kernel that quantises (the append kernels and
// the decode kernel's fused append) uses these, so their bytes agree.

// the scale of a row (or 32-value group) from its absolute maximum
__device__ __forceinline__ float q8_scale(float amax) {
    return __fdiv_rn(amax < 1e-8f ? 1e-8f : amax, 127.0f);
}

// round_half_away(x / s) for the IEEE-rounded fp32 quotient x / s, mostly
// without a division.  r = x * inv, inv = 1 / s rounded once and the product
// rounded once, is within 2^-23 |x / s| of the quotient, i.e. within 2.3e-5
// of the rounded quotient wherever |x / s| <= 128 (every in-range byte).  So
// unless r lies within 1e-4 of a point halfway between two integers, the
// rounded quotient lies strictly inside the same interval (k - 0.5, k + 0.5)
// and rounds to the same integer as r; those near-ties take the IEEE division.
// With t = |r| + 0.5 (exact while |r| < 2^22), |r| is within 1e-4 of a tie
// exactly when t is within 1e-4 of an integer, and round_half_away(|r|) is
// floor(t).  Beyond |x / s| = 128 every rounding clamps to the same byte (at
// and above 2^22 every t is an integer: the division decides).
__device__ __forceinline__ int round_quotient(float x, float s, float inv) {
    const float r = __fmul_rn(x, inv);
    const float t = __fadd_rn(fabsf(r), 0.5f);
    if (fabsf(__fadd_rn(t, -rintf(t))) < 1e-4f) return static_cast<int>(roundf(__fdiv_rn(x, s)));
    const int k = static_cast<int>(floorf(t));
    return r < 0.f ? -k : k;
}

// the stored byte of x under scale s (inv = __frcp_rn(s))
__device__ __forceinline__ uint32_t q8_byte(float x, float s, float inv) {
    const int v = round_quotient(x, s, inv) + 128;
    return static_cast<uint32_t>(v < 0 ? 0 : (v > 255 ? 255 : v));
}

// ---------------------------------------------------------------- append
struct AppendParams {
    const uint16_t* k_new;   // [B, Hk, T, D] bf16
    const uint16_t* v_new;
    uint8_t* k_dst;          // contiguous cache or paged arena
    uint8_t* v_dst;
    float* k_scale;
    float* v_scale;
    const int32_t* pos;      // [B]
    const int32_t* table;    // paged only: [B, max_pages]
    int32_t* d_err;
    int B, Hk, T, D;
    int group32;             // 1: 32-value groups, 0: one scale per row
    int fp8;                 // 0: INT8 with scales, 1: FP8 E4M3, 2: FP8 E5M2 (no scales)
    int static_ns;           // per-head (1) / per-channel (D) scales per (b, kv head); 0: per row
    int max_seq;             // contiguous capacity
    int page_size;           // 0: contiguous, else paged
    int max_pages, num_pages;
};
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);
// per-head / per-channel scales set from the call's tokens, then the tokens quantised
cudaError_t launch_append_calibrate(const AppendParams& p, cudaStream_t s);
// mixed cache: tokens leaving the bf16 window (ring [B, Hk, W, D]) are quantised
// into the INT8 part, the new ones enter the window; p.pos holds the old lengths
cudaError_t launch_append_mixed(const AppendParams& p, uint16_t* k_ring, uint16_t* v_ring, int W,
                                cudaStream_t s);

// --------------------------------------------------------------- dequant
cudaError_t launch_dequant(const uint8_t* q, const float* scale, int64_t rows, int D,
                           int group32, int fp8, int static_ns, float* out, cudaStream_t s);

// ---------------------------------------------------------------- decode
struct DecodeParams {
    const uint16_t* q;       // [B, Hq, D] bf16
    const uint8_t* k;        // cache / arena
    const uint8_t* v;
    const float* k_scale;
    const float* v_scale;
    const int32_t* table;    // paged: [B, max_pages]
    const int32_t* seq_lens; // [B]
    float* out;              // [B, Hq, D]
    float* ws_o;             // [B*Hq, splits, D] partial outputs (unnormalised)
    float* ws_m;             // [B*Hq, splits] running max (log2 domain)
    float* ws_l;             // [B*Hq, splits] running sum
    int32_t* d_err;
    int B, Hq, Hk, G, D;
    int group32;
    int fp8;                 // 0: INT8 with scales, 1: FP8 E4M3, 2: FP8 E5M2 (no scales)
    int static_ns;           // per-head (1) / per-channel (D) scales per (b, kv head); 0: per token
    int page_size, max_seq, max_pages, num_pages;
    int chunk;               // KV tokens per split
    int splits;              // chunks of the longest sequence
    int grid;                // persistent CTAs of the split kernel
    int seg_w;               // partition weight of a (sequence, kv head) start, in items
    int one_item;            // the plan's items fit the grid: CTA c takes item c
    int qlen;                // queries per (sequence, q head): 1 for decode, T for a chunk
                             // (Hq and G then count (head, query) rows, query fastest)
    int window;              // sliding window w (0: none): a query at position p sees p - w + 1 .. p
    int recent;              // mixed cache: the newest `recent` tokens are bf16 in a ring (0: none);
                             // the split kernel walks the INT8 part and writes partials only
    const uint16_t* rk;      // mixed cache: bf16 rings [B, Hk, recent, D] (K and V)
    const uint16_t* rv;
    float scale_log2;        // attn_scale * log2(e)
    // fused append (decode, INT8 per token / group-32): the step's new token
    // k_new / v_new bf16 [B, Hk, 1, D] is quantised into position L - 1 of
    // the cache (written through k_w / v_w / ks_w / vs_w, the same memory as
    // k / v / k_scale / v_scale) by the CTA whose range holds it; null: none
    const uint16_t* k_new;
    const uint16_t* v_new;
    uint8_t* k_w;
    uint8_t* v_w;
    float* ks_w;
    float* vs_w;
};


// Sliding window: the oldest position any of a sequence's qlen queries sees
// is L - qlen - window + 1.  The kernels count a sequence's tokens from that
// position rounded down to a multiple of 16 (whole pages, 16-byte aligned
// scale rows), mask the few below it, and plan over L - base tokens.
__host__ __device__ __forceinline__ int window_base(int L, int qlen, int window) {
    if (window <= 0) return 0;
    const int lo = L - qlen - window + 1;
    return lo > 0 ? (lo & ~15) : 0;
}

// The number of tokens the kernels walk for a sequence of length L: its INT8
// part (all of it, or L - recent for a mixed cache) from its window base; -1
// when L < 0 or the INT8 part is beyond the capacity or the plan.
__device__ __forceinline__ int walked_len(int L, int64_t cap, int64_t plan, int qlen, int window,
                                          int recent = 0) {
    if (L < 0) return -1;
    int n = L > recent ? L - recent : 0;
    if (n > cap) return -1;
    n -= window_base(n, qlen, window);
    return n > plan ? -1 : n;
}
constexpr int kMaxBatch = 1024;                              // sequences per call
constexpr int kMaxRecent = 2048;                             // mixed cache: bf16 window tokens
constexpr int kMaxGrid = 1024;                               // persistent CTAs
// the split kernel (tensor-core, or the CUDA-core one when simt) and, where
// the partials are not folded in it, the combine kernel
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s, bool simt = false);
// CUDA-core split kernel (kvq_decode_simt.cu): any D % 16 == 0 up to 256,
// any rows per kv head, one item per CTA
cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t s);
// mixed cache: the bf16 window's partial and the INT8 partials into the output
cudaError_t launch_recent_combine(const DecodeParams& p, cudaStream_t s);
// tensor-core split kernel (kvq_decode_tc.cu)
cudaError_t launch_decode_split_tc(const DecodeParams& p, cudaStream_t s);

// FP8 code of a bf16 value, truncated toward zero (the format's mantissa bits
// kept, the rest dropped), from the bf16 fields directly: E4M3 (fmt 1, bias
// 7, 3 mantissa bits) saturates at +-448 (0x7E, also where the truncated code
// would be the NaN pattern 0x7F); E5M2 (fmt 2, bias 15, 2 mantissa bits)
// gives +-inf (0x7C) from 2^16 up.  Below the smallest subnormal: a zero of
// the value's sign; +-0 -> 0x00; NaN -> 0xFF; inf -> 0x7F / 0xFF (E4M3),
// 0x7C / 0xFC (E5M2).
__device__ __forceinline__ uint32_t fp8_from_bf16(uint32_t h, int fmt) {
    const uint32_t s = (h >> 8) & 0x80u;                 // sign at bit 7
    const int eb = static_cast<int>((h >> 7) & 0xffu);    // bf16 biased exponent
    const uint32_t m7 = h & 0x7fu;                        // bf16 mantissa bits
    const bool e4 = fmt == 1;
    const int mb = e4 ? 3 : 2;
    if (eb == 0xff) {
        if (m7) return 0xffu;
        return e4 ? (s ? 0xffu : 0x7fu) : (s | 0x7cu);
    }
    if ((h & 0x7fffu) == 0) return 0u;                    // +-0
    const int E = eb - 127 + (e4 ? 7 : 15);               // FP8 biased exponent
    if (e4 ? E > 15 : E > 30) return s | (e4 ? 0x7eu : 0x7cu);
    if (E <= 0) {                                         // subnormal (or zero) code
        const int keep = mb + E;                          // significand bits kept
        if (keep <= 0 || eb == 0) return s;
        return s | ((0x80u | m7) >> (8 - keep));          // 8-bit significand, top bits
    }
    uint32_t c = s | (static_cast<uint32_t>(E) << mb) | (m7 >> (7 - mb));
    if (e4 && (c & 0x7fu) == 0x7fu) c = s | 0x7eu;
    return c;
}

// 2-D u8 TMA tensor map over `rows` rows of D bytes (box of box_rows rows,
// 128-byte swizzle for D = 128, 64-byte for D = 64), cached per host thread.
cudaError_t make_tile_map(CUtensorMap* map, const void* base, int D, int64_t rows, int box_rows);

// Dense chunk attention on the tcgen05 tensor cores (kvq_chunk_tc.cu): the
// shapes it covers, and its launch (dp as built for the chunk, Hq / G / T the
// call's own head count, group and chunk length).
bool chunk_tc_supported(int D, int G, int T, int group32, int fp8, int static_ns, int page_size,
                        int window, int recent);
cudaError_t launch_chunk_tc(const DecodeParams& dp, int Hq, int G, int T, cudaStream_t s);

// Programmatic dependent launch: wait for the preceding grid's writes, and
// let the next grid in the stream be scheduled early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace kvq

/*
 * kvq.h -- C ABI of libkvq: INT8 KV-cache quantisation on append and decode
 * attention computed directly on the INT8 cache, for NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are raw pointers to caller-owned DEVICE memory,
 *    densely packed in the row-major layout given for each argument.  The
 *    library never allocates, frees or copies host<->device inside these
 *    calls, and never synchronises the stream (except kvq_read_error).
 *  - bf16 tensors are passed as uint16_t* (the raw bf16 bits).
 *  - Every pointer that is read or written with vector loads must be 16-byte
 *    aligned (all tensor arguments except d_pos, d_seq_lens, page_table,
 *    d_err and the per-head scale arrays, which need 4-byte alignment).
 *    torch allocations satisfy this.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *    default stream.  All work is enqueued on it, in order.
 *  - Argument faults the host can see are reported synchronously as
 *    KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED before anything is enqueued.
 *    A failed launch returns KVQ_ERR_CUDA.
 *  - Faults only the device can see (a write position beyond the cache
 *    capacity, a page-table entry outside the arena, a sequence length
 *    beyond the capacity) never trap: the offending row / page is skipped
 *    and the matching KVQ_DEVERR_* bit is OR-ed into *d_err when d_err is
 *    not NULL.  kvq_read_error fetches and clears that word.
 *
 * Quantisation (both append calls), per (token, kv head) or per 32-value
 * group along head_dim: m = max(max_i |x_i|, 1e-8); s = m / 127 (IEEE fp32
 * division); byte_i = clamp(round_half_away_from_zero(x_i / s) + 128, 0, 255)
 * with x_i / s an IEEE fp32 division; s is stored as fp32.  The result is
 * bit-exact with that definition.  Source: abaddon 0.2.0-rc.1,
 * src/kv_cache_quant_cuda.rs, CudaQuantizedKvCache::quantize_tensor (per
 * token, offset-128 bytes); abaddon 0.2.0-rc.2, src/kv_cache_quant.rs, module
 * doc "Quantization Strategy"; group-32 fp32 scales as in realizar 0.8.5,
 * src/cuda/executor/kv_cache_q8_init.rs, init_kv_cache_q8_gpu, and
 * combs-models 0.2.2, src/kv.rs, kv_quantize (KV_QUANT_GROUP = 32).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, too small workspace */
    KVQ_ERR_UNSUPPORTED = 2,   /* valid but not built: head_dim or GQA group outside the kernels' set */
    KVQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    KVQ_ERR_DEVICE_FLAG = 4,   /* kvq_read_error found device-side error bits */
    KVQ_ERR_SCRATCH_TOO_SMALL = 5, /* kvq_decode_attn_noalloc: the problem needs more split-K
                                      scratch than the library's fixed array holds */
    KVQ_ERR_OUT_OF_PAGES = 6       /* kvq_pager_append: the free pages cannot hold the tokens */
} kvq_status;

/*
 * How the cache stores values: INT8 offset-128 bytes with fp32 scales (per
 * token or per 32-value group), or FP8 bytes with no scale.  The FP8 modes
 * follow llama-gguf 0.14.0, src/model/kv_quantized.rs, KVCacheFormat::
 * Fp8E4M3 / Fp8E5M2 with quantize_fp8_e4m3 / quantize_fp8_e5m2: each bf16
 * value is TRUNCATED toward zero to the format (a zero of its sign below the
 * smallest subnormal; E4M3 saturates at +-448 -- also for values in
 * [480, 512), whose truncated code would be the NaN pattern -- and E5M2 gives
 * +-inf from 2^16 up); attention reads the bytes' exact values.  In FP8 modes
 * every scale pointer is ignored and may be NULL (NG = 0).
 */
typedef enum kvq_scale_mode {
    KVQ_SCALE_PER_TOKEN = 0,   /* one fp32 scale per (token, kv head): NG = 1 */
    KVQ_SCALE_GROUP32 = 1,     /* one fp32 scale per 32 values along head_dim: NG = D / 32 */
    KVQ_FP8_E4M3 = 2,          /* FP8 E4M3 bytes (bias 7, 3 mantissa bits), no scale: NG = 0 */
    KVQ_FP8_E5M2 = 3,          /* FP8 E5M2 bytes (bias 15, 2 mantissa bits), no scale: NG = 0 */
    KVQ_SCALE_PER_HEAD = 4,    /* INT8, one fp32 scale per (sequence, kv head): scales [B, Hk, 1] */
    KVQ_SCALE_PER_CHANNEL = 5  /* INT8, one per (sequence, kv head, channel): scales [B, Hk, D] */
} kvq_scale_mode;

/*
 * Per-head and per-channel modes (abaddon 0.2.0-rc.1,
 * src/kv_cache_quant_cuda.rs, QuantGranularity::PerHead / PerChannel,
 * OptimizedQuantizedKvCache::quantize_with_granularity): the scale arrays are
 * not per token but per (sequence, kv head) -- the page's shapes (batch,
 * heads, 1, 1) and (batch, heads, 1, head_dim) -- for contiguous caches and
 * paged arenas alike.  kvq_append_calibrate sets them from one call's tokens
 * (max |x| over the tokens and head_dim, or over the tokens per channel,
 * floored at 1e-8, divided by 127) and quantises those tokens; kvq_append /
 * kvq_append_paged in these modes quantise with the stored scales (the page
 * concatenates later calls' scales along the token axis, which its own
 * dequantise cannot broadcast: here a sequence keeps the scales of its
 * calibrating call).  Every value uses the per-token rounding rule; values
 * beyond the calibrated range clamp to the byte range.
 */

/* Device-side error bits (OR-ed into *d_err). */
#define KVQ_DEVERR_POS 1u    /* append range [pos, pos + T) outside [0, capacity) */
#define KVQ_DEVERR_PAGE 2u   /* page-table entry outside [0, num_pages) in the used range */
#define KVQ_DEVERR_LEN 4u    /* decode sequence length outside [0, capacity] */
#define KVQ_DEVERR_TIMEOUT 8u /* a bounded wait inside a kernel gave up (never expected) */

typedef void *kvq_stream_t;  /* cudaStream_t */

/*
 * kvq_append -- quantise T new tokens per (sequence, kv head) and write them
 * in place into a contiguous INT8 cache.
 *   k_new, v_new  bf16 [B, Hk, T, D]        new keys / values (read)
 *   d_pos         int32 [B]                 first write position of each sequence
 *   k_cache, v_cache  u8 [B, Hk, max_seq, D]   offset-128 bytes (written at
 *                                              positions d_pos[b] .. d_pos[b]+T-1)
 *   k_scale, v_scale  fp32 [B, Hk, max_seq, NG]
 *   d_err         int32 [1] or NULL         device error word (KVQ_DEVERR_POS)
 * Requirements: B, Hk, T >= 1; 16 <= D <= 256, D % 16 == 0; GROUP32 needs
 * D % 32 == 0; max_seq >= 1.  Positions are arbitrary within capacity (a
 * later append may overwrite a slot); a sequence whose range leaves
 * [0, max_seq) is skipped and flagged.
 * Source: abaddon 0.2.0-rc.1, kv_cache_quant_cuda.rs, CudaQuantizedKvCache::
 * append (input layout [batch, kv_heads, new_seq, head_dim]); realizar 0.8.5,
 * kv_cache_q8_init.rs, write_kv_q8 (write at an explicit position below the
 * capacity, capacity-strided per head).
 */
kvq_status kvq_append(const uint16_t *k_new, const uint16_t *v_new, int B, int Hk, int T, int D,
                      kvq_scale_mode mode, const int32_t *d_pos, uint8_t *k_cache,
                      uint8_t *v_cache, float *k_scale, float *v_scale, int max_seq,
                      int32_t *d_err, kvq_stream_t stream);

/*
 * kvq_append_paged -- as kvq_append, but the cache is a paged arena.
 *   k_arena, v_arena  u8 [num_pages, Hk, page_size, D]
 *   k_scale, v_scale  fp32 [num_pages, Hk, page_size, NG]
 *   page_table    int32 [B, max_pages]      physical page of each logical page
 * Logical position g of sequence b is stored in physical page
 * page_table[b][g / page_size], slot g % page_size.  page_size must be 16.
 * A token whose page entry is outside [0, num_pages) is skipped and flagged
 * with KVQ_DEVERR_PAGE; a range beyond max_pages * page_size with
 * KVQ_DEVERR_POS.
 * Source: combs-models 0.2.2, src/kv.rs, PagedKVCache (arena layout,
 * DEFAULT_PAGE_SIZE = 16) and PagedKVCache::attention_opts (slot arithmetic;
 * each token quantised once, never re-quantised).
 */
kvq_status kvq_append_paged(const uint16_t *k_new, const uint16_t *v_new, int B, int Hk, int T,
                            int D, kvq_scale_mode mode, const int32_t *d_pos, uint8_t *k_arena,
                            uint8_t *v_arena, float *k_scale, float *v_scale,
                            const int32_t *page_table, int max_pages, int num_pages,
                            int page_size, int32_t *d_err, kvq_stream_t stream);

/*
 * kvq_append_calibrate -- per-head / per-channel quantisation of T new tokens
 * per (sequence, kv head) into a contiguous cache: first the scales of each
 * (sequence, kv head) are computed from these T tokens (mode
 * KVQ_SCALE_PER_HEAD: one from all T * D values; KVQ_SCALE_PER_CHANNEL: one
 * per channel from its T values) and written to k_scale / v_scale
 * ([B, Hk, 1] or [B, Hk, D]), then the tokens are quantised with them at
 * positions d_pos[b] .. d_pos[b] + T - 1 (bit-exact with that definition).
 * Other arguments, requirements and errors as for kvq_append; a sequence
 * whose range leaves the capacity is skipped (its scales untouched).
 * Source: abaddon 0.2.0-rc.1, kv_cache_quant_cuda.rs,
 * OptimizedQuantizedKvCache::quantize_with_granularity.
 */
kvq_status kvq_append_calibrate(const uint16_t *k_new, const uint16_t *v_new, int B, int Hk,
                                int T, int D, kvq_scale_mode mode, const int32_t *d_pos,
                                uint8_t *k_cache, uint8_t *v_cache, float *k_scale,
                                float *v_scale, int max_seq, int32_t *d_err, kvq_stream_t stream);

/*
 * Where decode attention finds the INT8 cache.  page_size == 0 selects the
 * contiguous layout of kvq_append, page_size == 16 the arena of
 * kvq_append_paged.  Unused fields are ignored.
 */
typedef struct kvq_cache_view {
    const uint8_t *k;          /* [B, Hk, max_seq, D] or [num_pages, Hk, page_size, D] */
    const uint8_t *v;
    const float *k_scale;      /* [B, Hk, max_seq, NG] or [num_pages, Hk, page_size, NG] */
    const float *v_scale;
    int32_t page_size;         /* 0 (contiguous) or 16 (paged) */
    int32_t max_seq;           /* contiguous: capacity per (sequence, kv head) */
    const int32_t *page_table; /* paged: int32 [B, max_pages] (device) */
    int32_t max_pages;         /* paged */
    int32_t num_pages;         /* paged: pages in the arena */
} kvq_cache_view;

/*
 * kvq_decode_attn -- one decode query per (sequence, q head) attending to
 * the sequence's whole cached window, with dequantisation fused into Q.K^T
 * and P.V:
 *   z_t = attn_scale * sum_d q_d * (k_t,d - 128) * sk_t,grp(d)
 *   out = sum_t softmax(z)_t * (v_t,d - 128) * sv_t,grp(d)
 * Query head h reads kv head h / (Hq / Hk) (GQA, heads repeated
 * consecutively).  A decode query is the newest position, so the causal
 * window is the whole cache: no mask is applied.
 *   q           bf16 [B, Hq, D]
 *   kv          cache view (see above)
 *   d_seq_lens  int32 [B]   cached length of each sequence INCLUDING the token
 *                           just appended; 0 gives a zero output row
 *   max_seq_len_hint  host upper bound of d_seq_lens (plans the split-K grid;
 *                     positions beyond it are not read)
 *   attn_scale  usually 1 / sqrt(D)
 *   out         fp32 [B, Hq, D]
 *   workspace   device scratch of at least kvq_decode_workspace_bytes(...)
 *               bytes (same B, Hq, Hk, D, hint, num_splits), 16-byte
 *               aligned; may be NULL when that size is 0.  Contents on entry
 *               are ignored.
 *   num_splits  0 = automatic; otherwise the requested number of KV splits
 *               per sequence (split-K / flash-decoding)
 *   d_err       int32 [1] or NULL (KVQ_DEVERR_LEN, KVQ_DEVERR_PAGE)
 * Requirements: Hq % Hk == 0; 16 <= D <= 256 with D % 16 == 0 (GROUP32:
 * D % 32 == 0); B <= 65535, Hq <= 65535 (otherwise KVQ_ERR_INVALID_ARG /
 * KVQ_ERR_UNSUPPORTED); B * Hk * splits below 2^31 (KVQ_ERR_UNSUPPORTED).
 * D in {64, 128} with Hq / Hk <= 16, B <= 1024 and the cache below 2^31
 * rows of D bytes runs on the tensor-core split kernel; every other shape
 * on the CUDA-core split kernel (same results within the stated bar,
 * lower throughput).
 * Source: abaddon 0.2.0-rc.1, kv_cache_quant_cuda.rs, module doc "Fused
 * approach" and CudaQuantizedKvCache::forward_attention (scores with
 * on-the-fly K dequantisation, softmax, P.V with on-the-fly V
 * dequantisation); combs-models 0.2.2, src/kv.rs, attend and repeat_kv
 * (scale applied after the dot product, GQA mapping, a single decode query
 * needs no mask).  Split-K with an online softmax and a combine step is this
 * library's own (flash-decoding), not from those pages.
 */
kvq_status kvq_decode_attn(const uint16_t *q, int B, int Hq, int Hk, int D, kvq_scale_mode mode,
                           const kvq_cache_view *kv, const int32_t *d_seq_lens,
                           int max_seq_len_hint, float attn_scale, float *out, void *workspace,
                           size_t workspace_bytes, int num_splits, int32_t *d_err,
                           kvq_stream_t stream);

/* Workspace bytes kvq_decode_attn needs for these arguments (0 when no split is needed). */
size_t kvq_decode_workspace_bytes(int B, int Hq, int Hk, int D, int max_seq_len_hint,
                                  int num_splits);

/*
 * kvq_append_decode -- one decode step in one call: the step's new token of
 * every (sequence, kv head) is quantised into the cache at position
 * L_b - 1, then the step's query attends to positions 0 .. L_b - 1, with the
 * same fused dequantisation as kvq_decode_attn.  The result (cache bytes,
 * scales and output) is that of kvq_append (or kvq_append_paged) with
 * d_pos[b] = L_b - 1 followed by kvq_decode_attn; the quantisation is the
 * same bit-exact rule.  The token is quantised by the CTA whose range of the
 * cache holds position L_b - 1, into its shared-memory tile and into the
 * cache, so no separate append launch runs.
 *   k_new, v_new  bf16 [B, Hk, 1, D]   the step's new keys / values (read)
 *   kv          cache view as for kvq_decode_attn; its k, v, k_scale and
 *               v_scale arrays are WRITTEN at position L_b - 1 (they must be
 *               writable device memory)
 *   d_seq_lens  int32 [B]  L_b, the length INCLUDING the new token; 0: no
 *               token is written and the output row is zero
 *   the other arguments as for kvq_decode_attn (workspace: at least
 *   kvq_decode_workspace_bytes(...) bytes).
 * Requirements: those of kvq_decode_attn, with mode PER_TOKEN or GROUP32
 * (other modes: KVQ_ERR_UNSUPPORTED).  A sequence whose length is beyond the
 * capacity writes nothing and is flagged KVQ_DEVERR_LEN; a missing page of
 * position L_b - 1 writes nothing and is flagged KVQ_DEVERR_PAGE.
 * Source: abaddon 0.2.0-rc.1, kv_cache_quant_cuda.rs, CudaQuantizedKvCache::
 * append followed by forward_attention (a decode step appends its token and
 * attends to the cache that now holds it).
 */
kvq_status kvq_append_decode(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                             int B, int Hq, int Hk, int D, kvq_scale_mode mode,
                             const kvq_cache_view *kv, const int32_t *d_seq_lens,
                             int max_seq_len_hint, float attn_scale, float *out, void *workspace,
                             size_t workspace_bytes, int num_splits, int32_t *d_err,
                             kvq_stream_t stream);

/*
 * kvq_chunk_attn -- a chunk of T new queries per (sequence, q head), causal
 * from the chunk's end: the chunk's T tokens are the last T positions of the
 * sequence (appended before the call), so query i sits at position
 * L - T + i and attends to positions 0 .. L - T + i, with the same fused
 * dequantisation as kvq_decode_attn.  T = 1 is kvq_decode_attn.
 *   q           bf16 [B, Hq, T, D]
 *   kv          cache view (see above)
 *   d_seq_lens  int32 [B]   L, the cached length INCLUDING the chunk's T
 *                           tokens; 0 gives zero output rows, and 0 < L < T
 *                           is a length error (KVQ_DEVERR_LEN, zero rows)
 *   out         fp32 [B, Hq, T, D]
 *   workspace   at least kvq_chunk_workspace_bytes(...) bytes, as for
 *               kvq_decode_attn
 *   the other arguments as for kvq_decode_attn.
 * Requirements: those of kvq_decode_attn with the GQA group counted in
 * (head, query) rows, (Hq / Hk) * T <= 2^19.  More than 16 rows per kv head
 * run on the dense tcgen05 kernel when D = 128, the scales are per token,
 * the cache is contiguous and there is no window (that kernel needs no
 * workspace); otherwise on the CUDA-core split kernel.  T < 1 is
 * KVQ_ERR_INVALID_ARG.
 * Source: abaddon 0.2.0-rc.1, kv_cache_quant_cuda.rs,
 * CudaQuantizedKvCache::forward_attention (prefill with q_len > 1: the cache
 * offset is seq_len - q_len and query q_pos sees the positions up to
 * cache_offset + q_pos); combs-models 0.2.2, src/kv.rs, attend (a query at
 * global position p attends the keys at positions <= p).
 */
kvq_status kvq_chunk_attn(const uint16_t *q, int B, int Hq, int Hk, int T, int D,
                          kvq_scale_mode mode, const kvq_cache_view *kv,
                          const int32_t *d_seq_lens, int max_seq_len_hint, float attn_scale,
                          float *out, void *workspace, size_t workspace_bytes, int num_splits,
                          int32_t *d_err, kvq_stream_t stream);

/* Workspace bytes kvq_chunk_attn needs for these arguments (0 when no split is needed). */
size_t kvq_chunk_workspace_bytes(int B, int Hq, int Hk, int T, int D, int max_seq_len_hint,
                                 int num_splits);

/*
 * kvq_window_attn -- sliding-window attention on the INT8 cache: T >= 1 new
 * queries per (sequence, q head) (T = 1: a decode step), query i at position
 * p = L - T + i attending to the positions max(0, p - window + 1) .. p, with
 * the fused dequantisation of kvq_decode_attn.  Only the last
 * T + window - 1 positions of each sequence (from a 16-aligned start) are
 * read, so the work is bounded by the window, not the length.
 *   q       bf16 [B, Hq, D] (T = 1) or [B, Hq, T, D];  out fp32 of q's shape
 *   window  w >= 1 keys per query, the newest included (a layer that keeps
 *           w - 1 past tokens and appends one sees w)
 *   workspace  at least kvq_window_workspace_bytes(...) bytes
 *   the other arguments as for kvq_chunk_attn (L counts the T new tokens,
 *   0 < L < T is a length error).
 * The cache holds every position (positions are rows, as for the other
 * calls).  A sliding layer that keeps only its last w tokens in a ring of w
 * rows (position g in row g % w) decodes with plain kvq_decode_attn over
 * min(L, w) rows instead: the softmax does not depend on the rows' order.
 * Requirements: those of kvq_chunk_attn; window < 1 or T < 1 is
 * KVQ_ERR_INVALID_ARG.
 * Source: combs-models 0.2.2, src/kv.rs, attend with a window (a key at k is
 * masked when k > p or k + w - 1 < p) as PagedKVCache::sliding_attention
 * uses it for sliding layers (transformers' sliding-window layers).
 */
kvq_status kvq_window_attn(const uint16_t *q, int B, int Hq, int Hk, int T, int D,
                           kvq_scale_mode mode, const kvq_cache_view *kv,
                           const int32_t *d_seq_lens, int max_seq_len_hint, int window,
                           float attn_scale, float *out, void *workspace, size_t workspace_bytes,
                           int num_splits, int32_t *d_err, kvq_stream_t stream);

/* Workspace bytes kvq_window_attn needs for these arguments (0 when no split is needed). */
size_t kvq_window_workspace_bytes(int B, int Hq, int Hk, int T, int D, int max_seq_len_hint,
                                  int window, int num_splits);

/*
 * Split plan kvq_decode_attn uses: KV tokens per split (*chunk) and the
 * largest number of splits of any sequence (*splits).  num_sms <= 0 means the
 * current device's SM count.  Returns KVQ_ERR_INVALID_ARG on bad sizes.
 */
kvq_status kvq_decode_plan(int B, int Hk, int max_seq_len_hint, int num_splits, int num_sms,
                           int *chunk, int *splits);

/*
 * ---- Mixed cache: the newest tokens unquantised --------------------------
 * A sequence's newest `window` tokens stay bf16 in a ring and the older ones
 * are INT8 (abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
 * DynamicQuantConfig::unquantized_window -- 128 by default -- and
 * OptimizedQuantizedKvCache::append / get_kv).  After any append of a
 * sequence of length L, positions 0 .. L - window - 1 are in the INT8 part (a
 * contiguous cache [B, Hk, max_seq, D] with the mode's scales) and the last
 * min(L, window) in the ring, bf16 [B, Hk, window, D], position g in row
 * g % window.
 */

/*
 * kvq_append_mixed -- append T new tokens per (sequence, kv head): they join
 * the window, and the tokens that leave it (positions max(0, L0 - window) ..
 * max(0, L0 + T - window) - 1, L0 = d_lens_old[b] the length before the
 * call) are quantised into the INT8 part with the mode's rule (per token,
 * group-32, or the stored per-head / per-channel scales).  Bit-exact with
 * that definition.
 *   k_new, v_new  bf16 [B, Hk, T, D];  d_lens_old int32 [B] (device)
 *   k_cache ... max_seq  the INT8 part, as for kvq_append
 *   k_ring, v_ring  bf16 [B, Hk, window, D];  1 <= window <= 2048
 * Modes: KVQ_SCALE_PER_TOKEN, GROUP32, PER_HEAD, PER_CHANNEL.  A sequence
 * whose INT8 part would exceed max_seq (or L0 < 0) is skipped and flagged
 * with KVQ_DEVERR_POS.  The caller advances its lengths by T.
 */
kvq_status kvq_append_mixed(const uint16_t *k_new, const uint16_t *v_new, int B, int Hk, int T,
                            int D, kvq_scale_mode mode, const int32_t *d_lens_old,
                            uint8_t *k_cache, uint8_t *v_cache, float *k_scale, float *v_scale,
                            int max_seq, uint16_t *k_ring, uint16_t *v_ring, int window,
                            int32_t *d_err, kvq_stream_t stream);

/*
 * kvq_decode_attn_mixed -- decode attention over a mixed cache: the query
 * attends to the INT8 part (fused dequantisation, split-K, any mode and
 * layout of kvq_decode_attn; kv views it) and to the bf16 window, in one
 * softmax.  d_seq_lens counts every token (INT8 part + window); the other
 * arguments as for kvq_decode_attn, with a workspace of at least
 * kvq_mixed_workspace_bytes(...) bytes (never 0: the INT8 partials of every
 * row pass through it).
 */
kvq_status kvq_decode_attn_mixed(const uint16_t *q, int B, int Hq, int Hk, int D,
                                 kvq_scale_mode mode, const kvq_cache_view *kv,
                                 const uint16_t *k_ring, const uint16_t *v_ring, int window,
                                 const int32_t *d_seq_lens, int max_seq_len_hint,
                                 float attn_scale, float *out, void *workspace,
                                 size_t workspace_bytes, int num_splits, int32_t *d_err,
                                 kvq_stream_t stream);

/* Workspace bytes kvq_decode_attn_mixed needs for these arguments. */
size_t kvq_mixed_workspace_bytes(int B, int Hq, int Hk, int D, int max_seq_len_hint, int window,
                                 int num_splits);

/*
 * kvq_dequant -- x = (byte - 128) * scale, one fp32 multiply per element,
 * bit-exact.
 *   q      u8 [rows, D];  scale fp32 [rows, NG];  out fp32 [rows, D]
 * Requirements: rows >= 0; 16 <= D, D % 16 == 0; GROUP32 needs D % 32 == 0.
 * Source: abaddon 0.2.0-rc.2, kv_cache_quant.rs, QuantizedKvCache::
 * dequantize; abaddon 0.2.0-rc.1, kv_cache_quant_cuda.rs, int8_dequant_bf16
 * (this library writes fp32 instead of bf16); realizar 0.8.5,
 * kv_cache_q8_init.rs, read_kv_q8.
 */
kvq_status kvq_dequant(const uint8_t *q, const float *scale, int64_t rows, int D,
                       kvq_scale_mode mode, float *out, kvq_stream_t stream);

/*
 * kvq_decode_attn_noalloc -- kvq_decode_attn for callers that cannot allocate
 * device memory.  The pages this library follows have no counterpart of this
 * call; it exists for integration.  Some callers cannot call cudaMalloc (or
 * any allocator) where they run attention: plugin or embedded hosts that
 * only hand over their own input and output buffers, runtimes whose
 * allocator this C interface cannot reach.  This entry point takes the same
 * arguments as
 * kvq_decode_attn minus the workspace, and uses instead a split-K scratch
 * array that lives inside the library: a file-scope __device__ array of
 * kvq_noalloc_scratch_bytes() bytes (16 MiB), present on every GPU that loads
 * the library until the process exits.
 *  - Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 *    library routine is called.
 *  - The first call on a device looks up the array's device address with
 *    cudaGetSymbolAddress (with that device current) and caches it.
 *  - Problems whose split-K scratch (kvq_decode_workspace_bytes for the same
 *    arguments) exceeds the array return KVQ_ERR_SCRATCH_TOO_SMALL before
 *    anything is enqueued.
 *  - Every call on a device shares the one array and leaves its last
 *    contents in it (nothing in it needs to start at zero).  Calls whose GPU
 *    work overlaps (different streams without ordering, or concurrent host
 *    threads on different streams) race on the array; serialise them.
 */
kvq_status kvq_decode_attn_noalloc(const uint16_t *q, int B, int Hq, int Hk, int D,
                                   kvq_scale_mode mode, const kvq_cache_view *kv,
                                   const int32_t *d_seq_lens, int max_seq_len_hint,
                                   float attn_scale, float *out, int num_splits, int32_t *d_err,
                                   kvq_stream_t stream);

/* Size in bytes of the scratch array kvq_decode_attn_noalloc uses (no counterpart on the pages). */
size_t kvq_noalloc_scratch_bytes(void);

/*
 * ---- Paged-cache bookkeeping on the host --------------------------------
 * A pager owns no device memory: it keeps, in caller-provided host memory,
 * the free-page allocator of one arena of num_pages pages, one page table and
 * one length per sequence, and the rollback rule of sliding-window layers.
 * Its table (kvq_pager_table) is the int32 [max_seqs, max_pages] page table,
 * -1 past each sequence's pages, that kvq_append_paged and the attention
 * calls read after the caller copies it to the device; kvq_pager_append
 * returns the write position to pass as d_pos.  Host code only; a pager is
 * not safe for concurrent use from several host threads.
 * Source: combs-models 0.2.2, src/kv.rs -- PageAllocator (free-page stack,
 * page 0 first, freed pages reused last-in first-out), CacheConfig::num_pages,
 * PagedKVCache::ensure_pages, popn, reset; one sequence there, one table per
 * sequence here, all sharing the allocator.
 */
typedef struct kvq_pager kvq_pager;

/* Host bytes a pager needs (0 on bad sizes).  num_windows: sliding-window
 * layers whose rollback rule the pager enforces (0 = none). */
size_t kvq_pager_bytes(int num_pages, int max_seqs, int max_pages, int num_windows);

/* Lays a pager out in `mem` (16-byte aligned, at least kvq_pager_bytes(...)
 * bytes, owned by the caller for the pager's lifetime): every page free,
 * every sequence empty.  windows[i] >= 2 are the sliding-window sizes w of
 * the model's sliding layers (a layer of window w keeps w - 1 past tokens).
 * Requirements: num_pages, max_seqs, max_pages, page_size >= 1;
 * max_pages * page_size < 2^31.  Otherwise KVQ_ERR_INVALID_ARG. */
kvq_status kvq_pager_init(void *mem, size_t bytes, int num_pages, int page_size, int max_seqs,
                          int max_pages, const int32_t *windows, int num_windows,
                          kvq_pager **pager);

/* Appends n >= 0 tokens to sequence seq: its table grows to
 * ceil((len + n) / page_size) pages, each new page popped from the free
 * stack, and the length becomes len + n; *pos (may be NULL) receives the old
 * length, the first write position.  KVQ_ERR_OUT_OF_PAGES when the free
 * pages cannot cover the growth and KVQ_ERR_INVALID_ARG beyond
 * max_pages * page_size tokens; in both cases nothing changes. */
kvq_status kvq_pager_append(kvq_pager *pager, int seq, int64_t n, int64_t *pos);

/* Rolls back the last n tokens of sequence seq (n clamped to its length):
 * pages that no longer hold a token go back onto the free stack, the last
 * page first.  Returns the number of tokens removed: 0 also when a sliding
 * layer has already evicted (length > w - 1 for some window w), in which
 * case nothing changes (the evicted tokens cannot be restored). */
int64_t kvq_pager_popn(kvq_pager *pager, int seq, int64_t n);

/* Sequence seq finished: all its pages freed, length 0 (no sliding-layer
 * rule: nothing is rolled back into).  Not on the page, whose cache holds
 * one sequence. */
kvq_status kvq_pager_release(kvq_pager *pager, int seq);

/* Every page free, every sequence empty. */
void kvq_pager_reset(kvq_pager *pager);

int kvq_pager_free_pages(const kvq_pager *pager);
int kvq_pager_pages_used(const kvq_pager *pager, int seq);
int64_t kvq_pager_seq_len(const kvq_pager *pager, int seq);
/* Host views into the pager's memory: table int32 [max_seqs, max_pages]
 * (-1 = no page) and lengths int32 [max_seqs]. */
const int32_t *kvq_pager_table(const kvq_pager *pager);
const int32_t *kvq_pager_lens(const kvq_pager *pager);

/* Human-readable name of a status code (static string). */
const char *kvq_status_string(kvq_status status);

/*
 * Synchronises `stream`, copies the device error word to *bits (may be NULL)
 * and clears it.  Returns KVQ_OK when it was 0, KVQ_ERR_DEVICE_FLAG when any
 * bit was set, KVQ_ERR_CUDA on a runtime failure.
 */
kvq_status kvq_read_error(int32_t *d_err, int32_t *bits, kvq_stream_t stream);

/* kvq_read_error without the bits: synchronises `stream`, clears the device
 * error word and returns KVQ_OK (it was 0) or KVQ_ERR_DEVICE_FLAG (for
 * tests; the name of the helper in the boundary's plan). */
kvq_status kvq_check_error(int32_t *d_err, kvq_stream_t stream);

/*
 * Bytes of an INT8 cache with fp32 scales: layers * 2 * Hk * seq * (D + 4 * NG)
 * (NG = 0 for the FP8 modes).
 * Source: realizar 0.8.5, kv_cache_q8_init.rs, kv_cache_q8_memory_bytes;
 * llama-gguf 0.14.0, kv_quantized.rs, memory_usage (FP8: one byte a value).
 */
int64_t kvq_cache_bytes(int64_t layers, int64_t Hk, int64_t seq, int D, kvq_scale_mode mode);

/* Library version string. */
const char *kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */

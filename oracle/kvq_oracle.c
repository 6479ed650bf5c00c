/*
 * kvq_oracle.c -- plain, slow CPU oracle for INT8 KV-cache append and decode
 * attention.  TEST INFRASTRUCTURE ONLY: it exists to check the CUDA library,
 * and only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may load it.  It shares no code, header or constant table with the CUDA
 * library and must never be reached from the product path.
 *
 * What it follows (page title, item):
 *  - Quantize: abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
 *    CudaQuantizedKvCache::quantize_tensor -- per token, the absolute maximum
 *    is floored at 1e-8, divided by 127 to give the scale, each element is
 *    divided by the scale, rounded (Rust f32::round: half away from zero),
 *    offset by +128 and clamped to [0, 255].  The scale is kept in fp32
 *    (the page stores bf16; the fp32 reading is the one that makes
 *    dequantization use the same scale the quantizer used).
 *    abaddon 0.2.0-rc.2, src/kv_cache_quant.rs, module doc "Quantization
 *    Strategy" states the same symmetric per-token method.
 *  - Group-32 variant: realizar 0.8.5, src/cuda/executor/kv_cache_q8_init.rs,
 *    init_kv_cache_q8_gpu (one fp32 scale per 32 values along head_dim,
 *    head_dim divisible by 32) and combs-models 0.2.2, src/kv.rs,
 *    KV_QUANT_GROUP / kv_quantize.  The per-element rule is the per-token one
 *    applied to each 32-element group.
 *  - Dequantize: abaddon 0.2.0-rc.2, kv_cache_quant.rs, QuantizedKvCache::
 *    dequantize -- (u8 - 128) * scale, one fp32 multiply.
 *  - Attention: combs-models 0.2.2, src/kv.rs, attend and repeat_kv --
 *    scores = q . k * scale, softmax over the cached window, P . V; query
 *    head h reads kv head h / (Hq/Hk) (heads repeated consecutively); a
 *    single decode query attends to every cached position (no mask).
 *    Computed here in fp64 over the dequantized fp32 cache.
 *  - Chunk attention (T new queries): abaddon 0.2.0-rc.1,
 *    src/kv_cache_quant_cuda.rs, forward_attention (prefill with q_len > 1:
 *    the cache offset is seq_len - q_len and query q_pos sees the positions
 *    up to offset + q_pos) and combs-models 0.2.2, src/kv.rs, attend (a
 *    query at global position p attends the keys at positions <= p).
 *  - Sliding-window attention: combs-models 0.2.2, src/kv.rs, attend with
 *    a window w (a query at position p sees the keys p - w + 1 .. p) as
 *    PagedKVCache::sliding_attention uses it for sliding layers.
 *  - Paged layout: combs-models 0.2.2, src/kv.rs, PagedKVCache (arena
 *    [num_pages, n_kv, page_size, head_dim]; logical token g lives in
 *    physical page table[g / page_size], slot g % page_size).
 *  - Memory accounting: realizar 0.8.5, kv_cache_q8_init.rs,
 *    kv_cache_q8_memory_bytes and kv_cache_fp32_equivalent_bytes.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math.
 * On x86-64 float arithmetic is IEEE single precision (SSE), so '/' is the
 * correctly rounded fp32 quotient.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Error bits returned by the oracle's append / attention routines. */
#define ORACLE_ERR_POS 1    /* append position outside [0, capacity - T] */
#define ORACLE_ERR_PAGE 2   /* page table entry outside [0, num_pages) */
#define ORACLE_ERR_LEN 4    /* sequence length outside [0, capacity] */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static float widen_bf16(uint16_t h) {
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* One group of n consecutive bf16 values -> n offset-128 bytes + one fp32 scale. */
static void quantize_group(const uint16_t *x, int n, uint8_t *q, float *scale_out) {
    float m = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(widen_bf16(x[i]));
        if (a > m) m = a;
    }
    if (m < 1e-8f) m = 1e-8f;            /* max(|x|, 1e-8) */
    float s = m / 127.0f;                /* scale = max / 127, fp32 division */
    for (int i = 0; i < n; ++i) {
        float r = widen_bf16(x[i]) / s;  /* fp32 division */
        int v = (int)roundf(r) + 128;    /* roundf: half away from zero */
        if (v < 0) v = 0;
        if (v > 255) v = 255;
        q[i] = (uint8_t)v;
    }
    *scale_out = s;
}

/* rows x D values; group = D (per token) or 32 (group-32). */
void oracle_quantize_rows(const uint16_t *x, int64_t rows, int D, int group,
                          uint8_t *q, float *scale) {
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r)
        for (int g = 0; g < ng; ++g)
            quantize_group(x + r * D + (int64_t)g * group, group,
                           q + r * D + (int64_t)g * group, scale + r * ng + g);
}

void oracle_dequant_rows(const uint8_t *q, const float *scale, int64_t rows, int D,
                         int group, float *out) {
    int ng = D / group;
    for (int64_t r = 0; r < rows; ++r)
        for (int i = 0; i < D; ++i) {
            float s = scale[r * ng + i / group];
            out[r * D + i] = (float)((int)q[r * D + i] - 128) * s;
        }
}

/*
 * Contiguous append: new tokens x_new [B, Hk, T, D] go to positions
 * pos[b] .. pos[b]+T-1 of cache [B, Hk, max_seq, D] / scales
 * [B, Hk, max_seq, NG].  A batch row whose range leaves the capacity is
 * skipped and flagged.
 */
int oracle_append_contig(const uint16_t *x_new, int B, int Hk, int T, int D, int group,
                         const int32_t *pos, uint8_t *cache, float *scale, int max_seq) {
    int err = 0, ng = D / group;
    for (int b = 0; b < B; ++b) {
        int64_t p0 = pos[b];
        if (p0 < 0 || p0 + T > max_seq) { err |= ORACLE_ERR_POS; continue; }
        for (int h = 0; h < Hk; ++h)
            for (int t = 0; t < T; ++t) {
                const uint16_t *src = x_new + (((int64_t)b * Hk + h) * T + t) * D;
                int64_t row = ((int64_t)b * Hk + h) * max_seq + p0 + t;
                oracle_quantize_rows(src, 1, D, group, cache + row * D, scale + row * ng);
            }
    }
    return err;
}

/*
 * Paged append: logical position g of sequence b goes to physical page
 * table[b][g / page_size], slot g % page_size, arena [num_pages, Hk,
 * page_size, D].  Tokens whose page entry is invalid are skipped and
 * flagged.
 */
int oracle_append_paged(const uint16_t *x_new, int B, int Hk, int T, int D, int group,
                        const int32_t *pos, uint8_t *arena, float *scale,
                        const int32_t *table, int max_pages, int num_pages, int page_size) {
    int err = 0, ng = D / group;
    for (int b = 0; b < B; ++b) {
        int64_t p0 = pos[b];
        if (p0 < 0 || p0 + T > (int64_t)max_pages * page_size) { err |= ORACLE_ERR_POS; continue; }
        for (int t = 0; t < T; ++t) {
            int64_t g = p0 + t;
            int32_t phys = table[(int64_t)b * max_pages + g / page_size];
            int slot = (int)(g % page_size);
            if (phys < 0 || phys >= num_pages) { err |= ORACLE_ERR_PAGE; continue; }
            for (int h = 0; h < Hk; ++h) {
                const uint16_t *src = x_new + (((int64_t)b * Hk + h) * T + t) * D;
                int64_t row = ((int64_t)phys * Hk + h) * page_size + slot;
                oracle_quantize_rows(src, 1, D, group, arena + row * D, scale + row * ng);
            }
        }
    }
    return err;
}

/*
 * Decode attention for one new query per (sequence, q head) over the
 * sequence's whole cached window, in fp64 over the dequantized cache.
 *   q       bf16 [B, Hq, D]
 *   page_size == 0: contiguous k/v [B, Hk, max_seq, D], scales [B, Hk, max_seq, NG]
 *   page_size  > 0: arenas [num_pages, Hk, page_size, D], table [B, max_pages]
 *   seq_lens int32 [B]; out fp64 [B, Hq, D].  A zero length gives a zero row.
 */
int oracle_decode_attn(const uint16_t *q, int B, int Hq, int Hk, int D, int group,
                       const uint8_t *k, const uint8_t *v, const float *k_scale,
                       const float *v_scale, int max_seq, int page_size,
                       const int32_t *table, int max_pages, int num_pages,
                       const int32_t *seq_lens, double attn_scale, double *out) {
    int err = 0, ng = D / group, G = Hq / Hk;
    int64_t cap = page_size > 0 ? (int64_t)max_pages * page_size : max_seq;
    double *z = NULL, *kh = (double *)malloc(sizeof(double) * D);
    double *acc = (double *)malloc(sizeof(double) * D);
    int64_t *rows = NULL;
    for (int b = 0; b < B; ++b) {
        int64_t L = seq_lens[b];
        if (L < 0 || L > cap) { err |= ORACLE_ERR_LEN; L = 0; }
        /* physical row of each logical position (independent of kv head) */
        rows = (int64_t *)realloc(rows, sizeof(int64_t) * (L > 0 ? L : 1));
        z = (double *)realloc(z, sizeof(double) * (L > 0 ? L : 1));
        int bad = 0;
        for (int64_t t = 0; t < L; ++t) {
            if (page_size > 0) {
                int32_t phys = table[(int64_t)b * max_pages + t / page_size];
                if (phys < 0 || phys >= num_pages) { bad = 1; break; }
                rows[t] = (int64_t)phys * Hk * page_size + t % page_size; /* + h*page_size later */
            } else {
                rows[t] = (int64_t)b * Hk * max_seq + t;                   /* + h*max_seq later */
            }
        }
        if (bad) { err |= ORACLE_ERR_PAGE; L = 0; }
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            int64_t hstride = page_size > 0 ? page_size : max_seq;
            double *o = out + ((int64_t)b * Hq + h) * D;
            if (L == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
            const uint16_t *qh = q + ((int64_t)b * Hq + h) * D;
            double zmax = -INFINITY;
            for (int64_t t = 0; t < L; ++t) {
                int64_t row = rows[t] + (int64_t)hk * hstride;
                for (int d = 0; d < D; ++d) {
                    float s = k_scale[row * ng + d / group];
                    kh[d] = (double)((float)((int)k[row * D + d] - 128) * s);
                }
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += (double)widen_bf16(qh[d]) * kh[d];
                z[t] = dot * attn_scale;
                if (z[t] > zmax) zmax = z[t];
            }
            double l = 0.0;
            for (int d = 0; d < D; ++d) acc[d] = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                int64_t row = rows[t] + (int64_t)hk * hstride;
                double p = exp(z[t] - zmax);
                l += p;
                for (int d = 0; d < D; ++d) {
                    float s = v_scale[row * ng + d / group];
                    acc[d] += p * (double)((float)((int)v[row * D + d] - 128) * s);
                }
            }
            for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
        }
    }
    free(z); free(kh); free(acc); free(rows);
    return err;
}

/*
 * Attention of a chunk of T new queries per (sequence, q head) over the
 * sequence's cache, causal from the chunk's end, in fp64 over the
 * dequantized cache.  seq_lens[b] = L counts every cached token including
 * the chunk's T, so query i sits at position L - T + i and attends to the
 * positions 0 .. L - T + i.  (abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
 * forward_attention: cache_offset = seq_len - q_len, query q_pos sees KV
 * positions up to cache_offset + q_pos; combs-models 0.2.2, src/kv.rs,
 * attend: a query at global position p attends the keys at positions <= p.)
 *   q   bf16 [B, Hq, T, D]; out fp64 [B, Hq, T, D]; cache arguments as in
 *   oracle_decode_attn.  L = 0 gives zero rows; 0 < L < T (a chunk longer
 *   than the cache it sits in) is a length error and gives zero rows.
 */
int oracle_chunk_attn(const uint16_t *q, int B, int Hq, int Hk, int T, int D, int group,
                      const uint8_t *k, const uint8_t *v, const float *k_scale,
                      const float *v_scale, int max_seq, int page_size,
                      const int32_t *table, int max_pages, int num_pages,
                      const int32_t *seq_lens, double attn_scale, double *out) {
    int err = 0, ng = D / group, G = Hq / Hk;
    int64_t cap = page_size > 0 ? (int64_t)max_pages * page_size : max_seq;
    double *z = NULL, *kh = (double *)malloc(sizeof(double) * D);
    double *acc = (double *)malloc(sizeof(double) * D);
    int64_t *rows = NULL;
    for (int b = 0; b < B; ++b) {
        int64_t L = seq_lens[b];
        if (L < 0 || L > cap || (L > 0 && L < T)) { err |= ORACLE_ERR_LEN; L = 0; }
        rows = (int64_t *)realloc(rows, sizeof(int64_t) * (L > 0 ? L : 1));
        z = (double *)realloc(z, sizeof(double) * (L > 0 ? L : 1));
        int bad = 0;
        for (int64_t t = 0; t < L; ++t) {
            if (page_size > 0) {
                int32_t phys = table[(int64_t)b * max_pages + t / page_size];
                if (phys < 0 || phys >= num_pages) { bad = 1; break; }
                rows[t] = (int64_t)phys * Hk * page_size + t % page_size;
            } else {
                rows[t] = (int64_t)b * Hk * max_seq + t;
            }
        }
        if (bad) { err |= ORACLE_ERR_PAGE; L = 0; }
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            int64_t hstride = page_size > 0 ? page_size : max_seq;
            for (int i = 0; i < T; ++i) {
                double *o = out + (((int64_t)b * Hq + h) * T + i) * D;
                if (L == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
                const uint16_t *qh = q + (((int64_t)b * Hq + h) * T + i) * D;
                int64_t visible = L - T + i + 1;          /* positions 0 .. L - T + i */
                double zmax = -INFINITY;
                for (int64_t t = 0; t < visible; ++t) {
                    int64_t row = rows[t] + (int64_t)hk * hstride;
                    for (int d = 0; d < D; ++d) {
                        float s = k_scale[row * ng + d / group];
                        kh[d] = (double)((float)((int)k[row * D + d] - 128) * s);
                    }
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += (double)widen_bf16(qh[d]) * kh[d];
                    z[t] = dot * attn_scale;
                    if (z[t] > zmax) zmax = z[t];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) acc[d] = 0.0;
                for (int64_t t = 0; t < visible; ++t) {
                    int64_t row = rows[t] + (int64_t)hk * hstride;
                    double p = exp(z[t] - zmax);
                    l += p;
                    for (int d = 0; d < D; ++d) {
                        float s = v_scale[row * ng + d / group];
                        acc[d] += p * (double)((float)((int)v[row * D + d] - 128) * s);
                    }
                }
                for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
            }
        }
    }
    free(z); free(kh); free(acc); free(rows);
    return err;
}

/*
 * Bytes of an INT8 cache: layers * 2 (K and V) * (values + scales), with one
 * byte per value and scale_bytes per scale (4 for fp32), as in
 * kv_cache_q8_memory_bytes; group = values per scale.
 */
int64_t oracle_cache_bytes(int64_t layers, int64_t Hk, int64_t seq, int64_t D, int64_t group,
                           int64_t scale_bytes) {
    int64_t values = Hk * seq * D;
    int64_t scales = Hk * seq * (D / group);
    return layers * 2 * (values + scales * scale_bytes);
}

/* fp32 equivalent, as in kv_cache_fp32_equivalent_bytes. */
int64_t oracle_fp32_cache_bytes(int64_t layers, int64_t Hk, int64_t seq, int64_t D) {
    return layers * 2 * Hk * seq * D * 4;
}

/*
 * Sliding-window attention of T queries per (sequence, q head) over the
 * dequantized cache, in fp64: query i sits at position p = L - T + i (L
 * counts the chunk's T tokens; T = 1 is a decode step) and attends to the
 * positions max(0, p - window + 1) .. p -- the causal mask with the window
 * rule of combs-models 0.2.2, src/kv.rs, attend (a key at position k is
 * forbidden when k > p or when k + window - 1 < p) as the sliding layers of
 * PagedKVCache::sliding_attention use it.  window >= 1; the cache arguments
 * are those of oracle_decode_attn.  L = 0 gives zero rows; 0 < L < T is a
 * length error (zero rows).
 */
int oracle_window_attn(const uint16_t *q, int B, int Hq, int Hk, int T, int D, int group,
                       const uint8_t *k, const uint8_t *v, const float *k_scale,
                       const float *v_scale, int max_seq, int page_size,
                       const int32_t *table, int max_pages, int num_pages,
                       const int32_t *seq_lens, int window, double attn_scale, double *out) {
    int err = 0, ng = D / group, G = Hq / Hk;
    int64_t cap = page_size > 0 ? (int64_t)max_pages * page_size : max_seq;
    double *z = NULL, *kh = (double *)malloc(sizeof(double) * D);
    double *acc = (double *)malloc(sizeof(double) * D);
    int64_t *rows = NULL;
    for (int b = 0; b < B; ++b) {
        int64_t L = seq_lens[b];
        if (L < 0 || L > cap || (L > 0 && L < T)) { err |= ORACLE_ERR_LEN; L = 0; }
        rows = (int64_t *)realloc(rows, sizeof(int64_t) * (L > 0 ? L : 1));
        z = (double *)realloc(z, sizeof(double) * (L > 0 ? L : 1));
        int bad = 0;
        for (int64_t t = 0; t < L; ++t) {
            if (page_size > 0) {
                int32_t phys = table[(int64_t)b * max_pages + t / page_size];
                if (phys < 0 || phys >= num_pages) { bad = 1; break; }
                rows[t] = (int64_t)phys * Hk * page_size + t % page_size;
            } else {
                rows[t] = (int64_t)b * Hk * max_seq + t;
            }
        }
        if (bad) { err |= ORACLE_ERR_PAGE; L = 0; }
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            int64_t hstride = page_size > 0 ? page_size : max_seq;
            for (int i = 0; i < T; ++i) {
                double *o = out + (((int64_t)b * Hq + h) * T + i) * D;
                if (L == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
                const uint16_t *qh = q + (((int64_t)b * Hq + h) * T + i) * D;
                int64_t p = L - T + i;                      /* the query's position */
                int64_t first = p - window + 1;             /* oldest key the window keeps */
                if (first < 0) first = 0;
                double zmax = -INFINITY;
                for (int64_t t = first; t <= p; ++t) {
                    int64_t row = rows[t] + (int64_t)hk * hstride;
                    for (int d = 0; d < D; ++d) {
                        float s = k_scale[row * ng + d / group];
                        kh[d] = (double)((float)((int)k[row * D + d] - 128) * s);
                    }
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += (double)widen_bf16(qh[d]) * kh[d];
                    z[t] = dot * attn_scale;
                    if (z[t] > zmax) zmax = z[t];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) acc[d] = 0.0;
                for (int64_t t = first; t <= p; ++t) {
                    int64_t row = rows[t] + (int64_t)hk * hstride;
                    double e = exp(z[t] - zmax);
                    l += e;
                    for (int d = 0; d < D; ++d) {
                        float s = v_scale[row * ng + d / group];
                        acc[d] += e * (double)((float)((int)v[row * D + d] - 128) * s);
                    }
                }
                for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
            }
        }
    }
    free(z); free(kh); free(acc); free(rows);
    return err;
}

/*
 * FP8 KV format: every value is stored as one FP8 byte and there is no
 * scale.  llama-gguf 0.14.0, src/model/kv_quantized.rs, KVCacheFormat::
 * Fp8E4M3 / Fp8E5M2 with quantize_fp8_e4m3 / quantize_fp8_e5m2 and their
 * dequantize_* counterparts.  fmt 0 = E4M3 (4 exponent bits, bias 7, 3
 * mantissa bits), fmt 1 = E5M2 (5 exponent bits, bias 15, 2 mantissa bits).
 *
 * The page's encoders TRUNCATE: the mantissa bits below the format's are
 * dropped (toward zero), numbers below the smallest subnormal become a zero
 * of their sign, and an exponent above the format's range saturates (E4M3:
 * to +-448, code 0x7E; E5M2: to +-inf, code 0x7C).  Two readings where the
 * page's code disagrees with its own decoders: an E4M3 value in [480, 512)
 * would get exponent 15 and mantissa 7, the NaN pattern of the page's
 * decoder, so it saturates to 0x7E like the larger ones; an E5M2 value in
 * [2^16, 2^17) would get exponent 31, the inf/NaN patterns, so it encodes as
 * inf (0x7C) like the larger ones.  +-0 encodes as 0x00; non-finite inputs
 * follow the page (NaN -> 0xFF, E4M3 inf -> 0x7F / 0xFF, E5M2 inf -> 0x7C /
 * 0xFC).
 */
uint8_t oracle_fp8_encode(float x, int fmt) {
    const int ebits = fmt ? 5 : 4, mbits = fmt ? 2 : 3, bias = fmt ? 15 : 7;
    const int emax = (1 << ebits) - 1;                     /* 15 or 31 */
    if (isnan(x)) return 0xFF;
    if (isinf(x)) return fmt ? (x > 0 ? 0x7C : 0xFC) : (x > 0 ? 0x7F : 0xFF);
    if (x == 0.0f) return 0x00;
    uint32_t bits;
    memcpy(&bits, &x, sizeof bits);
    const uint8_t sign = (uint8_t)(bits >> 31);
    const int e = (int)((bits >> 23) & 0xFF) - 127;        /* unbiased binary32 exponent */
    uint32_t sig = bits & 0x7FFFFF;
    if (e != -127) sig |= 0x800000;                         /* the implicit one, bit 23 */
    const int E = e + bias;                                 /* biased FP8 exponent */
    const uint8_t top = (uint8_t)(sign << 7);
    if (fmt == 0) {
        if (E > emax) return top | 0x7E;                    /* saturate: 448 */
    } else {
        if (E > emax - 1) return top | 0x7C;                /* inf (reading for E = 31) */
    }
    if (E <= 0) {
        const int keep = mbits + E;                         /* significand bits a subnormal keeps */
        if (keep <= 0) return top;                          /* below the smallest subnormal */
        return top | (uint8_t)(sig >> (24 - keep));         /* truncated subnormal mantissa */
    }
    uint8_t mant = (uint8_t)((sig >> (23 - mbits)) & ((1u << mbits) - 1));
    uint8_t code = top | (uint8_t)(E << mbits) | mant;
    if (fmt == 0 && (code & 0x7F) == 0x7F) code = top | 0x7E;   /* reading: not the NaN code */
    return code;
}

/* The exact value of an FP8 byte (the page's dequantize_fp8_*). */
float oracle_fp8_decode(uint8_t c, int fmt) {
    const int mbits = fmt ? 2 : 3, bias = fmt ? 15 : 7;
    const uint8_t mag = c & 0x7F;
    const float sgn = (c & 0x80) ? -1.0f : 1.0f;
    if (mag == 0) return 0.0f;
    if (fmt == 0 && mag == 0x7F) return NAN;
    if (fmt == 1 && mag == 0x7C) return sgn * INFINITY;
    if (fmt == 1 && mag > 0x7C) return NAN;
    const int E = mag >> mbits, M = mag & ((1 << mbits) - 1);
    if (E == 0) return sgn * ldexpf((float)M, 1 - bias - mbits);       /* M * 2^(1-bias-mbits) */
    return sgn * ldexpf((float)((1 << mbits) + M), E - bias - mbits);  /* 1.M * 2^(E-bias) */
}

void oracle_fp8_encode_rows(const uint16_t *x, int64_t n, int fmt, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_fp8_encode(widen_bf16(x[i]), fmt);
}

/*
 * Append of new tokens x_new [B, Hk, T, D] to an FP8 cache: contiguous
 * [B, Hk, max_seq, D] (page_size 0) or a paged arena [num_pages, Hk,
 * page_size, D] with table [B, max_pages]; positions and flags as in
 * oracle_append_contig / oracle_append_paged.
 */
int oracle_append_fp8(const uint16_t *x_new, int B, int Hk, int T, int D, int fmt,
                      const int32_t *pos, uint8_t *dst, int max_seq, int page_size,
                      const int32_t *table, int max_pages, int num_pages) {
    int err = 0;
    for (int b = 0; b < B; ++b) {
        int64_t p0 = pos[b];
        int64_t cap = page_size > 0 ? (int64_t)max_pages * page_size : max_seq;
        if (p0 < 0 || p0 + T > cap) { err |= ORACLE_ERR_POS; continue; }
        for (int t = 0; t < T; ++t) {
            int64_t g = p0 + t;
            for (int h = 0; h < Hk; ++h) {
                int64_t row;
                if (page_size > 0) {
                    int32_t phys = table[(int64_t)b * max_pages + g / page_size];
                    if (phys < 0 || phys >= num_pages) { err |= ORACLE_ERR_PAGE; continue; }
                    row = ((int64_t)phys * Hk + h) * page_size + g % page_size;
                } else {
                    row = ((int64_t)b * Hk + h) * max_seq + g;
                }
                oracle_fp8_encode_rows(x_new + (((int64_t)b * Hk + h) * T + t) * D, D, fmt,
                                       dst + row * D);
            }
        }
    }
    return err;
}

/*
 * Attention over an FP8 cache in fp64, k-hat / v-hat the exact values of the
 * bytes: T queries per (sequence, q head), query i at position p = L - T + i
 * attending to positions max(0, p - window + 1) .. p (window 0: 0 .. p; T = 1
 * with window 0 is a decode step over the whole cache).  Cache and length
 * arguments as in oracle_window_attn, without scales.
 */
int oracle_fp8_attn(const uint16_t *q, int B, int Hq, int Hk, int T, int D, int fmt,
                    const uint8_t *k, const uint8_t *v, int max_seq, int page_size,
                    const int32_t *table, int max_pages, int num_pages,
                    const int32_t *seq_lens, int window, double attn_scale, double *out) {
    int err = 0, G = Hq / Hk;
    int64_t cap = page_size > 0 ? (int64_t)max_pages * page_size : max_seq;
    double *z = NULL, *kh = (double *)malloc(sizeof(double) * D);
    double *acc = (double *)malloc(sizeof(double) * D);
    int64_t *rows = NULL;
    for (int b = 0; b < B; ++b) {
        int64_t L = seq_lens[b];
        if (L < 0 || L > cap || (L > 0 && L < T)) { err |= ORACLE_ERR_LEN; L = 0; }
        rows = (int64_t *)realloc(rows, sizeof(int64_t) * (L > 0 ? L : 1));
        z = (double *)realloc(z, sizeof(double) * (L > 0 ? L : 1));
        int bad = 0;
        for (int64_t t = 0; t < L; ++t) {
            if (page_size > 0) {
                int32_t phys = table[(int64_t)b * max_pages + t / page_size];
                if (phys < 0 || phys >= num_pages) { bad = 1; break; }
                rows[t] = (int64_t)phys * Hk * page_size + t % page_size;
            } else {
                rows[t] = (int64_t)b * Hk * max_seq + t;
            }
        }
        if (bad) { err |= ORACLE_ERR_PAGE; L = 0; }
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            int64_t hstride = page_size > 0 ? page_size : max_seq;
            for (int i = 0; i < T; ++i) {
                double *o = out + (((int64_t)b * Hq + h) * T + i) * D;
                if (L == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
                const uint16_t *qh = q + (((int64_t)b * Hq + h) * T + i) * D;
                int64_t p = L - T + i;
                int64_t first = window > 0 ? p - window + 1 : 0;
                if (first < 0) first = 0;
                double zmax = -INFINITY;
                for (int64_t t = first; t <= p; ++t) {
                    int64_t row = rows[t] + (int64_t)hk * hstride;
                    for (int d = 0; d < D; ++d) kh[d] = (double)oracle_fp8_decode(k[row * D + d], fmt);
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += (double)widen_bf16(qh[d]) * kh[d];
                    z[t] = dot * attn_scale;
                    if (z[t] > zmax) zmax = z[t];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) acc[d] = 0.0;
                for (int64_t t = first; t <= p; ++t) {
                    int64_t row = rows[t] + (int64_t)hk * hstride;
                    double e = exp(z[t] - zmax);
                    l += e;
                    for (int d = 0; d < D; ++d)
                        acc[d] += e * (double)oracle_fp8_decode(v[row * D + d], fmt);
                }
                for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
            }
        }
    }
    free(z); free(kh); free(acc); free(rows);
    return err;
}

/*
 * Per-head and per-channel scales (abaddon 0.2.0-rc.1,
 * src/kv_cache_quant_cuda.rs, QuantGranularity::PerHead / PerChannel,
 * OptimizedQuantizedKvCache::quantize_with_granularity): one fp32 scale per
 * (sequence, kv head) -- the page's shape (batch, heads, 1, 1) -- or one per
 * (sequence, kv head, channel) -- (batch, heads, 1, head_dim).  A calibrating
 * call sets them from all the tokens it quantises: m = max |x| over the
 * call's tokens and head_dim (per head) or over its tokens (per channel),
 * floored at 1e-8, s = m / 127.  Reading: the page concatenates a later
 * call's scales along the token axis, which its own dequantise cannot
 * broadcast against the tokens, so a sequence keeps the scales of its
 * calibrating call and later calls quantise with them.  Every value is then
 * quantised with the per-token rule (round(x / s) + 128, half away from
 * zero, clamped to [0, 255]; values beyond the calibrated range clamp).
 *   gran 1 = per head (NS = 1 scale), gran 2 = per channel (NS = D scales).
 *   x_new [B, Hk, T, D] bf16; cache [B, Hk, max_seq, D] at pos[b];
 *   scales [B, Hk, NS], read (calibrate == 0) or written (calibrate == 1).
 */
int oracle_append_static(const uint16_t *x_new, int B, int Hk, int T, int D, int gran,
                         int calibrate, const int32_t *pos, uint8_t *cache, float *scales,
                         int max_seq) {
    int err = 0, ns = gran == 1 ? 1 : D;
    for (int b = 0; b < B; ++b) {
        int64_t p0 = pos[b];
        if (p0 < 0 || p0 + T > max_seq) { err |= ORACLE_ERR_POS; continue; }
        for (int h = 0; h < Hk; ++h) {
            const uint16_t *x = x_new + ((int64_t)b * Hk + h) * T * D;
            float *s = scales + ((int64_t)b * Hk + h) * ns;
            if (calibrate) {
                for (int c = 0; c < ns; ++c) {
                    float m = 0.0f;
                    for (int t = 0; t < T; ++t)
                        for (int d = 0; d < D; ++d) {
                            if (ns > 1 && d != c) continue;
                            float a = fabsf(widen_bf16(x[(int64_t)t * D + d]));
                            if (a > m) m = a;
                        }
                    if (m < 1e-8f) m = 1e-8f;
                    s[c] = m / 127.0f;
                }
            }
            for (int t = 0; t < T; ++t)
                for (int d = 0; d < D; ++d) {
                    float r = widen_bf16(x[(int64_t)t * D + d]) / s[ns > 1 ? d : 0];
                    int v = (int)roundf(r) + 128;
                    if (v < 0) v = 0;
                    if (v > 255) v = 255;
                    cache[(((int64_t)b * Hk + h) * max_seq + p0 + t) * D + d] = (uint8_t)v;
                }
        }
    }
    return err;
}

/*
 * Attention over a contiguous INT8 cache with per-head / per-channel scales
 * (k-hat = (byte - 128) * s[channel or 0], one fp32 multiply), in fp64: T
 * queries per (sequence, q head), causal from the chunk's end, with an
 * optional sliding window (window 0: none), as in oracle_fp8_attn.
 *   k_scales, v_scales [B, Hk, NS].
 */
int oracle_static_attn(const uint16_t *q, int B, int Hq, int Hk, int T, int D, int gran,
                       const uint8_t *k, const uint8_t *v, const float *k_scales,
                       const float *v_scales, int max_seq, const int32_t *seq_lens, int window,
                       double attn_scale, double *out) {
    int err = 0, G = Hq / Hk, ns = gran == 1 ? 1 : D;
    double *z = NULL, *kh = (double *)malloc(sizeof(double) * D);
    double *acc = (double *)malloc(sizeof(double) * D);
    for (int b = 0; b < B; ++b) {
        int64_t L = seq_lens[b];
        if (L < 0 || L > max_seq || (L > 0 && L < T)) { err |= ORACLE_ERR_LEN; L = 0; }
        z = (double *)realloc(z, sizeof(double) * (L > 0 ? L : 1));
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            const float *sk = k_scales + ((int64_t)b * Hk + hk) * ns;
            const float *sv = v_scales + ((int64_t)b * Hk + hk) * ns;
            for (int i = 0; i < T; ++i) {
                double *o = out + (((int64_t)b * Hq + h) * T + i) * D;
                if (L == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
                const uint16_t *qh = q + (((int64_t)b * Hq + h) * T + i) * D;
                int64_t p = L - T + i;
                int64_t first = window > 0 ? p - window + 1 : 0;
                if (first < 0) first = 0;
                double zmax = -INFINITY;
                for (int64_t t = first; t <= p; ++t) {
                    int64_t row = ((int64_t)b * Hk + hk) * max_seq + t;
                    for (int d = 0; d < D; ++d)
                        kh[d] = (double)((float)((int)k[row * D + d] - 128) * sk[ns > 1 ? d : 0]);
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d) dot += (double)widen_bf16(qh[d]) * kh[d];
                    z[t] = dot * attn_scale;
                    if (z[t] > zmax) zmax = z[t];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d) acc[d] = 0.0;
                for (int64_t t = first; t <= p; ++t) {
                    int64_t row = ((int64_t)b * Hk + hk) * max_seq + t;
                    double e = exp(z[t] - zmax);
                    l += e;
                    for (int d = 0; d < D; ++d)
                        acc[d] += e * (double)((float)((int)v[row * D + d] - 128) * sv[ns > 1 ? d : 0]);
                }
                for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
            }
        }
    }
    free(z); free(kh); free(acc);
    return err;
}

/* INT8 value of byte q at (row, d) for the INT8 modes of the mixed cache:
 * mode 0 per token (scales [rows]), 1 group-32 ([rows, D/32]), 3 per head and
 * 4 per channel (static scales of the (sequence, kv head): 1 or D floats). */
static float mixed_int8_value(int mode, const uint8_t *q, const float *scales, int64_t row,
                              int64_t unit, int D, int d) {
    float s;
    if (mode == 0) s = scales[row];
    else if (mode == 1) s = scales[row * (D / 32) + d / 32];
    else if (mode == 3) s = scales[unit];
    else s = scales[unit * D + d];
    return (float)((int)q[row * D + d] - 128) * s;
}

/*
 * Mixed cache (abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
 * DynamicQuantConfig::unquantized_window, OptimizedQuantizedKvCache::append
 * and get_kv): the newest W tokens of a sequence stay unquantised (bf16) and
 * the older ones are INT8.  An append adds the new tokens to the recent
 * window; when the window holds more than W tokens the oldest ones are
 * quantised (per the cache's INT8 mode) and move to the INT8 part, so after
 * any append the INT8 part holds positions 0 .. L - W - 1 and the window the
 * last min(L, W).  Layout: the INT8 part is a contiguous cache [B, Hk,
 * max_seq, D] with its scales (mode 0: [B, Hk, max_seq, 1]; 1: [B, Hk,
 * max_seq, D/32]; 3 / 4: static [B, Hk, 1 or D], read, set earlier by a
 * calibrating call); the window is a ring [B, Hk, W, D] of bf16 in which
 * position g sits in row g % W.
 *   x_new [B, Hk, T, D]; lens_old [B] = L before the append.
 */
int oracle_append_mixed(const uint16_t *x_new, int B, int Hk, int T, int D, int mode,
                        const int32_t *lens_old, uint8_t *cache, float *scales,
                        uint16_t *ring, int W, int max_seq) {
    int err = 0, ng = mode == 1 ? D / 32 : 1, ns = mode == 4 ? D : 1;
    for (int b = 0; b < B; ++b) {
        int64_t L0 = lens_old[b], L1 = L0 + T;
        if (L0 < 0 || L1 > max_seq) { err |= ORACLE_ERR_POS; continue; }
        int64_t q0 = L0 > W ? L0 - W : 0;                  /* INT8 part before */
        int64_t q1 = L1 > W ? L1 - W : 0;                  /* and after */
        for (int h = 0; h < Hk; ++h) {
            int64_t unit = (int64_t)b * Hk + h;
            /* quantise positions q0 .. q1 - 1, oldest first, from the window
             * (older than this call) or from the new tokens */
            for (int64_t g = q0; g < q1; ++g) {
                const uint16_t *src = g < L0 ? ring + (unit * W + g % W) * D
                                             : x_new + (unit * T + (g - L0)) * D;
                int64_t row = unit * max_seq + g;
                if (mode == 0 || mode == 1) {
                    oracle_quantize_rows(src, 1, D, mode == 0 ? D : 32, cache + row * D,
                                         scales + row * ng);
                } else {
                    const float *s = scales + unit * ns;
                    for (int d = 0; d < D; ++d) {
                        float r = widen_bf16(src[d]) / s[ns > 1 ? d : 0];
                        int v = (int)roundf(r) + 128;
                        if (v < 0) v = 0;
                        if (v > 255) v = 255;
                        cache[row * D + d] = (uint8_t)v;
                    }
                }
            }
            /* the new tokens that stay in the window */
            for (int64_t g = (q1 > L0 ? q1 : L0); g < L1; ++g)
                memcpy(ring + (unit * W + g % W) * D, x_new + (unit * T + (g - L0)) * D,
                       sizeof(uint16_t) * D);
        }
    }
    return err;
}

/*
 * Decode attention over a mixed cache in fp64 (one query per (sequence, q
 * head) at the newest position, no mask): positions 0 .. L - W - 1 from the
 * INT8 part (dequantised per mode), the rest from the bf16 window ring.
 */
int oracle_mixed_attn(const uint16_t *q, int B, int Hq, int Hk, int D, int mode,
                      const uint8_t *k, const uint8_t *v, const float *k_scales,
                      const float *v_scales, const uint16_t *rk, const uint16_t *rv, int W,
                      int max_seq, const int32_t *seq_lens, double attn_scale, double *out) {
    int err = 0, G = Hq / Hk;
    double *z = NULL, *kh = (double *)malloc(sizeof(double) * D);
    double *acc = (double *)malloc(sizeof(double) * D);
    for (int b = 0; b < B; ++b) {
        int64_t L = seq_lens[b];
        if (L < 0 || L > max_seq) { err |= ORACLE_ERR_LEN; L = 0; }
        int64_t Lq = L > W ? L - W : 0;
        z = (double *)realloc(z, sizeof(double) * (L > 0 ? L : 1));
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            int64_t unit = (int64_t)b * Hk + hk;
            double *o = out + ((int64_t)b * Hq + h) * D;
            if (L == 0) { for (int d = 0; d < D; ++d) o[d] = 0.0; continue; }
            const uint16_t *qh = q + ((int64_t)b * Hq + h) * D;
            double zmax = -INFINITY;
            for (int64_t t = 0; t < L; ++t) {
                for (int d = 0; d < D; ++d)
                    kh[d] = t < Lq ? (double)mixed_int8_value(mode, k, k_scales,
                                                              unit * max_seq + t, unit, D, d)
                                   : (double)widen_bf16(rk[(unit * W + t % W) * D + d]);
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += (double)widen_bf16(qh[d]) * kh[d];
                z[t] = dot * attn_scale;
                if (z[t] > zmax) zmax = z[t];
            }
            double l = 0.0;
            for (int d = 0; d < D; ++d) acc[d] = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                double e = exp(z[t] - zmax);
                l += e;
                for (int d = 0; d < D; ++d)
                    acc[d] += e * (t < Lq ? (double)mixed_int8_value(mode, v, v_scales,
                                                                     unit * max_seq + t, unit, D, d)
                                          : (double)widen_bf16(rv[(unit * W + t % W) * D + d]));
            }
            for (int d = 0; d < D; ++d) o[d] = acc[d] / l;
        }
    }
    free(z); free(kh); free(acc);
    return err;
}

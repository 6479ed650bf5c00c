// kvq_api.cu -- the extern "C" entry points declared in include/kvq.h:
// argument validation, split planning and kernel launches.  No allocation,
// no host<->device copies and no synchronisation happen here, except in
// kvq_read_error, whose job is to read the device error word.
#include <stdint.h>

#include <atomic>
#include <cstdint>

#include "kvq_internal.cuh"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

constexpr int kMaxSplits = 4096;     // bound on splits per sequence (combine smem)

kvq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

// SM count of the current device, read once per device (a device's SM count
// does not change while the process runs; the attribute query costs more
// than the rest of a call's host work)
constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];

bool current_sms(int* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (dev >= 0 && dev < kMaxDevices) {
        const int c = g_sms[dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *out = c;
            return true;
        }
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return false;
    if (dev >= 0 && dev < kMaxDevices) g_sms[dev].store(sms, std::memory_order_relaxed);
    *out = sms;
    return true;
}

bool valid_mode(kvq_scale_mode m) {
    return m == KVQ_SCALE_PER_TOKEN || m == KVQ_SCALE_GROUP32 || m == KVQ_FP8_E4M3 ||
           m == KVQ_FP8_E5M2 || m == KVQ_SCALE_PER_HEAD || m == KVQ_SCALE_PER_CHANNEL;
}
bool is_static(kvq_scale_mode m) { return m == KVQ_SCALE_PER_HEAD || m == KVQ_SCALE_PER_CHANNEL; }
// scales per (sequence, kv head) of the per-head / per-channel modes (0: per row)
int static_ns(kvq_scale_mode m, int D) {
    return m == KVQ_SCALE_PER_HEAD ? 1 : m == KVQ_SCALE_PER_CHANNEL ? D : 0;
}
bool is_fp8(kvq_scale_mode m) { return m == KVQ_FP8_E4M3 || m == KVQ_FP8_E5M2; }
// 0: INT8 with scales, 1: E4M3, 2: E5M2 (the kernels' encoding)
int fp8_code(kvq_scale_mode m) { return m == KVQ_FP8_E4M3 ? 1 : m == KVQ_FP8_E5M2 ? 2 : 0; }

kvq_status check_append_common(const uint16_t* k_new, const uint16_t* v_new, int B, int Hk, int T,
                               int D, kvq_scale_mode mode, const int32_t* d_pos,
                               const void* kd, const void* vd, const float* ks,
                               const float* vs, const int32_t* d_err) {
    if (!valid_mode(mode)) return KVQ_ERR_INVALID_ARG;
    const bool scaled = !is_fp8(mode);                 // FP8 modes have no scale arrays
    if (!k_new || !v_new || !d_pos || !kd || !vd || (scaled && (!ks || !vs)))
        return KVQ_ERR_INVALID_ARG;
    if (B < 1 || Hk < 1 || T < 1 || D < 16 || D > 256 || (D % 16) != 0) return KVQ_ERR_INVALID_ARG;
    if (mode == KVQ_SCALE_GROUP32 && (D % 32) != 0) return KVQ_ERR_INVALID_ARG;
    // per-head scales are read one float at a time: 4-byte alignment suffices
    const uintptr_t sa = mode == KVQ_SCALE_PER_HEAD ? 4 : 16;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(kd, 16) || !aligned(vd, 16) ||
        !aligned(ks, sa) || !aligned(vs, sa) || !aligned(d_pos, 4) || !aligned(d_err, 4))
        return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
}

kvq_status plan(int B, int Hk, int hint, int num_splits, int num_sms, int* chunk_out,
                int* splits_out) {
    if (B < 0 || Hk < 1 || hint < 0 || num_splits < 0) return KVQ_ERR_INVALID_ARG;
    if (num_sms <= 0 && !current_sms(&num_sms)) return KVQ_ERR_CUDA;
    int64_t chunk;
    if (hint <= 16) {
        chunk = 16;
    } else if (num_splits > 0) {
        const int64_t s = num_splits < ceil_div(hint, 16) ? num_splits : ceil_div(hint, 16);
        chunk = ceil_div(ceil_div(hint, s), 16) * 16;
    } else {
        // Few (sequence, kv head) units: one chunk per CTA, units * per_unit <=
        // #SM chunks of equal length.  Many units: 128-token chunks (one
        // stage), so that the contiguous item blocks of the persistent CTAs
        // hold equal numbers of stages whatever the length mix.
        const int64_t units = static_cast<int64_t>(B > 0 ? B : 1) * Hk;
        const int64_t per_unit = num_sms / units;
        if (per_unit >= 8) {
            // a short sequence (at most four 128-token stages, which the CTA's
            // two consumer groups take in two rounds) stays one chunk: its
            // CTA writes the final rows, and no combine launch follows, which
            // costs more than the stages that splitting would spread
            chunk = hint <= 4 * 128 ? ceil_div(hint, 16) * 16
                                    : ceil_div(ceil_div(hint, per_unit), 16) * 16;
        } else {
            chunk = 128;
        }
        const int64_t cap = ceil_div(hint, 16) * 16;
        if (chunk > cap) chunk = cap;
    }
    if (ceil_div(hint, chunk) > kMaxSplits) chunk = ceil_div(ceil_div(hint, kMaxSplits), 16) * 16;
    int64_t splits = ceil_div(hint, chunk);
    if (splits < 1) splits = 1;
    *chunk_out = static_cast<int>(chunk);
    *splits_out = static_cast<int>(splits);
    return KVQ_OK;
}

// [o: n_part * D][m: n_part][l: n_part] floats
size_t workspace_for(int B, int Hq, int D, int splits) {
    if (splits <= 1) return 0;
    return static_cast<size_t>(B) * Hq * splits * (D + 2) * sizeof(float);
}

// Decode (T = 1) and chunk (T > 1) attention: the T queries of a (sequence,
// q head) ride as T rows of the GQA group, so the split kernel sees Hq * T
// heads, G * T per kv head, and masks each row causally.
// The longest run of tokens a sequence's queries walk: everything up to the
// hint, or with a sliding window at most T + window - 1 positions plus the
// up-to-15 below the window that its 16-aligned base adds.
int walked_hint(int hint, int T, int window) {
    if (window <= 0) return hint;
    const int64_t w = static_cast<int64_t>(window) + T - 1 + 15;
    return w < hint ? static_cast<int>(w) : hint;
}

// mixed cache: split-K slots for every row even without a split (the
// window kernel folds them)
size_t mixed_workspace_for(int B, int Hq, int D, int splits) {
    return static_cast<size_t>(B) * Hq * (splits > 1 ? splits : 1) * (D + 2) * sizeof(float);
}

kvq_status attend(const uint16_t* q, int B, int Hq, int Hk, int T, int D, kvq_scale_mode mode,
                  const kvq_cache_view* kv, const int32_t* d_seq_lens, int max_seq_len_hint,
                  int window, float attn_scale, float* out, void* workspace,
                  size_t workspace_bytes, int num_splits, int32_t* d_err, kvq_stream_t stream,
                  int recent = 0, const uint16_t* rk = nullptr, const uint16_t* rv = nullptr,
                  const uint16_t* k_new = nullptr, const uint16_t* v_new = nullptr) {
    if (window < 0 || recent < 0) return KVQ_ERR_INVALID_ARG;
    if (!valid_mode(mode)) return KVQ_ERR_INVALID_ARG;
    if (!q || !kv || !kv->k || !kv->v || !d_seq_lens || !out) return KVQ_ERR_INVALID_ARG;
    if (!is_fp8(mode) && (!kv->k_scale || !kv->v_scale)) return KVQ_ERR_INVALID_ARG;
    if (B < 0 || Hq < 1 || Hk < 1 || (Hq % Hk) != 0 || D < 16 || (D % 16) != 0 ||
        max_seq_len_hint < 0 || num_splits < 0 || B > 65535 || Hk > 65535)
        return KVQ_ERR_INVALID_ARG;
    if (mode == KVQ_SCALE_GROUP32 && (D % 32) != 0) return KVQ_ERR_INVALID_ARG;
    if (kv->page_size == 16) {
        if (!kv->page_table || !aligned(kv->page_table, 4) || kv->max_pages < 1 ||
            kv->num_pages < 1)
            return KVQ_ERR_INVALID_ARG;
    } else if (kv->page_size == 0) {
        if (kv->max_seq < 1) return KVQ_ERR_INVALID_ARG;
    } else {
        return KVQ_ERR_INVALID_ARG;
    }
    const uintptr_t sa = mode == KVQ_SCALE_PER_HEAD ? 4 : 16;   // per-head: scalar reads
    if (!aligned(q, 16) || !aligned(kv->k, 16) || !aligned(kv->v, 16) ||
        !aligned(kv->k_scale, sa) || !aligned(kv->v_scale, sa) || !aligned(d_seq_lens, 4) ||
        !aligned(out, 16) || !aligned(workspace, 16) || !aligned(d_err, 4))
        return KVQ_ERR_INVALID_ARG;
    if (Hq > 65535) return KVQ_ERR_UNSUPPORTED;
    // more than 16 (head, query) rows per kv head: the dense chunk kernel on
    // the tcgen05 tensor cores where it covers the shape (otherwise the
    // CUDA-core split kernel below)
    const bool dense = static_cast<int64_t>(Hq / Hk) * T > 16;
    if (dense && !k_new &&
        kvq::chunk_tc_supported(D, Hq / Hk, T, mode == KVQ_SCALE_GROUP32, is_fp8(mode),
                                static_ns(mode, D), kv->page_size, window, recent)) {
        if (static_cast<int64_t>(B) * Hq * T >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
        if (B == 0) return KVQ_OK;
        if (static_cast<int64_t>(B) * Hk * kv->max_seq >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
        kvq::DecodeParams p{};
        p.q = q; p.k = kv->k; p.v = kv->v; p.k_scale = kv->k_scale; p.v_scale = kv->v_scale;
        p.seq_lens = d_seq_lens; p.out = out; p.d_err = d_err;
        p.B = B; p.Hk = Hk; p.D = D; p.max_seq = kv->max_seq;
        p.scale_log2 = attn_scale * 1.4426950408889634f;
        return from_cuda(kvq::launch_chunk_tc(p, Hq, Hq / Hk, T, static_cast<cudaStream_t>(stream)));
    }
    if (static_cast<int64_t>(Hq / Hk) * T > (1ll << 19)) return KVQ_ERR_UNSUPPORTED;
    const int G = Hq / Hk * T;          // rows per kv head: (head, query), query fastest
    // The tensor-core split kernel takes D 64 / 128, at most 16 rows per kv
    // head, at most kMaxBatch sequences (their lengths sit in shared memory)
    // and caches whose TMA row coordinates fit 32 bits; every other shape runs
    // on the CUDA-core split kernel.
    const int64_t rows = kv->page_size ? static_cast<int64_t>(kv->num_pages) * Hk * 16
                                       : static_cast<int64_t>(B) * Hk * kv->max_seq;
    const bool simt = dense || (D != 64 && D != 128) || B > kvq::kMaxBatch ||
                      rows >= (1ll << 31);
    if (B == 0) return KVQ_OK;

    int chunk = 0, splits = 0;
    // (mixed cache: the split kernel walks the INT8 part, the hint less the window)
    const int hint = recent ? (max_seq_len_hint > recent ? max_seq_len_hint - recent : 0)
                            : walked_hint(max_seq_len_hint, T, window);
    kvq_status st = plan(B, Hk, hint, num_splits, 0, &chunk, &splits);
    if (st != KVQ_OK) return st;
    // work items (sequence, kv head, chunk) are counted in 32-bit integers
    if (static_cast<int64_t>(B) * Hk * (splits + 3) >= (1ll << 31)) return KVQ_ERR_UNSUPPORTED;
    const size_t need = recent ? mixed_workspace_for(B, Hq * T, D, splits)
                               : workspace_for(B, Hq * T, D, splits);
    if (need > 0 && (!workspace || workspace_bytes < need)) return KVQ_ERR_INVALID_ARG;

    kvq::DecodeParams p{};
    p.q = q; p.k = kv->k; p.v = kv->v; p.k_scale = kv->k_scale; p.v_scale = kv->v_scale;
    p.table = kv->page_table; p.seq_lens = d_seq_lens; p.out = out; p.d_err = d_err;
    // [o: n_part * D][m: n_part][l: n_part]
    float* ws = static_cast<float*>(workspace);
    const size_t n_part = static_cast<size_t>(B) * Hq * T * splits;
    p.ws_o = ws;
    p.ws_m = ws ? ws + n_part * D : nullptr;
    p.ws_l = ws ? ws + n_part * (D + 1) : nullptr;
    if (k_new) {                        // fused append: the view's arrays are written
        p.k_new = k_new; p.v_new = v_new;
        p.k_w = const_cast<uint8_t*>(kv->k); p.v_w = const_cast<uint8_t*>(kv->v);
        p.ks_w = const_cast<float*>(kv->k_scale); p.vs_w = const_cast<float*>(kv->v_scale);
    }
    p.B = B; p.Hq = Hq * T; p.Hk = Hk; p.G = G; p.D = D; p.group32 = mode == KVQ_SCALE_GROUP32;
    p.fp8 = fp8_code(mode);
    p.static_ns = static_ns(mode, D);
    p.qlen = T;
    p.window = window;
    p.recent = recent;
    p.rk = rk;
    p.rv = rv;
    p.page_size = kv->page_size; p.max_seq = kv->max_seq; p.max_pages = kv->max_pages;
    p.num_pages = kv->num_pages; p.chunk = chunk; p.splits = splits;
    if (simt) {
        p.grid = 0;                     // one CTA per item (and block of rows)
        p.one_item = 1;
    } else {
        int sms = 0;
        if (!current_sms(&sms)) return KVQ_ERR_CUDA;
        const int64_t items = static_cast<int64_t>(B) * Hk * splits;
        p.grid = static_cast<int>(items < sms ? items : sms);   // persistent: one CTA per SM
        if (p.grid > kvq::kMaxGrid) p.grid = kvq::kMaxGrid;
        p.one_item = items <= p.grid ? 1 : 0;
    }
    p.scale_log2 = attn_scale * 1.4426950408889634f;
    // one-stage chunks (many units): a CTA pays about three stages of time
    // for every (sequence, kv head) it starts (merge, query set-up), so each
    // unit start weighs three items when the items are divided among the CTAs
    p.seg_w = (chunk <= 128 && !p.one_item) ? 3 : 0;
    if (recent) {                       // mixed cache: INT8 partials, then the window kernel
        const cudaStream_t cs = static_cast<cudaStream_t>(stream);
        if (hint > 0) {
            const cudaError_t e = simt ? kvq::launch_decode_simt(p, cs)
                                       : kvq::launch_decode_split_tc(p, cs);
            if (e != cudaSuccess) return KVQ_ERR_CUDA;
        }
        return from_cuda(kvq::launch_recent_combine(p, cs));
    }
    return from_cuda(kvq::launch_decode(p, static_cast<cudaStream_t>(stream), simt));
}

}  // namespace

extern "C" {

kvq_status kvq_append(const uint16_t* k_new, const uint16_t* v_new, int B, int Hk, int T, int D,
                      kvq_scale_mode mode, const int32_t* d_pos, uint8_t* k_cache,
                      uint8_t* v_cache, float* k_scale, float* v_scale, int max_seq,
                      int32_t* d_err, kvq_stream_t stream) {
    kvq_status st = check_append_common(k_new, v_new, B, Hk, T, D, mode, d_pos, k_cache, v_cache,
                                        k_scale, v_scale, d_err);
    if (st != KVQ_OK) return st;
    if (max_seq < 1) return KVQ_ERR_INVALID_ARG;
    kvq::AppendParams p{};
    p.k_new = k_new; p.v_new = v_new; p.k_dst = k_cache; p.v_dst = v_cache;
    p.k_scale = k_scale; p.v_scale = v_scale; p.pos = d_pos; p.table = nullptr; p.d_err = d_err;
    p.B = B; p.Hk = Hk; p.T = T; p.D = D; p.group32 = mode == KVQ_SCALE_GROUP32;
    p.fp8 = fp8_code(mode);
    p.static_ns = static_ns(mode, D);
    p.max_seq = max_seq; p.page_size = 0;
    return from_cuda(kvq::launch_append(p, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_append_paged(const uint16_t* k_new, const uint16_t* v_new, int B, int Hk, int T,
                            int D, kvq_scale_mode mode, const int32_t* d_pos, uint8_t* k_arena,
                            uint8_t* v_arena, float* k_scale, float* v_scale,
                            const int32_t* page_table, int max_pages, int num_pages,
                            int page_size, int32_t* d_err, kvq_stream_t stream) {
    kvq_status st = check_append_common(k_new, v_new, B, Hk, T, D, mode, d_pos, k_arena, v_arena,
                                        k_scale, v_scale, d_err);
    if (st != KVQ_OK) return st;
    if (!page_table || !aligned(page_table, 4) || max_pages < 1 || num_pages < 1 ||
        page_size != 16)
        return KVQ_ERR_INVALID_ARG;
    kvq::AppendParams p{};
    p.k_new = k_new; p.v_new = v_new; p.k_dst = k_arena; p.v_dst = v_arena;
    p.k_scale = k_scale; p.v_scale = v_scale; p.pos = d_pos; p.table = page_table;
    p.d_err = d_err; p.B = B; p.Hk = Hk; p.T = T; p.D = D;
    p.group32 = mode == KVQ_SCALE_GROUP32; p.fp8 = fp8_code(mode);
    p.static_ns = static_ns(mode, D);
    p.max_seq = 0; p.page_size = page_size;
    p.max_pages = max_pages; p.num_pages = num_pages;
    return from_cuda(kvq::launch_append(p, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_append_calibrate(const uint16_t* k_new, const uint16_t* v_new, int B, int Hk,
                                int T, int D, kvq_scale_mode mode, const int32_t* d_pos,
                                uint8_t* k_cache, uint8_t* v_cache, float* k_scale,
                                float* v_scale, int max_seq, int32_t* d_err, kvq_stream_t stream) {
    if (!is_static(mode)) return KVQ_ERR_INVALID_ARG;
    kvq_status st = check_append_common(k_new, v_new, B, Hk, T, D, mode, d_pos, k_cache, v_cache,
                                        k_scale, v_scale, d_err);
    if (st != KVQ_OK) return st;
    if (max_seq < 1) return KVQ_ERR_INVALID_ARG;
    kvq::AppendParams p{};
    p.k_new = k_new; p.v_new = v_new; p.k_dst = k_cache; p.v_dst = v_cache;
    p.k_scale = k_scale; p.v_scale = v_scale; p.pos = d_pos; p.table = nullptr; p.d_err = d_err;
    p.B = B; p.Hk = Hk; p.T = T; p.D = D; p.static_ns = static_ns(mode, D);
    p.max_seq = max_seq; p.page_size = 0;
    return from_cuda(kvq::launch_append_calibrate(p, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_decode_plan(int B, int Hk, int max_seq_len_hint, int num_splits, int num_sms,
                           int* chunk, int* splits) {
    if (!chunk || !splits) return KVQ_ERR_INVALID_ARG;
    return plan(B, Hk, max_seq_len_hint, num_splits, num_sms, chunk, splits);
}

size_t kvq_decode_workspace_bytes(int B, int Hq, int Hk, int D, int max_seq_len_hint,
                                  int num_splits) {
    int chunk = 0, splits = 0;
    if (B < 1 || Hq < 1 || D < 1) return 0;
    if (plan(B, Hk, max_seq_len_hint, num_splits, 0, &chunk, &splits) != KVQ_OK) return 0;
    return workspace_for(B, Hq, D, splits);
}

kvq_status kvq_decode_attn(const uint16_t* q, int B, int Hq, int Hk, int D, kvq_scale_mode mode,
                           const kvq_cache_view* kv, const int32_t* d_seq_lens,
                           int max_seq_len_hint, float attn_scale, float* out, void* workspace,
                           size_t workspace_bytes, int num_splits, int32_t* d_err,
                           kvq_stream_t stream) {
    return attend(q, B, Hq, Hk, 1, D, mode, kv, d_seq_lens, max_seq_len_hint, 0, attn_scale, out,
                  workspace, workspace_bytes, num_splits, d_err, stream);
}

kvq_status kvq_append_decode(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                             int B, int Hq, int Hk, int D, kvq_scale_mode mode,
                             const kvq_cache_view* kv, const int32_t* d_seq_lens,
                             int max_seq_len_hint, float attn_scale, float* out, void* workspace,
                             size_t workspace_bytes, int num_splits, int32_t* d_err,
                             kvq_stream_t stream) {
    if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)) return KVQ_ERR_INVALID_ARG;
    if (!valid_mode(mode)) return KVQ_ERR_INVALID_ARG;
    if (mode != KVQ_SCALE_PER_TOKEN && mode != KVQ_SCALE_GROUP32) return KVQ_ERR_UNSUPPORTED;
    return attend(q, B, Hq, Hk, 1, D, mode, kv, d_seq_lens, max_seq_len_hint, 0, attn_scale, out,
                  workspace, workspace_bytes, num_splits, d_err, stream, 0, nullptr, nullptr,
                  k_new, v_new);
}

kvq_status kvq_chunk_attn(const uint16_t* q, int B, int Hq, int Hk, int T, int D,
                          kvq_scale_mode mode, const kvq_cache_view* kv,
                          const int32_t* d_seq_lens, int max_seq_len_hint, float attn_scale,
                          float* out, void* workspace, size_t workspace_bytes, int num_splits,
                          int32_t* d_err, kvq_stream_t stream) {
    if (T < 1) return KVQ_ERR_INVALID_ARG;
    return attend(q, B, Hq, Hk, T, D, mode, kv, d_seq_lens, max_seq_len_hint, 0, attn_scale, out,
                  workspace, workspace_bytes, num_splits, d_err, stream);
}

kvq_status kvq_append_mixed(const uint16_t* k_new, const uint16_t* v_new, int B, int Hk, int T,
                            int D, kvq_scale_mode mode, const int32_t* d_lens_old,
                            uint8_t* k_cache, uint8_t* v_cache, float* k_scale, float* v_scale,
                            int max_seq, uint16_t* k_ring, uint16_t* v_ring, int window,
                            int32_t* d_err, kvq_stream_t stream) {
    if (mode != KVQ_SCALE_PER_TOKEN && mode != KVQ_SCALE_GROUP32 && !is_static(mode))
        return KVQ_ERR_INVALID_ARG;
    kvq_status st = check_append_common(k_new, v_new, B, Hk, T, D, mode, d_lens_old, k_cache,
                                        v_cache, k_scale, v_scale, d_err);
    if (st != KVQ_OK) return st;
    if (max_seq < 1 || window < 1 || window > kvq::kMaxRecent || !k_ring || !v_ring ||
        !aligned(k_ring, 16) || !aligned(v_ring, 16))
        return KVQ_ERR_INVALID_ARG;
    kvq::AppendParams p{};
    p.k_new = k_new; p.v_new = v_new; p.k_dst = k_cache; p.v_dst = v_cache;
    p.k_scale = k_scale; p.v_scale = v_scale; p.pos = d_lens_old; p.table = nullptr;
    p.d_err = d_err; p.B = B; p.Hk = Hk; p.T = T; p.D = D;
    p.group32 = mode == KVQ_SCALE_GROUP32; p.static_ns = static_ns(mode, D);
    p.max_seq = max_seq; p.page_size = 0;
    return from_cuda(kvq::launch_append_mixed(p, k_ring, v_ring, window,
                                              static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_decode_attn_mixed(const uint16_t* q, int B, int Hq, int Hk, int D,
                                 kvq_scale_mode mode, const kvq_cache_view* kv,
                                 const uint16_t* k_ring, const uint16_t* v_ring, int window,
                                 const int32_t* d_seq_lens, int max_seq_len_hint,
                                 float attn_scale, float* out, void* workspace,
                                 size_t workspace_bytes, int num_splits, int32_t* d_err,
                                 kvq_stream_t stream) {
    if (window < 1 || window > kvq::kMaxRecent || !k_ring || !v_ring || !aligned(k_ring, 16) ||
        !aligned(v_ring, 16))
        return KVQ_ERR_INVALID_ARG;
    if (B > 0 && !workspace) return KVQ_ERR_INVALID_ARG;
    return attend(q, B, Hq, Hk, 1, D, mode, kv, d_seq_lens, max_seq_len_hint, 0, attn_scale, out,
                  workspace, workspace_bytes, num_splits, d_err, stream, window, k_ring, v_ring);
}

size_t kvq_mixed_workspace_bytes(int B, int Hq, int Hk, int D, int max_seq_len_hint, int window,
                                 int num_splits) {
    int chunk = 0, splits = 0;
    if (B < 1 || Hq < 1 || D < 1 || window < 1) return 0;
    const int hint = max_seq_len_hint > window ? max_seq_len_hint - window : 0;
    if (plan(B, Hk, hint, num_splits, 0, &chunk, &splits) != KVQ_OK) return 0;
    return mixed_workspace_for(B, Hq, D, splits);
}

kvq_status kvq_window_attn(const uint16_t* q, int B, int Hq, int Hk, int T, int D,
                           kvq_scale_mode mode, const kvq_cache_view* kv,
                           const int32_t* d_seq_lens, int max_seq_len_hint, int window,
                           float attn_scale, float* out, void* workspace, size_t workspace_bytes,
                           int num_splits, int32_t* d_err, kvq_stream_t stream) {
    if (T < 1 || window < 1) return KVQ_ERR_INVALID_ARG;
    return attend(q, B, Hq, Hk, T, D, mode, kv, d_seq_lens, max_seq_len_hint, window, attn_scale,
                  out, workspace, workspace_bytes, num_splits, d_err, stream);
}

size_t kvq_window_workspace_bytes(int B, int Hq, int Hk, int T, int D, int max_seq_len_hint,
                                  int window, int num_splits) {
    if (T < 1 || window < 1 || Hq > INT32_MAX / T) return 0;
    return kvq_decode_workspace_bytes(B, Hq * T, Hk, D, walked_hint(max_seq_len_hint, T, window),
                                      num_splits);
}

size_t kvq_chunk_workspace_bytes(int B, int Hq, int Hk, int T, int D, int max_seq_len_hint,
                                 int num_splits) {
    if (T < 1 || Hq > INT32_MAX / T || Hk < 1) return 0;
    // (above 16 rows per kv head the dense kernel needs none, but the shapes it
    // does not cover run on the CUDA-core split kernel, which does)
    return kvq_decode_workspace_bytes(B, Hq * T, Hk, D, max_seq_len_hint, num_splits);
}

kvq_status kvq_dequant(const uint8_t* q, const float* scale, int64_t rows, int D,
                       kvq_scale_mode mode, float* out, kvq_stream_t stream) {
    if (rows < 0 || D < 16 || (D % 16) != 0) return KVQ_ERR_INVALID_ARG;
    if (!valid_mode(mode)) return KVQ_ERR_INVALID_ARG;
    if (mode == KVQ_SCALE_GROUP32 && (D % 32) != 0) return KVQ_ERR_INVALID_ARG;
    if (rows == 0) return KVQ_OK;
    if (!q || (!scale && !is_fp8(mode)) || !out || !aligned(q, 16) || !aligned(out, 16) ||
        !aligned(scale, mode == KVQ_SCALE_PER_HEAD ? 4 : 16))
        return KVQ_ERR_INVALID_ARG;
    return from_cuda(kvq::launch_dequant(q, scale, rows, D, mode == KVQ_SCALE_GROUP32,
                                         fp8_code(mode), static_ns(mode, D), out,
                                         static_cast<cudaStream_t>(stream)));
}

const char* kvq_status_string(kvq_status status) {
    switch (status) {
        case KVQ_OK: return "KVQ_OK";
        case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
        case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
        case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
        case KVQ_ERR_DEVICE_FLAG: return "KVQ_ERR_DEVICE_FLAG";
        case KVQ_ERR_SCRATCH_TOO_SMALL: return "KVQ_ERR_SCRATCH_TOO_SMALL";
        case KVQ_ERR_OUT_OF_PAGES: return "KVQ_ERR_OUT_OF_PAGES";
    }
    return "KVQ_UNKNOWN_STATUS";
}

kvq_status kvq_read_error(int32_t* d_err, int32_t* bits, kvq_stream_t stream) {
    if (!d_err || !aligned(d_err, 4)) return KVQ_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, d_err, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return KVQ_ERR_CUDA;
    if (cudaMemsetAsync(d_err, 0, sizeof(int32_t), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return KVQ_ERR_CUDA;
    if (bits) *bits = h;
    return h ? KVQ_ERR_DEVICE_FLAG : KVQ_OK;
}

kvq_status kvq_check_error(int32_t* d_err, kvq_stream_t stream) {
    return kvq_read_error(d_err, nullptr, stream);
}

int64_t kvq_cache_bytes(int64_t layers, int64_t Hk, int64_t seq, int D, kvq_scale_mode mode) {
    // per-head / per-channel scales are per (sequence, kv head), not per token
    const int64_t ng = mode == KVQ_SCALE_GROUP32 ? D / 32 : (is_fp8(mode) || is_static(mode)) ? 0 : 1;
    return layers * 2 * Hk * seq * (static_cast<int64_t>(D) + 4 * ng);
}

const char* kvq_version(void) { return "kvq 0.1.0 (sm_100a)"; }

}  // extern "C"

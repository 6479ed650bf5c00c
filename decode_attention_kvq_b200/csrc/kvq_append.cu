// kvq_append.cu -- quantise new K/V tokens and store them in the INT8 cache.
//
// FP8 modes (llama-gguf 0.14.0, src/model/kv_quantized.rs,
// quantize_fp8_e4m3 / quantize_fp8_e5m2): each value becomes its truncated
// FP8 byte (fp8_from_bf16), with no scale.
//
// Method (abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
// CudaQuantizedKvCache::quantize_tensor; group-32 variant after realizar
// 0.8.5 kv_cache_q8_init.rs and combs-models 0.2.2 kv.rs kv_quantize):
//   m = max(max_i |x_i|, 1e-8);  s = m / 127;
//   byte_i = clamp(round_half_away(x_i / s) + 128, 0, 255);  scale = s (fp32).
// Both divisions are IEEE round-to-nearest fp32 divisions, and roundf rounds
// half away from zero, so the bytes and scales are bit-exact with that
// definition; the per-element quotient is taken by a reciprocal multiply
// except within 1e-4 of a rounding tie (round_quotient in kvq_internal.cuh),
// which gives the same byte.
//
// Mapping: one "row" is the D values of one (which in {K, V}, b, h, t).  A
// row is handled by P = next_pow2(D / 16) lanes of a warp, each lane loading
// 16 bf16 (two 16-byte loads) and storing 16 bytes; the absolute maximum is
// reduced with xor shuffles inside the row (per token) or inside each lane
// pair that covers 32 values (group-32).  The kernel is HBM-bound: per
// row it reads 2*D bytes and writes D + 4*NG bytes.  It is launched as a
// programmatic dependent (waits for the preceding grid before reading).
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads)
append_kernel(AppendParams p, int lanes_log2) {
    grid_dep_wait();                             // inputs written by the preceding grid
    grid_dep_launch();
    const int P = 1 << lanes_log2;               // lanes per row
    const int lane = threadIdx.x & 31;
    const int sub = lane & (P - 1);              // lane index inside the row
    // CTA = one (K or V, sequence, kv head) unit (blockIdx.x) and a block of
    // its tokens (blockIdx.y): the unit's indices are the same for the whole
    // CTA, and a lane's token is its row within the block
    const int units = p.B * p.Hk;
    const int which = static_cast<int>(blockIdx.x) >= units;      // 0: K, 1: V
    const int bh = static_cast<int>(blockIdx.x) - which * units;
    const int b = bh / p.Hk;
    const int h = bh - b * p.Hk;
    const int rows_per_cta = (static_cast<int>(blockDim.x) >> 5) * (32 >> lanes_log2);
    const int t = static_cast<int>(blockIdx.y) * rows_per_cta +
                  (static_cast<int>(threadIdx.x) >> 5) * (32 >> lanes_log2) + (lane >> lanes_log2);
    // Every lane stays to the end of the shuffles below (full-warp masks);
    // lanes past the last token just carry no data.
    const bool row_ok = t < p.T;
    const int64_t r = static_cast<int64_t>(bh) * p.T + (row_ok ? t : 0);   // source row

    // ---- destination row (skip and flag when out of range)
    int64_t dst_row = -1;
    uint32_t flag = 0;
    if (row_ok) {
        const int64_t p0 = p.pos[b];
        if (p.page_size == 0) {
            if (p0 < 0 || p0 + p.T > p.max_seq) flag = KVQ_DEVERR_POS;
            else dst_row = (static_cast<int64_t>(b) * p.Hk + h) * p.max_seq + p0 + t;
        } else {
            const int64_t cap = static_cast<int64_t>(p.max_pages) * p.page_size;
            if (p0 < 0 || p0 + p.T > cap) {
                flag = KVQ_DEVERR_POS;
            } else {
                const int64_t g = p0 + t;                // (pages of 16 tokens)
                const int32_t page = p.table[static_cast<int64_t>(b) * p.max_pages + (g >> 4)];
                if (page < 0 || page >= p.num_pages) flag = KVQ_DEVERR_PAGE;
                else dst_row = (static_cast<int64_t>(page) * p.Hk + h) * 16 + (g & 15);
            }
        }
    }
    if (flag && sub == 0) raise_flag(p.d_err, flag);

    const int nvec = p.D >> 4;                   // 16-value vectors per row (lanes)
    const bool active = row_ok && sub < nvec;
    const uint16_t* src = (which ? p.v_new : p.k_new) + r * p.D;
    uint8_t* dst = (which ? p.v_dst : p.k_dst) + dst_row * p.D + sub * 16;

    // the lane's 16 values: two 16-byte loads
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (active) {
        const uint4 a = *reinterpret_cast<const uint4*>(src + sub * 16);
        const uint4 c = *reinterpret_cast<const uint4*>(src + sub * 16 + 8);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = c.x; w[5] = c.y; w[6] = c.z; w[7] = c.w;
    }
    if (p.fp8) {                                 // FP8: one byte a value, no scale
        if (!active || dst_row < 0) return;
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t hb = (w[i >> 1] >> (16 * (i & 1))) & 0xffffu;
            packed[i >> 2] |= fp8_from_bf16(hb, p.fp8) << (8 * (i & 3));
        }
        *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        return;
    }

    float x[16];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = bf16_bits_to_f32(w[i] & 0xffffu);
        x[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    if (p.static_ns) {                           // per head / per channel: stored scales
        if (!active || dst_row < 0) return;
        const float* sc = (which ? p.v_scale : p.k_scale) +
                          (static_cast<int64_t>(b) * p.Hk + h) * p.static_ns;
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float si = sc[p.static_ns > 1 ? sub * 16 + i : 0];
            packed[i >> 2] |= q8_byte(x[i], si, __frcp_rn(si)) << (8 * (i & 3));
        }
        *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        return;
    }
    // reduce inside the group of lanes sharing one scale (group-32: two lanes)
    const int red_lanes = p.group32 ? 2 : P;
    for (int off = 1; off < red_lanes; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));

    if (!active || dst_row < 0) return;
    const float s = q8_scale(amax);
    const float inv = __frcp_rn(s);
    uint32_t packed[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) packed[i >> 2] |= q8_byte(x[i], s, inv) << (8 * (i & 3));
    *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    float* sdst = which ? p.v_scale : p.k_scale;
    if (p.group32) {
        if ((sub & 1) == 0) sdst[dst_row * (p.D >> 5) + (sub >> 1)] = s;
    } else if (sub == 0) {
        sdst[dst_row] = s;
    }
}

// Per-head / per-channel calibration (abaddon 0.2.0-rc.1,
// OptimizedQuantizedKvCache::quantize_with_granularity), contiguous caches:
// one CTA per (K or V, b, h).  Thread (c, r) owns channel c and the tokens
// t = r (mod lanes); the maxima are reduced through shared memory (over the
// token lanes per channel, or over everything per head), the scales written,
// then the same threads quantise their tokens with them.
constexpr int kCalThreads = 256;
__global__ void __launch_bounds__(kCalThreads)
calibrate_kernel(AppendParams p) {
    grid_dep_wait();
    grid_dep_launch();
    __shared__ float red[kCalThreads];
    __shared__ float scl[256];
    const int units = p.B * p.Hk;
    const int which = blockIdx.x / units;
    const int bh = blockIdx.x % units;
    const int b = bh / p.Hk;
    const int D = p.D, T = p.T, tid = threadIdx.x;
    const int lanes = kCalThreads / D;           // token lanes per channel (D <= 256)
    const int c = tid % D, r = tid / D;
    const bool act = r < lanes;
    const int64_t p0 = p.pos[b];
    if (p0 < 0 || p0 + T > p.max_seq) {          // the whole unit is skipped
        if (tid == 0 && which == 0 && bh % p.Hk == 0) raise_flag(p.d_err, KVQ_DEVERR_POS);
        return;
    }
    const uint16_t* x = (which ? p.v_new : p.k_new) + static_cast<int64_t>(bh) * T * D;
    float m = 0.f;
    if (act)
        for (int t = r; t < T; t += lanes)
            m = fmaxf(m, fabsf(bf16_bits_to_f32(x[static_cast<int64_t>(t) * D + c])));
    red[tid] = m;
    __syncthreads();
    float* sc = (which ? p.v_scale : p.k_scale) + static_cast<int64_t>(bh) * p.static_ns;
    if (p.static_ns > 1) {                       // per channel: over the token lanes
        if (act && r == 0) {
            for (int k = 1; k < lanes; ++k) m = fmaxf(m, red[k * D + c]);
            const float s = q8_scale(m);
            scl[c] = s;
            sc[c] = s;
        }
    } else {                                     // per head: over every thread
        for (int off = kCalThreads / 2; off > 0; off >>= 1) {
            if (tid < off) red[tid] = fmaxf(red[tid], red[tid + off]);
            __syncthreads();
        }
        if (tid == 0) {
            const float s = q8_scale(red[0]);
            scl[0] = s;
            sc[0] = s;
        }
    }
    __syncthreads();
    if (!act) return;
    const float s = scl[p.static_ns > 1 ? c : 0];
    const float inv = __frcp_rn(s);
    uint8_t* dst = (which ? p.v_dst : p.k_dst) + (static_cast<int64_t>(bh) * p.max_seq + p0) * D;
    for (int t = r; t < T; t += lanes) {
        const float xv = bf16_bits_to_f32(x[static_cast<int64_t>(t) * D + c]);
        dst[static_cast<int64_t>(t) * D + c] = static_cast<uint8_t>(q8_byte(xv, s, inv));
    }
}

// Mixed cache append (abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
// OptimizedQuantizedKvCache::append): one CTA per (K or V, b, h).  With the
// old length L0 and the new L1 = L0 + T, the window keeps the last W tokens,
// so positions max(0, L0 - W) .. max(0, L1 - W) - 1 leave it: first each of
// them is quantised into the INT8 part (a warp per position: from the ring
// if it was appended earlier, else from the new tokens), then, behind a
// barrier (a new token can land in the ring row an old one is read from),
// the new tokens that stay are copied into the ring (row g % W).
__global__ void __launch_bounds__(kAppendThreads)
append_mixed_kernel(AppendParams p, uint16_t* k_ring, uint16_t* v_ring, int W) {
    grid_dep_wait();
    grid_dep_launch();
    const int units = p.B * p.Hk;
    const int which = blockIdx.x / units;
    const int bh = blockIdx.x % units;
    const int b = bh / p.Hk;
    const int D = p.D, T = p.T;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t L0 = p.pos[b], L1 = L0 + T;
    const int64_t q0 = L0 > W ? L0 - W : 0, q1 = L1 > W ? L1 - W : 0;
    if (L0 < 0 || q1 > p.max_seq) {
        if (threadIdx.x == 0 && which == 0 && bh % p.Hk == 0) raise_flag(p.d_err, KVQ_DEVERR_POS);
        return;
    }
    const uint16_t* x = (which ? p.v_new : p.k_new) + static_cast<int64_t>(bh) * T * D;
    uint16_t* ring = (which ? v_ring : k_ring) + static_cast<int64_t>(bh) * W * D;
    uint8_t* dst = (which ? p.v_dst : p.k_dst) + static_cast<int64_t>(bh) * p.max_seq * D;
    float* sdst = which ? p.v_scale : p.k_scale;
    const int nvec = D >> 3;
    const bool act = lane < nvec;
    for (int64_t g = q0 + warp; g < q1; g += kAppendThreads / 32) {
        const uint16_t* src = g < L0 ? ring + (g % W) * D : x + (g - L0) * D;
        float xv[8];
        float amax = 0.f;
        if (act) {
            const uint4 raw = *reinterpret_cast<const uint4*>(src + lane * 8);
            const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xv[2 * i] = bf16_bits_to_f32(w4[i] & 0xffffu);
                xv[2 * i + 1] = bf16_bits_to_f32(w4[i] >> 16);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(xv[i]));
        }
        float sc[8];
        if (p.static_ns) {                        // stored per-head / per-channel scales
            const float* st = sdst + static_cast<int64_t>(bh) * p.static_ns;
#pragma unroll
            for (int i = 0; i < 8; ++i) sc[i] = act ? st[p.static_ns > 1 ? lane * 8 + i : 0] : 1.f;
        } else {                                  // per token or per 32-value group
            const int red = p.group32 ? 4 : 32;
            for (int off = 1; off < red; off <<= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            const float s = q8_scale(amax);
#pragma unroll
            for (int i = 0; i < 8; ++i) sc[i] = s;
            if (act) {
                const int64_t row = static_cast<int64_t>(bh) * p.max_seq + g;
                if (p.group32) {
                    if ((lane & 3) == 0) sdst[row * (D >> 5) + (lane >> 2)] = s;
                } else if (lane == 0) {
                    sdst[row] = s;
                }
            }
        }
        if (act) {
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; ++i)
                packed[i >> 2] |= q8_byte(xv[i], sc[i], __frcp_rn(sc[i])) << (8 * (i & 3));
            *reinterpret_cast<uint2*>(dst + g * D + lane * 8) = make_uint2(packed[0], packed[1]);
        }
    }
    __syncthreads();
    const int64_t g0 = q1 > L0 ? q1 : L0;         // the new tokens that stay in the window
    for (int64_t i = threadIdx.x; i < (L1 - g0) * nvec; i += kAppendThreads) {
        const int64_t g = g0 + i / nvec;
        const int c = static_cast<int>(i % nvec);
        *reinterpret_cast<uint4*>(ring + (g % W) * D + c * 8) =
            *reinterpret_cast<const uint4*>(x + (g - L0) * D + c * 8);
    }
}

}  // namespace

cudaError_t launch_append_mixed(const AppendParams& p, uint16_t* k_ring, uint16_t* v_ring, int W,
                                cudaStream_t s) {
    const int64_t blocks = 2ll * p.B * p.Hk;
    if (blocks > 0x7fffffffll || W < 1 || p.D > 256) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(kAppendThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, append_mixed_kernel, p, k_ring, v_ring, W);
}

cudaError_t launch_append_calibrate(const AppendParams& p, cudaStream_t s) {
    if (p.D > 256 || p.D < 1) return cudaErrorInvalidValue;
    const int64_t blocks = 2ll * p.B * p.Hk;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(kCalThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, calibrate_kernel, p);
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    const int nvec = p.D >> 4;                   // lanes per row: 16 values each
    int lanes_log2 = 0;
    while ((1 << lanes_log2) < nvec) ++lanes_log2;
    // one CTA per (K or V, sequence, kv head) and block of tokens; a small
    // append takes only the warps its tokens need
    const int64_t units = 2ll * p.B * p.Hk;
    const int64_t lanes = static_cast<int64_t>(p.T) << lanes_log2;
    const int threads = static_cast<int>(lanes >= kAppendThreads ? kAppendThreads : (lanes + 31) / 32 * 32);
    const int rows_per_block = (threads / 32) * (32 >> lanes_log2);
    const int64_t tblocks = (p.T + rows_per_block - 1) / rows_per_block;
    if (units > 0x7fffffffll || tblocks > 65535) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units), static_cast<unsigned>(tblocks), 1);
    cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, append_kernel, p, lanes_log2);
}

}  // namespace kvq

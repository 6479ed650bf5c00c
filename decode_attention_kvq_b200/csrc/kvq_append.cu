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
// Both divisions are IEEE round-to-nearest fp32 divisions (__fdiv_rn), and
// roundf rounds half away from zero, so the bytes and scales are bit-exact
// with that definition.
//
// Mapping: one "row" is the D values of one (which in {K, V}, b, h, t).  A
// row is handled by P = next_pow2(D / 8) lanes of a warp, each lane loading
// 8 bf16 (16 bytes) and storing 8 bytes; the absolute maximum is reduced
// with xor shuffles inside the row (per token) or inside each 4-lane
// quarter that covers 32 values (group-32).  The kernel is HBM-bound: per
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
    const int rows_per_warp = 32 >> lanes_log2;
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * kAppendThreads + threadIdx.x) >> 5;
    const int64_t row = warp_global * rows_per_warp + (lane >> lanes_log2);
    const int64_t rows_per_tensor = static_cast<int64_t>(p.B) * p.Hk * p.T;
    // Every lane stays to the end of the shuffles below (full-warp masks);
    // lanes past the last row just carry no data.
    const bool row_ok = row < 2 * rows_per_tensor;

    const int which = row_ok && row >= rows_per_tensor;    // 0: K, 1: V
    const int64_t r = row_ok ? row - which * rows_per_tensor : 0;
    const int t = static_cast<int>(r % p.T);
    const int h = static_cast<int>((r / p.T) % p.Hk);
    const int b = static_cast<int>(r / (static_cast<int64_t>(p.T) * p.Hk));

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
                const int64_t g = p0 + t;
                const int32_t page =
                    p.table[static_cast<int64_t>(b) * p.max_pages + g / p.page_size];
                if (page < 0 || page >= p.num_pages) flag = KVQ_DEVERR_PAGE;
                else dst_row = (static_cast<int64_t>(page) * p.Hk + h) * p.page_size
                               + g % p.page_size;
            }
        }
    }
    if (flag && sub == 0) raise_flag(p.d_err, flag);

    const int nvec = p.D >> 3;                   // 8-value vectors per row
    const bool active = row_ok && sub < nvec;
    const uint16_t* src = (which ? p.v_new : p.k_new) + r * p.D;

    if (p.fp8) {                                 // FP8: one byte a value, no scale
        if (!active || dst_row < 0) return;
        const uint4 raw = *reinterpret_cast<const uint4*>(src + sub * 8);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t h = (w[i >> 1] >> (16 * (i & 1))) & 0xffffu;
            packed[i >> 2] |= fp8_from_bf16(h, p.fp8) << (8 * (i & 3));
        }
        uint8_t* dst = (which ? p.v_dst : p.k_dst) + dst_row * p.D + sub * 8;
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
        return;
    }

    float x[8];
    float amax = 0.f;
    if (active) {
        const uint4 raw = *reinterpret_cast<const uint4*>(src + sub * 8);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = bf16_bits_to_f32(w[i] & 0xffffu);
            x[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
    }
    // reduce inside the group of lanes sharing one scale
    const int red_lanes = p.group32 ? 4 : P;
    for (int off = 1; off < red_lanes; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));

    if (!active || dst_row < 0) return;
    const float m = amax < 1e-8f ? 1e-8f : amax;
    const float s = __fdiv_rn(m, 127.0f);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int v = static_cast<int>(roundf(__fdiv_rn(x[i], s))) + 128;
        v = v < 0 ? 0 : (v > 255 ? 255 : v);
        packed[i >> 2] |= static_cast<uint32_t>(v) << (8 * (i & 3));
    }
    uint8_t* dst = (which ? p.v_dst : p.k_dst) + dst_row * p.D + sub * 8;
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    float* sdst = which ? p.v_scale : p.k_scale;
    if (p.group32) {
        if ((sub & 3) == 0) sdst[dst_row * (p.D >> 5) + (sub >> 2)] = s;
    } else if (sub == 0) {
        sdst[dst_row] = s;
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    const int nvec = p.D >> 3;
    int lanes_log2 = 0;
    while ((1 << lanes_log2) < nvec) ++lanes_log2;
    const int64_t rows = 2ll * p.B * p.Hk * p.T;
    const int rows_per_block = (kAppendThreads / 32) * (32 >> lanes_log2);
    const int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(kAppendThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, append_kernel, p, lanes_log2);
}

}  // namespace kvq

// kvq_dequant.cu -- x = (byte - 128) * scale, one fp32 multiply per element;
// in the FP8 modes x = the byte's exact E4M3 / E5M2 value (llama-gguf 0.14.0,
// src/model/kv_quantized.rs, dequantize_fp8_e4m3 / dequantize_fp8_e5m2).
//
// Method: abaddon 0.2.0-rc.2, src/kv_cache_quant.rs, QuantizedKvCache::
// dequantize ((u8 - 128) * scale); abaddon 0.2.0-rc.1, kv_cache_quant_cuda.rs,
// int8_dequant_bf16 (per-element scale index = element / values-per-scale;
// this kernel writes fp32).  (byte - 128) is exact in fp32 and __fmul_rn
// rounds the product once, so the output is bit-exact.
//
// Each thread converts 16 bytes (one 16-byte load, four 16-byte stores); a
// 16-value vector never straddles a row or a 32-value group because D and the
// vector start are multiples of 16.  HBM-bound: 1 byte read + 4 bytes written
// per value plus the scales.
#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kDequantThreads = 256;

// The exact value of an FP8 byte (fmt 1: E4M3, bias 7, 3 mantissa bits, 0x7F
// and 0xFF NaN; fmt 2: E5M2, bias 15, 2 mantissa bits, inf at 0x7C, NaN
// above): the magnitude bits moved under the fp32 exponent field and scaled
// by the power of two between the two biases (exact, subnormal codes
// included).
__device__ __forceinline__ float fp8_value(uint32_t c, int fmt) {
    const uint32_t mag = c & 0x7fu;
    const float sgn = (c & 0x80u) ? -1.f : 1.f;
    if (fmt == 1) {
        if (mag == 0x7fu) return __int_as_float(0x7fc00000);
        // E M3 under binary32's exponent / mantissa: 2^(E-127) * 1.M, times 2^(127-7)
        return sgn * __fmul_rn(__uint_as_float(mag << 20), 0x1p120f);
    }
    if (mag == 0x7cu) return sgn * __int_as_float(0x7f800000);
    if (mag > 0x7cu) return __int_as_float(0x7fc00000);
    return sgn * __fmul_rn(__uint_as_float(mag << 21), 0x1p112f);
}

__global__ void __launch_bounds__(kDequantThreads)
dequant_fp8_kernel(const uint8_t* __restrict__ q, int64_t n_vec, int fmt,
                   float* __restrict__ out) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kDequantThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kDequantThreads + threadIdx.x; i < n_vec;
         i += stride) {
        const uint4 raw = *reinterpret_cast<const uint4*>(q + i * 16);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float4* o = reinterpret_cast<float4*>(out + i * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = make_float4(fp8_value(w[j] & 0xffu, fmt), fp8_value((w[j] >> 8) & 0xffu, fmt),
                               fp8_value((w[j] >> 16) & 0xffu, fmt), fp8_value(w[j] >> 24, fmt));
    }
}

// Per-head (ns = 1) / per-channel (ns = D) scales: `scale` holds the
// (sequence, kv head)'s scales, applied to every row.
__global__ void __launch_bounds__(kDequantThreads)
dequant_static_kernel(const uint8_t* __restrict__ q, const float* __restrict__ scale,
                      int64_t n_vec, int D, int ns, float* __restrict__ out) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kDequantThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kDequantThreads + threadIdx.x; i < n_vec;
         i += stride) {
        const int64_t e = i * 16;
        const int d0 = static_cast<int>(e % D);
        const uint4 raw = *reinterpret_cast<const uint4*>(q + e);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float* o = out + e;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float s = scale[ns > 1 ? d0 + j : 0];
            o[j] = __fmul_rn(static_cast<float>(static_cast<int>((w[j >> 2] >> (8 * (j & 3))) & 0xffu) - 128), s);
        }
    }
}

__global__ void __launch_bounds__(kDequantThreads)
dequant_kernel(const uint8_t* __restrict__ q, const float* __restrict__ scale, int64_t n_vec,
               int D, int group32, float* __restrict__ out) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kDequantThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kDequantThreads + threadIdx.x; i < n_vec;
         i += stride) {
        const int64_t e = i * 16;
        const int64_t row = e / D;
        const int d0 = static_cast<int>(e - row * D);
        const float s = group32 ? scale[row * (D >> 5) + (d0 >> 5)] : scale[row];
        const uint4 raw = *reinterpret_cast<const uint4*>(q + e);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        float4* o = reinterpret_cast<float4*>(out + e);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float4 v;
            v.x = __fmul_rn(static_cast<float>(static_cast<int>(w[j] & 0xffu) - 128), s);
            v.y = __fmul_rn(static_cast<float>(static_cast<int>((w[j] >> 8) & 0xffu) - 128), s);
            v.z = __fmul_rn(static_cast<float>(static_cast<int>((w[j] >> 16) & 0xffu) - 128), s);
            v.w = __fmul_rn(static_cast<float>(static_cast<int>(w[j] >> 24) - 128), s);
            o[j] = v;
        }
    }
}

}  // namespace

cudaError_t launch_dequant(const uint8_t* q, const float* scale, int64_t rows, int D,
                           int group32, int fp8, int static_ns, float* out, cudaStream_t s) {
    const int64_t n_vec = rows * D / 16;
    if (n_vec == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n_vec + kDequantThreads - 1) / kDequantThreads;
    const int64_t cap = static_cast<int64_t>(sms) * 8;   // grid-stride beyond 8 blocks per SM
    if (blocks > cap) blocks = cap;
    if (static_ns)
        dequant_static_kernel<<<static_cast<unsigned>(blocks), kDequantThreads, 0, s>>>(
            q, scale, n_vec, D, static_ns, out);
    else if (fp8)
        dequant_fp8_kernel<<<static_cast<unsigned>(blocks), kDequantThreads, 0, s>>>(q, n_vec, fp8,
                                                                                 out);
    else
        dequant_kernel<<<static_cast<unsigned>(blocks), kDequantThreads, 0, s>>>(q, scale, n_vec,
                                                                                 D, group32, out);
    return cudaGetLastError();
}

}  // namespace kvq

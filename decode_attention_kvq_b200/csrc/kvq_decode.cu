// kvq_decode.cu -- decode attention on the INT8 cache with the dequantisation
// fused into Q.K^T and P.V, split-K (flash-decoding) across CTAs, and a
// combine kernel.
//
// Method: abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs, module doc "Fused
// approach" (Q.K^T with K dequantised on the fly, softmax, P.V with V
// dequantised on the fly) and CudaQuantizedKvCache::forward_attention;
// combs-models 0.2.2, src/kv.rs, attend / repeat_kv (scale applied to the
// dot product, query head h reads kv head h / G, a single decode query needs
// no causal mask).  The split-K online softmax and combine are this
// library's own.
//
// Arithmetic per token t and query head g of the CTA's kv head:
//   z = (attn_scale*log2 e) * sum_d q_d * (k_d - 128) * sk(t, group(d))
//   online softmax in base 2 over the split: m, l = sum 2^(z - m),
//   o_d = sum 2^(z - m) * (v_d - 128) * sv(t, group(d))
// A split writes (o, m, l); the combine rescales the splits to the common
// maximum.  A sequence with a single split writes o / l directly.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ float byte_f(uint32_t w, int i) {
    return static_cast<float>(static_cast<int>((w >> (8 * i)) & 0xffu) - 128);
}

// SIMT split kernel: grid (splits, Hk, B), 4 warps.  A warp handles TPI
// consecutive tokens per iteration; each token's D bytes are spread over
// LPT = D/8 lanes (8 bytes per lane), so one warp load covers 256 bytes of
// the K (or V) tile.
template <int D, int GT, bool PAGED, bool G32>
__global__ void __launch_bounds__(kThreads)
decode_split_simt(DecodeParams p) {
    constexpr int VEC = 8;
    constexpr int LPT = D / VEC;
    constexpr int TPI = 32 / LPT;
    constexpr int NG = G32 ? D / 32 : 1;

    __shared__ float s_m[kWarps][GT];
    __shared__ float s_l[kWarps][GT];
    __shared__ __align__(16) float s_o[kWarps][GT][D];

    const int j = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int ltok = lane / LPT, d0 = (lane % LPT) * VEC;
    const int G = p.G;

    const int64_t cap = PAGED ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t lim = min(cap, static_cast<int64_t>(p.splits) * p.chunk);
    int L = p.seq_lens[b];
    if (L < 0 || L > lim) {
        if (j == 0 && hk == 0 && tid == 0) raise_flag(p.d_err, KVQ_DEVERR_LEN);
        L = 0;
    }
    if (L == 0) {                       // empty window: zero output rows
        if (j == 0)
            for (int i = tid; i < G * D; i += kThreads)
                p.out[(static_cast<int64_t>(b) * p.Hq + hk * G) * D + i] = 0.f;
        return;
    }
    const int t0 = j * p.chunk;
    if (t0 >= L) return;
    const int t1 = min(t0 + p.chunk, L);
    const int nsplit = (L + p.chunk - 1) / p.chunk;

    // q slice of this lane, pre-multiplied by attn_scale * log2(e)
    float qr[GT][VEC];
#pragma unroll
    for (int g = 0; g < GT; ++g) {
        if (g < G) {
            const uint4 raw = *reinterpret_cast<const uint4*>(
                p.q + (static_cast<int64_t>(b) * p.Hq + hk * G + g) * D + d0);
            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                qr[g][2 * i] = bf16_bits_to_f32(wv[i] & 0xffffu) * p.scale_log2;
                qr[g][2 * i + 1] = bf16_bits_to_f32(wv[i] >> 16) * p.scale_log2;
            }
        } else {
#pragma unroll
            for (int i = 0; i < VEC; ++i) qr[g][i] = 0.f;
        }
    }

    float m[GT], l[GT], o[GT][VEC];
#pragma unroll
    for (int g = 0; g < GT; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int i = 0; i < VEC; ++i) o[g][i] = 0.f;
    }

    for (int tb = t0 + w * TPI; tb < t1; tb += kWarps * TPI) {
        const int t = tb + ltok;
        bool valid = t < t1;
        int64_t row = 0;
        if (valid) {
            if (PAGED) {
                const int32_t page = p.table[static_cast<int64_t>(b) * p.max_pages + t / 16];
                if (page < 0 || page >= p.num_pages) {
                    if (d0 == 0) raise_flag(p.d_err, KVQ_DEVERR_PAGE);
                    valid = false;
                } else {
                    row = (static_cast<int64_t>(page) * p.Hk + hk) * 16 + (t & 15);
                }
            } else {
                row = (static_cast<int64_t>(b) * p.Hk + hk) * p.max_seq + t;
            }
        }
        uint2 kr = make_uint2(0u, 0u), vr = make_uint2(0u, 0u);
        float ks = 0.f, vs = 0.f;
        if (valid) {
            kr = *reinterpret_cast<const uint2*>(p.k + row * D + d0);
            vr = *reinterpret_cast<const uint2*>(p.v + row * D + d0);
            const int64_t si = row * NG + (G32 ? d0 / 32 : 0);
            ks = p.k_scale[si];
            vs = p.v_scale[si];
        }
        float z[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc = fmaf(qr[g][i], byte_f(kr.x, i), acc);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc = fmaf(qr[g][4 + i], byte_f(kr.y, i), acc);
            z[g] = acc * ks;
        }
#pragma unroll
        for (int off = 1; off < LPT; off <<= 1)
#pragma unroll
            for (int g = 0; g < GT; ++g) z[g] += __shfl_xor_sync(0xffffffffu, z[g], off);
        // a token with a bad page (or past the split) contributes nothing;
        // all LPT lanes of a token agree on `valid`
        const bool tok_valid = valid;
#pragma unroll
        for (int g = 0; g < GT; ++g) {
            float mt = tok_valid ? z[g] : -INFINITY;
#pragma unroll
            for (int off = LPT; off < 32; off <<= 1)
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float m_new = fmaxf(m[g], mt);
            const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m[g] - m_new);
            const float pz = tok_valid ? exp2f(z[g] - m_new) : 0.f;
            l[g] = l[g] * alpha + pz;
            m[g] = m_new;
            const float pv = pz * vs;
#pragma unroll
            for (int i = 0; i < 4; ++i) o[g][i] = fmaf(pv, byte_f(vr.x, i), o[g][i] * alpha);
#pragma unroll
            for (int i = 0; i < 4; ++i) o[g][4 + i] = fmaf(pv, byte_f(vr.y, i), o[g][4 + i] * alpha);
        }
    }

    // fold the TPI token lanes of the warp (m is warp-uniform)
#pragma unroll
    for (int off = LPT; off < 32; off <<= 1)
#pragma unroll
        for (int g = 0; g < GT; ++g) {
            l[g] += __shfl_xor_sync(0xffffffffu, l[g], off);
#pragma unroll
            for (int i = 0; i < VEC; ++i) o[g][i] += __shfl_xor_sync(0xffffffffu, o[g][i], off);
        }
    if (ltok == 0) {
#pragma unroll
        for (int g = 0; g < GT; ++g)
#pragma unroll
            for (int i = 0; i < VEC; ++i) s_o[w][g][d0 + i] = o[g][i];
    }
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < GT; ++g) {
            s_m[w][g] = m[g];
            s_l[w][g] = l[g];
        }
    }
    __syncthreads();

    // fold the warps and write the split (or the final row)
    for (int idx = tid; idx < G * D; idx += kThreads) {
        const int g = idx / D, d = idx - g * D;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, s_m[ww][g]);
        float acc = 0.f, lsum = 0.f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
            const float f = (s_m[ww][g] == -INFINITY) ? 0.f : exp2f(s_m[ww][g] - M);
            acc = fmaf(f, s_o[ww][g][d], acc);
            lsum = fmaf(f, s_l[ww][g], lsum);
        }
        const int64_t bh = static_cast<int64_t>(b) * p.Hq + hk * G + g;
        if (nsplit == 1) {
            p.out[bh * D + d] = lsum > 0.f ? acc / lsum : 0.f;   // 0 only when every page was bad
        } else {
            p.ws_o[(bh * p.splits + j) * D + d] = acc;
            if (d == 0) {
                p.ws_m[bh * p.splits + j] = M;
                p.ws_l[bh * p.splits + j] = lsum;
            }
        }
    }
}

// Combine: one CTA per (b, q head); rescales the splits to their common
// maximum and normalises.  Sequences with at most one split were finished by
// the split kernel.
__global__ void __launch_bounds__(kThreads)
decode_combine(DecodeParams p) {
    extern __shared__ float s_w[];      // [splits] weights 2^(m_j - M)
    __shared__ float s_red[kWarps];
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / p.Hq);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int64_t cap = p.page_size ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t lim = min(cap, static_cast<int64_t>(p.splits) * p.chunk);
    int L = p.seq_lens[b];
    if (L < 0 || L > lim) L = 0;
    const int ns = (L + p.chunk - 1) / p.chunk;
    if (ns <= 1) return;

    const float* m = p.ws_m + bh * p.splits;
    const float* lv = p.ws_l + bh * p.splits;
    float M = -INFINITY;
    for (int j = tid; j < ns; j += kThreads) M = fmaxf(M, m[j]);
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if (lane == 0) s_red[w] = M;
    __syncthreads();
    M = s_red[0];
    for (int ww = 1; ww < kWarps; ++ww) M = fmaxf(M, s_red[ww]);
    __syncthreads();
    float lsum = 0.f;
    for (int j = tid; j < ns; j += kThreads) {
        const float wj = (M == -INFINITY) ? 0.f : exp2f(m[j] - M);
        s_w[j] = wj;
        lsum = fmaf(wj, lv[j], lsum);
    }
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    if (lane == 0) s_red[w] = lsum;
    __syncthreads();
    lsum = 0.f;
    for (int ww = 0; ww < kWarps; ++ww) lsum += s_red[ww];
    const float* o = p.ws_o + bh * p.splits * p.D;
    for (int d = tid; d < p.D; d += kThreads) {
        float acc = 0.f;
        for (int j = 0; j < ns; ++j) acc = fmaf(s_w[j], o[static_cast<int64_t>(j) * p.D + d], acc);
        p.out[bh * p.D + d] = lsum > 0.f ? acc / lsum : 0.f;
    }
}

template <int D, int GT, bool PAGED, bool G32>
cudaError_t launch_split(const DecodeParams& p, cudaStream_t s) {
    dim3 grid(p.splits, p.Hk, p.B);
    decode_split_simt<D, GT, PAGED, G32><<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <int D, int GT>
cudaError_t dispatch_layout(const DecodeParams& p, cudaStream_t s) {
    if (p.page_size) {
        return p.group32 ? launch_split<D, GT, true, true>(p, s)
                         : launch_split<D, GT, true, false>(p, s);
    }
    return p.group32 ? launch_split<D, GT, false, true>(p, s)
                     : launch_split<D, GT, false, false>(p, s);
}

template <int D>
cudaError_t dispatch_group(const DecodeParams& p, cudaStream_t s) {
    if (p.G <= 1) return dispatch_layout<D, 1>(p, s);
    if (p.G <= 2) return dispatch_layout<D, 2>(p, s);
    if (p.G <= 4) return dispatch_layout<D, 4>(p, s);
    if (p.G <= 8) return dispatch_layout<D, 8>(p, s);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s) {
    cudaError_t e = p.D == 64 ? dispatch_group<64>(p, s)
                  : p.D == 128 ? dispatch_group<128>(p, s) : cudaErrorInvalidValue;
    if (e != cudaSuccess || p.splits <= 1) return e;
    const size_t smem = static_cast<size_t>(p.splits) * sizeof(float);
    decode_combine<<<p.B * p.Hq, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace kvq

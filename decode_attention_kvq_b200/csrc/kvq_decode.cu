// kvq_decode.cu -- decode attention driver: the persistent split kernel
// (kvq_decode_tc.cu) followed, when some sequence spans more than one chunk,
// by the combine kernel below (launched as a programmatic dependent so its
// launch overlaps the split kernel).
//
// Combine (flash-decoding): for each (sequence, q head) with splits j =
// 0..ns-1 holding unnormalised (o_j, m_j, l_j) in base 2,
//   M = max_j m_j,  w_j = 2^(m_j - M),  out = sum_j w_j o_j / sum_j w_j l_j.
// Sequences with a single split were finished by the split kernel.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

// One CTA per (b, q head).  Warp w folds splits w, w+4, ... with 16-byte
// loads (lane l owns head_dim [4l, 4l+4)), then the four warps are summed.
__global__ void __launch_bounds__(kThreads)
decode_combine(DecodeParams p) {
    extern __shared__ float s_w[];                 // [splits] weights
    __shared__ float s_red[kWarps];
    __shared__ __align__(16) float s_acc[kWarps][256];
    grid_dep_wait();                    // the split kernel's partials are complete
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
    M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
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
    lsum = s_red[0] + s_red[1] + s_red[2] + s_red[3];

    const int D = p.D;
    const bool active = lane * 4 < D;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float* o = p.ws_o + bh * p.splits * D;
    if (active) {
#pragma unroll 4
        for (int j = w; j < ns; j += kWarps) {
            const float4 v = *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D + lane * 4);
            const float wj = s_w[j];
            acc.x = fmaf(wj, v.x, acc.x);
            acc.y = fmaf(wj, v.y, acc.y);
            acc.z = fmaf(wj, v.z, acc.z);
            acc.w = fmaf(wj, v.w, acc.w);
        }
        *reinterpret_cast<float4*>(&s_acc[w][lane * 4]) = acc;
    }
    __syncthreads();
    for (int d = tid; d < D; d += kThreads) {
        const float sum = s_acc[0][d] + s_acc[1][d] + s_acc[2][d] + s_acc[3][d];
        p.out[bh * D + d] = lsum > 0.f ? sum / lsum : 0.f;
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s) {
    cudaError_t e = launch_decode_split_tc(p, s);
    if (e != cudaSuccess || p.splits <= 1) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.B * p.Hq, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(p.splits) * sizeof(float);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine, p);
}

}  // namespace kvq

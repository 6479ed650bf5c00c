// kvq_decode.cu -- decode attention driver: the persistent split kernel
// (kvq_decode_tc.cu) followed, when some sequence spans more than one chunk,
// by the combine kernel below (launched as a programmatic dependent so its
// launch overlaps the split kernel).
//
// Combine (flash-decoding): for each (sequence, q head) with chunk slots j =
// 0..ns-1 holding unnormalised (o_j, m_j, l_j) in base 2,
//   M = max_j m_j,  w_j = 2^(m_j - M),  out = sum_j w_j o_j / sum_j w_j l_j.
// The split kernel merges consecutive chunks it owns into the slot of the
// first of them and marks the others empty (m = -inf, l = 0); a slot of
// weight zero is skipped, never multiplied (its o was not written).  A
// sequence finished whole by one CTA carries l_0 = -1 and is left alone, as
// are sequences with a single chunk.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kBatch = 8;                       // slots in flight per warp
constexpr int kDirect = kWarps * kBatch;        // up to this many slots: one round of loads
constexpr int kMaxList = 4096;                  // = the planner's bound on splits

// One CTA per (b, q head); lane l of a warp owns head_dim [4l, 4l + 4).
__global__ void __launch_bounds__(kThreads)
decode_combine(DecodeParams p) {
    __shared__ float s_m[kWarps], s_l[kWarps];
    __shared__ __align__(16) float s_acc[kWarps][128];
    __shared__ int s_cnt[kWarps];
    __shared__ int s_list[kMaxList];            // slots of non-zero weight (long sequences)
    grid_dep_wait();                    // the split kernel's partials are complete
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / p.Hq);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int L0 = p.seq_lens[b];
    const float* m = p.ws_m + bh * p.splits;
    const float* lv = p.ws_l + bh * p.splits;
    const int D = p.D;
    const bool active = lane * 4 < D;
    const float* o = p.ws_o + bh * p.splits * D + lane * 4;

    // per-warp online fold over a list of slots: running max Mw, sums lw, acc
    float Mw = -INFINITY, lw = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fold = [&](const float (&mj)[kBatch], const float (&lj)[kBatch],
                    const float4 (&oj)[kBatch]) {
        float Mn = Mw;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) Mn = fmaxf(Mn, mj[u]);
        if (Mn == -INFINITY) return;
        const float a = exp2f(Mw - Mn);                   // 0 while Mw is -inf
        acc.x *= a; acc.y *= a; acc.z *= a; acc.w *= a;
        lw *= a;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (mj[u] == -INFINITY) continue;             // empty slot: o unwritten
            const float wj = exp2f(mj[u] - Mn);
            acc.x = fmaf(wj, oj[u].x, acc.x);
            acc.y = fmaf(wj, oj[u].y, acc.y);
            acc.z = fmaf(wj, oj[u].z, acc.z);
            acc.w = fmaf(wj, oj[u].w, acc.w);
            lw = fmaf(wj, lj[u], lw);
        }
        Mw = Mn;
    };

    const int64_t cap = p.page_size ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t lim = min(cap, static_cast<int64_t>(p.splits) * p.chunk);
    bool finished;
    if (p.splits <= kDirect) {
        // one round: every slot of the workspace row is loaded together with the
        // length (slots past the sequence's chunk count are in bounds and masked
        // afterwards, before any arithmetic reads them)
        float mj[kBatch], lj[kBatch];
        float4 oj[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = w + u * kWarps;
            const bool in = j < p.splits;
            mj[u] = in ? m[j] : -INFINITY;
            lj[u] = in ? lv[j] : 0.f;
            oj[u] = (in && active) ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        finished = lv[0] < 0.f;
        const int L = (L0 < 0 || L0 > lim) ? 0 : L0;
        const int ns = (L + p.chunk - 1) / p.chunk;
        if (ns <= 1 || finished) return;               // uniform over the CTA
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (w + u * kWarps >= ns) mj[u] = -INFINITY;
        fold(mj, lj, oj);
    } else {
        const int L = (L0 < 0 || L0 > lim) ? 0 : L0;
        const int ns = (L + p.chunk - 1) / p.chunk;
        if (ns <= 1) return;
        finished = lv[0] < 0.f;
        if (finished) return;                          // uniform over the CTA
        // long sequences: list the slots that hold a partial (in slot order),
        // then load only those
        int n = 0;
        for (int base = 0; base < ns; base += kThreads) {
            const int j = base + tid;
            const bool live = j < ns && m[j] != -INFINITY;
            const uint32_t bal = __ballot_sync(0xffffffffu, live);
            if (lane == 0) s_cnt[w] = __popc(bal);
            __syncthreads();
            int off = n;
            for (int x = 0; x < w; ++x) off += s_cnt[x];
            if (live) s_list[off + __popc(bal & ((1u << lane) - 1u))] = j;
            for (int x = 0; x < kWarps; ++x) n += s_cnt[x];
            __syncthreads();
        }
        for (int u0 = w; u0 < n; u0 += kWarps * kBatch) {
            float mj[kBatch], lj[kBatch];
            float4 oj[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int k = u0 + u * kWarps;
                const int j = k < n ? s_list[k] : 0;
                mj[u] = k < n ? m[j] : -INFINITY;
                lj[u] = k < n ? lv[j] : 0.f;
                oj[u] = (k < n && active)
                            ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            fold(mj, lj, oj);
        }
    }
    if (lane == 0) {
        s_m[w] = Mw;
        s_l[w] = lw;
    }
    if (active) *reinterpret_cast<float4*>(&s_acc[w][lane * 4]) = acc;
    __syncthreads();
    float M = s_m[0];
#pragma unroll
    for (int x = 1; x < kWarps; ++x) M = fmaxf(M, s_m[x]);
    float f[kWarps], lsum = 0.f;
#pragma unroll
    for (int x = 0; x < kWarps; ++x) {
        f[x] = s_m[x] == -INFINITY ? 0.f : exp2f(s_m[x] - M);
        lsum = fmaf(f[x], s_l[x], lsum);
    }
    for (int d = tid; d < D; d += kThreads) {
        float sum = 0.f;
#pragma unroll
        for (int x = 0; x < kWarps; ++x) sum = fmaf(f[x], s_acc[x][d], sum);
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
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine, p);
}

}  // namespace kvq

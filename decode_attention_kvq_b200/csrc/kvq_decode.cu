// kvq_decode.cu -- decode attention driver: the persistent split kernel
// (kvq_decode_tc.cu) followed, when the plan splits a sequence, by the combine
// kernel below (launched as a programmatic dependent so its launch overlaps
// the split kernel).
//
// Combine (flash-decoding): for each (sequence, q head) whose kv head's
// chunks were split over several CTAs, the partial states (o_k, m_k, l_k) in
// base 2 are merged:
//   M = max_k m_k,  w_k = 2^(m_k - M),  out = sum_k w_k o_k / sum_k w_k l_k.
// The split kernel's CTA c owns the items [start(c), start(c + 1)); a unit
// (sequence, kv head) with items [u0, u0 + ns) therefore has its partials in
// chunk 0 and in the first chunk of every CTA block that starts inside it.
// The split kernel publishes the CTA starts, the item prefix sums and the
// chunk counts in the workspace header.  A unit inside one CTA block was
// finished by the split kernel.
#include <math.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kBatch = 8;                       // slots in flight per warp

// One item per CTA (one_item): CTA c of the split kernel held item c of the
// plan, so chunk j < ns of every unit holds a partial and nothing else does.
// One CTA per (b, q head); lane l of a warp owns head_dim [4l, 4l + 4).
__global__ void __launch_bounds__(kThreads)
decode_combine_one(DecodeParams p) {
    __shared__ float s_m[kWarps], s_l[kWarps];
    __shared__ __align__(16) float s_acc[kWarps][128];
    grid_dep_wait();                    // the split kernel's partials are complete
    grid_dep_launch();                  // the next kernel may run its prologue now
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / p.Hq);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const float* m = p.ws_m + bh * p.splits;
    const float* lv = p.ws_l + bh * p.splits;
    const int D = p.D;
    const bool active = lane * 4 < D;
    const float* o = p.ws_o + bh * p.splits * D + lane * 4;
    const int64_t cap = p.page_size ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t lim = min(cap, static_cast<int64_t>(p.splits) * p.chunk);
    const int L0 = p.seq_lens[b];

    float Mw = -INFINITY, lw = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float mj[kBatch], lj[kBatch];
    float4 oj[kBatch];
    auto load = [&](int k0) {                   // slots k0 + u * kWarps
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = k0 + u * kWarps;
            const bool in = j < p.splits;
            mj[u] = in ? m[j] : -INFINITY;
            lj[u] = in ? lv[j] : 0.f;
            oj[u] = (in && active) ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto fold = [&](int k0, int ns) {           // slots past the chunk count are dropped
        float Mn = Mw;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (k0 + u * kWarps >= ns) mj[u] = -INFINITY;
            Mn = fmaxf(Mn, mj[u]);
        }
        if (Mn == -INFINITY) return;
        const float a = exp2f(Mw - Mn);                   // 0 while Mw is -inf
        acc.x *= a; acc.y *= a; acc.z *= a; acc.w *= a;
        lw *= a;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (mj[u] == -INFINITY) continue;             // no weight: o not used
            const float wj = exp2f(mj[u] - Mn);
            acc.x = fmaf(wj, oj[u].x, acc.x);
            acc.y = fmaf(wj, oj[u].y, acc.y);
            acc.z = fmaf(wj, oj[u].z, acc.z);
            acc.w = fmaf(wj, oj[u].w, acc.w);
            lw = fmaf(wj, lj[u], lw);
        }
        Mw = Mn;
    };
    // the first round of loads is issued together with the length
    load(w);
    const int L = (L0 < 0 || L0 > lim) ? 0 : L0;
    const int ns = (L + p.chunk - 1) / p.chunk;
    if (ns <= 1) return;                        // finished by the split kernel
    fold(w, ns);
#pragma unroll 1
    for (int k0 = w + kWarps * kBatch; k0 < ns; k0 += kWarps * kBatch) {
        load(k0);
        fold(k0, ns);
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

// Unweighted partition (seg_w == 0): CTA c of the split kernel starts at item
// c * (T / grid) + min(c, T % grid), so the live slots follow arithmetically.
// One CTA per (b, q head); lane l of a warp owns head_dim [4l, 4l + 4).
__global__ void __launch_bounds__(kThreads)
decode_combine_even(DecodeParams p) {
    __shared__ float s_m[kWarps], s_l[kWarps];
    __shared__ __align__(16) float s_acc[kWarps][128];
    grid_dep_wait();                    // the split kernel's partials are complete
    grid_dep_launch();                  // the next kernel may run its prologue now
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / p.Hq);
    const int hk = static_cast<int>(bh % p.Hq) / p.G;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int* hdr = p.ws_hdr;
    const float* m = p.ws_m + bh * p.splits;
    const float* lv = p.ws_l + bh * p.splits;
    const int D = p.D;
    const bool active = lane * 4 < D;
    const float* o = p.ws_o + bh * p.splits * D + lane * 4;
    const bool direct = p.splits <= kWarps * kBatch;

    // with few slots, every slot's m, l and o are loaded together with the
    // header (one round of loads); the header then says which slots hold
    // partials and the others are dropped unread
    float mj[kBatch], lj[kBatch];
    float4 oj[kBatch];
    if (direct) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = w + u * kWarps;
            const bool in = j < p.splits;
            mj[u] = in ? m[j] : -INFINITY;
            lj[u] = in ? lv[j] : 0.f;
            oj[u] = (in && active) ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    const int T = hdr[0];
    const int ns = hdr[2 + kMaxBatch + 1 + b];
    const int u0 = hdr[2 + b] + hk * ns;        // the unit's first item
    if (ns <= 1) return;
    const int grid = p.grid;
    const int cq = T / grid, cr = T % grid;
    auto cstart = [&](int c) { return c * cq + min(c, cr); };
    auto first_above = [&](int x) {             // smallest c in [1, grid] with cstart(c) > x
        int lo = 1, hi = grid;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (cstart(mid) > x) hi = mid;
            else lo = mid + 1;
        }
        return lo;
    };
    // item x is the first of a CTA block
    auto is_start = [&](int x) {
        const int big = cr * (cq + 1);
        return x < big ? x % (cq + 1) == 0 : (cq > 0 && (x - big) % cq == 0);
    };
    uint32_t live = 1u;                         // direct path: bit j = chunk j holds a partial
    int c_lo = 0, nlive = 0;
    if (direct) {
        const bool bit = lane < ns && (lane == 0 || is_start(u0 + lane));
        live = __ballot_sync(0xffffffffu, bit);
        if (live == 1u) return;                 // one CTA block held the whole unit
    } else {
        c_lo = first_above(u0);
        nlive = 1 + (first_above(u0 + ns - 1) - c_lo);
        if (nlive == 1) return;
    }

    // per-warp online fold over slots, running max Mw, sums lw, acc
    float Mw = -INFINITY, lw = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fold = [&]() {
        float Mn = Mw;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) Mn = fmaxf(Mn, mj[u]);
        if (Mn == -INFINITY) return;
        const float a = exp2f(Mw - Mn);                   // 0 while Mw is -inf
        acc.x *= a; acc.y *= a; acc.z *= a; acc.w *= a;
        lw *= a;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (mj[u] == -INFINITY) continue;             // not a partial: not used
            const float wj = exp2f(mj[u] - Mn);
            acc.x = fmaf(wj, oj[u].x, acc.x);
            acc.y = fmaf(wj, oj[u].y, acc.y);
            acc.z = fmaf(wj, oj[u].z, acc.z);
            acc.w = fmaf(wj, oj[u].w, acc.w);
            lw = fmaf(wj, lj[u], lw);
        }
        Mw = Mn;
    };
    if (direct) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (!((live >> (w + u * kWarps)) & 1u)) mj[u] = -INFINITY;
        fold();
    } else {
        // slots k = w, w + kWarps, ... of the live list, kBatch per round of loads
#pragma unroll 1
        for (int k0 = w; k0 < nlive; k0 += kWarps * kBatch) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int k = k0 + u * kWarps;
                const bool in = k < nlive;
                const int j = k == 0 ? 0 : cstart(c_lo + k - 1) - u0;
                mj[u] = in ? m[j] : -INFINITY;
                lj[u] = in ? lv[j] : 0.f;
                oj[u] = (in && active) ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            fold();
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

// Weighted partition (seg_w != 0): the CTA starts come from the header.
// One CTA per (b, q head); lane l of a warp owns head_dim [4l, 4l + 4).
__global__ void __launch_bounds__(kThreads)
decode_combine_weighted(DecodeParams p) {
    __shared__ float s_m[kWarps], s_l[kWarps];
    __shared__ __align__(16) float s_acc[kWarps][128];
    // dynamic shared memory, sized at launch: the first item of every
    // split-kernel CTA, then the list of live chunks
    extern __shared__ int s_dyn[];
    int* const s_start = s_dyn;                 // [grid + 1]
    grid_dep_wait();                    // the split kernel's partials are complete
    grid_dep_launch();                  // the next kernel may run its prologue now
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / p.Hq);
    const int hk = static_cast<int>(bh % p.Hq) / p.G;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int* hdr = p.ws_hdr;
    const float* m = p.ws_m + bh * p.splits;
    const float* lv = p.ws_l + bh * p.splits;
    const int D = p.D;
    const bool active = lane * 4 < D;
    const float* o = p.ws_o + bh * p.splits * D + lane * 4;
    const bool direct = p.splits <= kWarps * kBatch;

    // with few slots, every slot's m, l and o are loaded together with the
    // header (one round of loads); the header then says which slots hold
    // partials and the others are dropped unread
    float mj[kBatch], lj[kBatch];
    float4 oj[kBatch];
    if (direct) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = w + u * kWarps;
            const bool in = j < p.splits;
            mj[u] = in ? m[j] : -INFINITY;
            lj[u] = in ? lv[j] : 0.f;
            oj[u] = (in && active) ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    const int grid = p.grid;
    const int ns = hdr[kHdrNs + b];
    const int u0 = hdr[kHdrCum + b] + hk * ns;  // the unit's first item
    // CTA blocks from the split kernel's weighted partition, as published
    for (int c = tid; c <= grid; c += kThreads) s_start[c] = hdr[kHdrStart + c];
    __syncthreads();
    if (ns <= 1) return;
    auto start = [&](int c) { return s_start[c]; };
    auto first_at_least = [&](int x) {          // smallest c in [0, grid] with start(c) >= x
        int lo = 0, hi = grid;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (start(mid) >= x) hi = mid;
            else lo = mid + 1;
        }
        return lo;
    };
    auto is_start = [&](int x) { return start(first_at_least(x)) == x; };   // x begins a block
    // the unit's partials: chunk 0, and chunk x - u0 for every CTA block that
    // starts at an item x inside the unit (equal starts are empty blocks)
    uint32_t live = 1u;                         // direct path: bit j = chunk j holds a partial
    int c_lo = 0, c_hi = 0, nlive = 1;
    if (direct) {
        const bool bit = lane < ns && (lane == 0 || is_start(u0 + lane));
        live = __ballot_sync(0xffffffffu, bit);
        if (live == 1u) return;                 // one CTA block held the whole unit
    } else {
        c_lo = first_at_least(u0 + 1);
        c_hi = first_at_least(u0 + ns);
        for (int c = c_lo; c < c_hi; ++c) nlive += (c == c_lo || start(c) != start(c - 1));
        if (nlive == 1) return;
    }

    // per-warp online fold over slots, running max Mw, sums lw, acc
    float Mw = -INFINITY, lw = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fold = [&]() {
        float Mn = Mw;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) Mn = fmaxf(Mn, mj[u]);
        if (Mn == -INFINITY) return;
        const float a = exp2f(Mw - Mn);                   // 0 while Mw is -inf
        acc.x *= a; acc.y *= a; acc.z *= a; acc.w *= a;
        lw *= a;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (mj[u] == -INFINITY) continue;             // not a partial: not used
            const float wj = exp2f(mj[u] - Mn);
            acc.x = fmaf(wj, oj[u].x, acc.x);
            acc.y = fmaf(wj, oj[u].y, acc.y);
            acc.z = fmaf(wj, oj[u].z, acc.z);
            acc.w = fmaf(wj, oj[u].w, acc.w);
            lw = fmaf(wj, lj[u], lw);
        }
        Mw = Mn;
    };
    if (direct) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
            if (!((live >> (w + u * kWarps)) & 1u)) mj[u] = -INFINITY;
        fold();
    } else {
        // the live chunks, in order, are listed once in shared memory
        int* const s_list = s_dyn + grid + 1;     // [grid + 1]
        if (tid == 0) {
            int n = 0;
            s_list[n++] = 0;
            for (int c = c_lo; c < c_hi; ++c)
                if (c == c_lo || start(c) != start(c - 1)) s_list[n++] = start(c) - u0;
        }
        __syncthreads();
        // slots k = w, w + kWarps, ... of the list, kBatch per round of loads
#pragma unroll 1
        for (int k0 = w; k0 < nlive; k0 += kWarps * kBatch) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int k = k0 + u * kWarps;
                const bool in = k < nlive;
                const int j = in ? s_list[k] : 0;
                mj[u] = in ? m[j] : -INFINITY;
                lj[u] = in ? lv[j] : 0.f;
                oj[u] = (in && active) ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            fold();
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
    // the weighted partition's CTA starts and the live-chunk list
    cfg.dynamicSmemBytes = (p.seg_w || p.splits > kWarps * kBatch)
                               ? static_cast<size_t>(2 * (p.grid + 1)) * sizeof(int)
                               : 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (p.one_item) {
        cfg.dynamicSmemBytes = 0;
        return cudaLaunchKernelEx(&cfg, decode_combine_one, p);
    }
    if (p.seg_w == 0) {
        cfg.dynamicSmemBytes = 0;
        return cudaLaunchKernelEx(&cfg, decode_combine_even, p);
    }
    return cudaLaunchKernelEx(&cfg, decode_combine_weighted, p);
}

}  // namespace kvq

// kvq_decode.cu -- decode attention driver: the split kernel (the persistent
// tensor-core one of kvq_decode_tc.cu, or the CUDA-core one of
// kvq_decode_simt.cu) followed, when the plan splits a sequence, by the
// combine kernel below (launched as a programmatic dependent so its launch
// overlaps the split kernel).
//
// Combine (flash-decoding): for each (sequence, q head) whose kv head's
// chunks were split over several CTAs, the partial states (o_k, m_k, l_k) in
// base 2 are merged:
//   M = max_k m_k,  w_k = 2^(m_k - M),  out = sum_k w_k o_k / sum_k w_k l_k.
// A partial sits in the slot of the first chunk of the run of chunks that
// one CTA took.  Which slots hold one: with one item per CTA, every chunk
// below the chunk count; otherwise the split kernel writes m = -inf into
// every other slot below the chunk count, so a unit (sequence, kv head) that
// one CTA took whole (and finished itself) has no finite m at all.
#include <math.h>

#include <atomic>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kBatch = 8;                       // slots in flight per warp

// the cross-warp step: the warps' states (Mw, lw, acc) into the D floats at
// out_row.  With kSkipEmpty, a row with no partial (M = -inf: the split
// kernel wrote it) is left alone.
template <bool kSkipEmpty>
__device__ __forceinline__ void finish_row(float* out_row, int D, float Mw, float lw, float4 acc,
                                           float* s_m, float* s_l, float (*s_acc)[128]) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (lane == 0) {
        s_m[w] = Mw;
        s_l[w] = lw;
    }
    if (lane * 4 < D) *reinterpret_cast<float4*>(&s_acc[w][lane * 4]) = acc;
    __syncthreads();
    float M = s_m[0];
#pragma unroll
    for (int x = 1; x < kWarps; ++x) M = fmaxf(M, s_m[x]);
    if (kSkipEmpty && M == -INFINITY) return;
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
        out_row[d] = lsum > 0.f ? sum / lsum : 0.f;
    }
}

// One item per CTA (one_item): CTA c of the split kernel held item c of the
// plan, so chunk j < ns of every unit holds a partial and nothing else does.
// One CTA per (b, q head) and 128 columns of head_dim (blockIdx.y: columns
// 128 y ..); lane l of a warp owns columns [4l, 4l + 4) of those.
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
    const int dh = 128 * static_cast<int>(blockIdx.y);   // this CTA's first column
    const bool active = dh + lane * 4 < D;
    const float* o = p.ws_o + bh * p.splits * D + dh + lane * 4;
    const int64_t cap = p.page_size ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t plan = static_cast<int64_t>(p.splits) * p.chunk;
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
    const int L = max(walked_len(L0, cap, plan, p.qlen, p.window, p.recent), 0);
    const int ns = (L + p.chunk - 1) / p.chunk;
    if (ns <= 1) return;                        // finished by the split kernel
    fold(w, ns);
#pragma unroll 1
    for (int k0 = w + kWarps * kBatch; k0 < ns; k0 += kWarps * kBatch) {
        load(k0);
        fold(k0, ns);
    }
    finish_row<false>(p.out + bh * D + dh, min(D - dh, 128), Mw, lw, acc, s_m, s_l, s_acc);
}

// Blocks of several items per CTA (one_item == 0): a unit's partials are its
// chunk slots j < ns with finite m.  The first kWords * 32 m slots are loaded
// together with the length; a ballot per 32 slots picks the live ones, and
// warp w loads and folds those with j % kWarps == w (at most kBatch per 32
// slots).  One CTA per (b, q head) and 128 columns of head_dim (blockIdx.y);
// lane l of a warp owns columns [4l, 4l + 4) of those.
constexpr int kWords = 4;
__global__ void __launch_bounds__(kThreads)
decode_combine_live(DecodeParams p) {
    __shared__ float s_m[kWarps], s_l[kWarps];
    __shared__ __align__(16) float s_acc[kWarps][128];
    grid_dep_wait();                    // the split kernel's partials are complete
    grid_dep_launch();                  // the next kernel may run its prologue now
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / p.Hq);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const float* m = p.ws_m + bh * p.splits;
    const float* lv = p.ws_l + bh * p.splits;
    const int D = p.D;
    const int dh = 128 * static_cast<int>(blockIdx.y);   // this CTA's first column
    const bool active = dh + lane * 4 < D;
    const float* o = p.ws_o + bh * p.splits * D + dh + lane * 4;
    const int64_t cap = p.page_size ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t plan = static_cast<int64_t>(p.splits) * p.chunk;
    const int L0 = p.seq_lens[b];
    float mv0[kWords];
#pragma unroll
    for (int x = 0; x < kWords; ++x) {
        const int j = 32 * x + lane;
        mv0[x] = j < p.splits ? m[j] : -INFINITY;
    }
    const int L = max(walked_len(L0, cap, plan, p.qlen, p.window, p.recent), 0);
    const int ns = (L + p.chunk - 1) / p.chunk;
    if (ns <= 1) return;                        // finished by the split kernel

    float Mw = -INFINITY, lw = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // slots base .. base + 31, lane's m value mv
    auto word = [&](int base, float mv) {
        const bool live = base + lane < ns && mv != -INFINITY;
        uint32_t bits = __ballot_sync(0xffffffffu, live) & (0x11111111u << w);
        if (bits == 0u) return;
        float mj[kBatch], lj[kBatch];
        float4 oj[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const bool in = bits != 0u;
            const int pos = in ? __ffs(bits) - 1 : 0;
            bits &= bits - 1u;
            const int j = base + pos;
            const float mp = __shfl_sync(0xffffffffu, mv, pos);
            mj[u] = in ? mp : -INFINITY;
            lj[u] = in ? lv[j] : 0.f;
            oj[u] = (in && active) ? *reinterpret_cast<const float4*>(o + static_cast<int64_t>(j) * D)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float Mn = Mw;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) Mn = fmaxf(Mn, mj[u]);
        const float a = exp2f(Mw - Mn);                   // 0 while Mw is -inf
        acc.x *= a; acc.y *= a; acc.z *= a; acc.w *= a;
        lw *= a;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            if (mj[u] == -INFINITY) continue;
            const float wj = exp2f(mj[u] - Mn);
            acc.x = fmaf(wj, oj[u].x, acc.x);
            acc.y = fmaf(wj, oj[u].y, acc.y);
            acc.z = fmaf(wj, oj[u].z, acc.z);
            acc.w = fmaf(wj, oj[u].w, acc.w);
            lw = fmaf(wj, lj[u], lw);
        }
        Mw = Mn;
    };
#pragma unroll
    for (int x = 0; x < kWords; ++x)
        if (32 * x < ns) word(32 * x, mv0[x]);
#pragma unroll 1
    for (int base = 32 * kWords; base < ns; base += 32)
        word(base, base + lane < ns ? m[base + lane] : -INFINITY);
    finish_row<true>(p.out + bh * D + dh, min(D - dh, 128), Mw, lw, acc, s_m, s_l, s_acc);
}

// Dynamic shared memory for decode_combine_one so that at most k =
// ceil(rows / SMs) of its CTAs share an SM.  The combine launches early, next
// to the split kernel, and without this its CTAs crowd onto the few SMs the
// split kernel leaves idle, where the L2 reads of the partials queue behind
// one another.  0 when the attributes cannot be read or k > 2.  The device
// figures are read once per device.
constexpr int kMaxDevices = 64;
std::atomic<int> g_spread_state[kMaxDevices];   // 0 not read, 1 ready, -1 unavailable
int g_spread_sms[kMaxDevices];
int g_spread_dyn[kMaxDevices][2];                // bytes for k = 1, 2

size_t combine_one_spread_smem(int rows) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    int st = g_spread_state[dev].load(std::memory_order_acquire);
    if (st == 0) {
        int sms = 0, cap = 0, reserved = 0;
        cudaFuncAttributes fa;
        st = -1;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&cap, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
                cudaSuccess &&
            cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) ==
                cudaSuccess &&
            cudaFuncGetAttributes(&fa, decode_combine_one) == cudaSuccess && sms > 0) {
            // a CTA's footprint F = cap / k: k of them fit on an SM, k + 1 do not
            for (int k = 1; k <= 2; ++k)
                g_spread_dyn[dev][k - 1] = static_cast<int>(
                    (cap / k - static_cast<long long>(fa.sharedSizeBytes) - reserved) / 16 * 16);
            g_spread_sms[dev] = sms;
            if (g_spread_dyn[dev][1] > 0 &&
                cudaFuncSetAttribute(decode_combine_one, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     g_spread_dyn[dev][0]) == cudaSuccess)
                st = 1;
        }
        g_spread_state[dev].store(st, std::memory_order_release);
    }
    if (st < 0) return 0;
    const int k = (rows + g_spread_sms[dev] - 1) / g_spread_sms[dev];
    return k <= 2 ? static_cast<size_t>(g_spread_dyn[dev][k - 1]) : 0;
}

}  // namespace

// Mixed cache (abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
// OptimizedQuantizedKvCache::get_kv: the INT8 part dequantised, then the
// unquantised recent tokens): one CTA per (b, kv head) and its G query heads.
// The newest min(L, W) tokens sit in the bf16 ring (position g in row g % W);
// they are walked in tiles of kRecTile tokens staged in shared memory (K and V
// rows by 16-byte loads), with an online softmax per head in fp32: scores by
// one warp per token (lanes over head_dim, all G heads at once), then each
// thread updates its (head, head_dim) outputs from the tile's V rows.  The
// split kernel's INT8 partials (every slot below the INT8 part's chunk count
// with a finite m) are folded in at the end and the rows written.
constexpr int kRecThreads = 256;
constexpr int kRecWarps = kRecThreads / 32;
constexpr int kRecTile = 16;                    // window tokens per shared-memory tile
constexpr int kRecMaxG = 16;
__global__ void __launch_bounds__(kRecThreads)
decode_recent_combine(DecodeParams p) {
    __shared__ __align__(16) float s_q[kRecMaxG * 256];             // the G query rows (fp32)
    __shared__ __align__(16) uint16_t s_k[kRecTile * 256], s_v[kRecTile * 256];
    __shared__ float s_p[kRecMaxG][kRecTile];                       // scores, then weights
    __shared__ float s_m[kRecMaxG], s_l[kRecMaxG], s_a[kRecMaxG];   // running max, sum, rescale
    grid_dep_wait();                    // the split kernel's partials are complete
    grid_dep_launch();
    const int unit = blockIdx.x;                        // b * Hk + hk
    const int b = unit / p.Hk;
    const int G = p.G, D = p.D, W = p.recent;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh0 = static_cast<int64_t>(unit) * G;  // first q row (b * Hq + hk * G)
    const int64_t cap = p.page_size ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t plan = static_cast<int64_t>(p.splits) * p.chunk;
    const int L = p.seq_lens[b];
    const int n8 = walked_len(L, cap, plan, 1, 0, W);   // INT8 part walked by the split kernel
    if (n8 < 0) {                                       // flagged by the split kernel
        for (int i = tid; i < G * D; i += kRecThreads) p.out[bh0 * D + i] = 0.f;
        return;
    }
    const int Lq = L > W ? L - W : 0;
    const int nr = L - Lq;                              // tokens in the window
    for (int i = tid; i < G * D; i += kRecThreads)
        s_q[i] = bf16_bits_to_f32(p.q[bh0 * D + i]);
    if (tid < G) {
        s_m[tid] = -INFINITY;
        s_l[tid] = 0.f;
    }
    // this thread's (head, head_dim) outputs: pairs tid + kRecThreads * k
    constexpr int kMaxPairs = kRecMaxG * 256 / kRecThreads;
    float o[kMaxPairs];
#pragma unroll
    for (int k = 0; k < kMaxPairs; ++k) o[k] = 0.f;
    const int npair = G * D;
    const int64_t ring0 = static_cast<int64_t>(unit) * W;
    const int vec = D / 8;                              // 16-byte chunks per row
    for (int i0 = 0; i0 < nr; i0 += kRecTile) {
        const int n = min(kRecTile, nr - i0);
        __syncthreads();                                // the previous tile is consumed
        for (int c = tid; c < n * vec; c += kRecThreads) {
            const int t = c / vec, x = c % vec;
            const int64_t row = ring0 + (Lq + i0 + t) % W;
            reinterpret_cast<uint4*>(s_k)[t * vec + x] =
                reinterpret_cast<const uint4*>(p.rk + row * D)[x];
            reinterpret_cast<uint4*>(s_v)[t * vec + x] =
                reinterpret_cast<const uint4*>(p.rv + row * D)[x];
        }
        __syncthreads();
        // scores (log2 domain): one warp per token, lanes over head_dim
        for (int t = warp; t < n; t += kRecWarps) {
            float acc[kRecMaxG];
#pragma unroll
            for (int h = 0; h < kRecMaxG; ++h) acc[h] = 0.f;
            for (int d = lane; d < D; d += 32) {
                const float kv = bf16_bits_to_f32(s_k[t * D + d]);
#pragma unroll
                for (int h = 0; h < kRecMaxG; ++h)
                    if (h < G) acc[h] = fmaf(s_q[h * D + d], kv, acc[h]);
            }
#pragma unroll
            for (int h = 0; h < kRecMaxG; ++h) {
                if (h >= G) break;
                float a = acc[h];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
                if (lane == 0) s_p[h][t] = a * p.scale_log2;
            }
        }
        __syncthreads();
        // online softmax per head (one thread per head)
        if (tid < G) {
            float mt = -INFINITY;
            for (int t = 0; t < n; ++t) mt = fmaxf(mt, s_p[tid][t]);
            const float mn = fmaxf(s_m[tid], mt);
            const float a = exp2f(s_m[tid] - mn);       // 0 while the max was -inf
            float add = 0.f;
            for (int t = 0; t < n; ++t) {
                const float e = exp2f(s_p[tid][t] - mn);
                s_p[tid][t] = e;
                add += e;
            }
            s_l[tid] = s_l[tid] * a + add;
            s_m[tid] = mn;
            s_a[tid] = a;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kMaxPairs; ++k) {
            const int idx = tid + kRecThreads * k;
            if (idx >= npair) break;
            const int h = idx / D, d = idx % D;
            float acc = o[k] * s_a[h];
            for (int t = 0; t < n; ++t) acc = fmaf(s_p[h][t], bf16_bits_to_f32(s_v[t * D + d]), acc);
            o[k] = acc;
        }
    }
    __syncthreads();
    // the INT8 partials of each head: their max and weighted sum (warp per head)
    const int ns = (n8 + p.chunk - 1) / p.chunk;
    for (int h = warp; h < G; h += kRecWarps) {
        const float* m8 = p.ws_m + (bh0 + h) * p.splits;
        const float* l8 = p.ws_l + (bh0 + h) * p.splits;
        float M = s_m[h];
        for (int j = lane; j < ns; j += 32) M = fmaxf(M, m8[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float ls = 0.f;
        for (int j = lane; j < ns; j += 32)
            if (m8[j] != -INFINITY) ls = fmaf(exp2f(m8[j] - M), l8[j], ls);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        if (lane == 0) {
            const float aw = s_m[h] == -INFINITY ? 0.f : exp2f(s_m[h] - M);
            const float tot = ls + s_l[h] * aw;
            s_a[h] = aw;                                // the window's weight
            s_l[h] = tot > 0.f ? 1.f / tot : 0.f;       // the normaliser
            s_m[h] = M;
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kMaxPairs; ++k) {
        const int idx = tid + kRecThreads * k;
        if (idx >= npair) break;
        const int h = idx / D, d = idx % D;
        const int64_t row = bh0 + h;
        const float M = s_m[h];
        const float* m8 = p.ws_m + row * p.splits;
        const float* o8 = p.ws_o + row * p.splits * D + d;
        float acc = o[k] * s_a[h];
        int j = 0;
        for (; j + 4 <= ns; j += 4) {                   // four slots' loads in flight
            float mj[4], oj[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                mj[u] = m8[j + u];
                oj[u] = o8[static_cast<int64_t>(j + u) * D];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (mj[u] != -INFINITY) acc = fmaf(exp2f(mj[u] - M), oj[u], acc);
        }
        for (; j < ns; ++j) {
            const float mj = m8[j];
            if (mj != -INFINITY) acc = fmaf(exp2f(mj - M), o8[static_cast<int64_t>(j) * D], acc);
        }
        p.out[row * D + d] = acc * s_l[h];
    }
}

cudaError_t launch_recent_combine(const DecodeParams& p, cudaStream_t s) {
    if (p.recent < 1 || p.recent > kMaxRecent || p.G > kRecMaxG || p.D > 256 || p.qlen != 1)
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.B * p.Hk, 1, 1);
    cfg.blockDim = dim3(kRecThreads, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_recent_combine, p);
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s, bool simt) {
    cudaError_t e = simt ? launch_decode_simt(p, s) : launch_decode_split_tc(p, s);
    if (e != cudaSuccess || p.splits <= 1) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.B * p.Hq, (p.D + 127) / 128, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (p.one_item) {
        cfg.dynamicSmemBytes = combine_one_spread_smem(p.B * p.Hq);
        return cudaLaunchKernelEx(&cfg, decode_combine_one, p);
    }
    return cudaLaunchKernelEx(&cfg, decode_combine_live, p);
}

}  // namespace kvq

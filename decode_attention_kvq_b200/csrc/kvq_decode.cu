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

#include "kvq_devonce.h"
#include "kvq_internal.cuh"
#include "kvq_ptx.cuh"

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
// unquantised recent tokens): a cluster of kRecParts CTAs per (b, q head).
// The newest min(L, W) tokens sit in the bf16 ring of the head's kv head
// (position g in row g % W); CTA (cluster rank) r takes the r-th quarter of
// them and the row's INT8 partial slots j with j % kRecParts == r (every
// slot below the INT8 part's chunk count with a finite m).  Its window
// tokens are walked in tiles of up to tw tokens (all of them when they fit
// the dynamic shared memory), each tile's K and V rows brought in by one
// round of asynchronous 16-byte copies, with an online softmax in fp32: the
// tile's scores by the eight warps (a warp per token, lanes over head_dim),
// its maximum and weights by one warp (lanes over tokens), then P.V with the
// tokens split among the threads of each output value.  Its slots' m, l and
// values are loaded before the window work, so their latency overlaps it.
// Each CTA leaves its state (max M, sum l and unnormalised output, relative
// to M) in shared memory; after a cluster barrier rank 0 reads the others'
// through distributed shared memory and writes the row, and a second
// barrier keeps every CTA's shared memory alive until it has.
namespace {
constexpr int kRecThreads = 256;
constexpr int kRecWarps = kRecThreads / 32;
constexpr int kRecParts = 4;                    // CTAs (one cluster) per (b, q head)
constexpr int kRecSmem = 96 * 1024;             // dynamic shared memory budget of a tile
constexpr int kRecMaxSlots = 64;                // INT8 partials staged per round
constexpr int kRecPre = 16;                     // partial slots prefetched into registers

int recent_tile(int W, int D) {                 // window tokens per tile (per CTA)
    const int w = (W + kRecParts - 1) / kRecParts;
    const int fit = (kRecSmem - 64) / (4 * D + 4);
    return w < fit ? w : fit;
}
size_t recent_smem(int tw, int D) { return static_cast<size_t>(tw) * (4 * D + 4); }

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a float in CTA `rank`'s shared memory at this CTA's address `a` of the same variable
__device__ __forceinline__ float ld_peer_f32(uint32_t a, uint32_t rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

__global__ void __cluster_dims__(kRecParts, 1, 1) __launch_bounds__(kRecThreads)
decode_recent_combine(DecodeParams p, int tw) {
    extern __shared__ __align__(16) uint8_t rec_smem[];
    uint16_t* s_k = reinterpret_cast<uint16_t*>(rec_smem);            // [tw][D]
    uint16_t* s_v = s_k + static_cast<size_t>(tw) * p.D;              // [tw][D]
    float* s_p = reinterpret_cast<float*>(s_v + static_cast<size_t>(tw) * p.D);   // [tw]
    __shared__ __align__(16) float s_q[256];                          // the query row (fp32)
    __shared__ float s_st[4];                                         // m, l, tile rescale
    __shared__ float s_m8[kRecMaxSlots], s_l8[kRecMaxSlots];
    __shared__ __align__(16) float s_red[kRecThreads];                // P.V part sums
    __shared__ __align__(16) float s_fo[256];                         // this CTA's state
    __shared__ float s_fm, s_fl;
    grid_dep_wait();                    // the split kernel's partials are complete
    grid_dep_launch();
    const int r = static_cast<int>(cluster_rank());
    const int64_t row = blockIdx.x / kRecParts;         // b * Hq + q head
    const int b = static_cast<int>(row / p.Hq);
    const int unit = static_cast<int>(row / p.G);       // b * Hk + kv head
    const int D = p.D, W = p.recent;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t cap = p.page_size ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t plan = static_cast<int64_t>(p.splits) * p.chunk;
    const int L = p.seq_lens[b];
    const int n8 = walked_len(L, cap, plan, 1, 0, W);   // INT8 part walked by the split kernel
    if (n8 < 0) {                                       // flagged by the split kernel
        // (the same for every CTA of the cluster: all of them leave here)
        if (r == 0)
            for (int d = tid; d < D; d += kRecThreads) p.out[row * D + d] = 0.f;
        return;
    }
    const int Lq = L > W ? L - W : 0;
    const int nr = L - Lq;                              // tokens in the window
    const int i_lo = static_cast<int>(static_cast<int64_t>(nr) * r / kRecParts);
    const int i_hi = static_cast<int>(static_cast<int64_t>(nr) * (r + 1) / kRecParts);
    const int ns = (n8 + p.chunk - 1) / p.chunk;        // INT8 partial slots
    const int nsr = ns > r ? (ns - r + kRecParts - 1) / kRecParts : 0;   // this CTA's slots
    const float* m8 = p.ws_m + row * p.splits;
    const float* l8 = p.ws_l + row * p.splits;
    const float* o8 = p.ws_o + row * p.splits * D + (tid < D ? tid : 0);
    // the first of this CTA's slots (j = r + kRecParts u): m, l (shared) and
    // this thread's values (registers)
    const int npre = min(nsr, kRecPre);
    if (tid < npre) {
        s_m8[tid] = m8[r + kRecParts * tid];
        s_l8[tid] = l8[r + kRecParts * tid];
    }
    float ovp[kRecPre];
#pragma unroll
    for (int u = 0; u < kRecPre; ++u)
        ovp[u] = u < npre ? o8[static_cast<int64_t>(r + kRecParts * u) * D] : 0.f;
    for (int d = tid; d < D; d += kRecThreads) s_q[d] = bf16_bits_to_f32(p.q[row * D + d]);
    if (tid == 0) {
        s_st[0] = -INFINITY;
        s_st[1] = 0.f;
    }
    float o = 0.f;                                      // output value d = tid
    const int64_t ring0 = static_cast<int64_t>(unit) * W;
    const int vec = D / 8;                              // 16-byte chunks per row
    const uint32_t sk_a = ptx::smem_u32(s_k), sv_a = ptx::smem_u32(s_v);
    const int parts = D <= kRecThreads / 2 ? kRecThreads / D : 1;   // P.V threads per value
    for (int i0 = i_lo; i0 < i_hi; i0 += tw) {
        const int n = min(tw, i_hi - i0);
        __syncthreads();                                // the previous tile is consumed
        for (int c = tid; c < n * vec; c += kRecThreads) {
            const int t = c / vec, x = c - (c / vec) * vec;
            const int64_t rr = ring0 + (Lq + i0 + t) % W;
            ptx::cp_async_16(sk_a + 16u * static_cast<uint32_t>(c), p.rk + rr * D + 8 * x);
            ptx::cp_async_16(sv_a + 16u * static_cast<uint32_t>(c), p.rv + rr * D + 8 * x);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
        // scores (log2 domain): a warp takes four tokens at a time (lanes over
        // head_dim), their four reduction trees interleaved
        for (int t0 = 4 * warp; t0 < n; t0 += 4 * kRecWarps) {
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int d = lane; d < D; d += 32) {
                const float qd = s_q[d];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (t0 + u < n) a[u] = fmaf(qd, bf16_bits_to_f32(s_k[(t0 + u) * D + d]), a[u]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int u = 0; u < 4; ++u) a[u] += __shfl_xor_sync(0xffffffffu, a[u], off);
            if (lane < 4 && t0 + lane < n) {
                const float v = lane == 0 ? a[0] : lane == 1 ? a[1] : lane == 2 ? a[2] : a[3];
                s_p[t0 + lane] = v * p.scale_log2;
            }
        }
        __syncthreads();
        // online softmax over the tile: one warp, lanes over tokens
        if (warp == 0) {
            float mt = -INFINITY;
            for (int t = lane; t < n; t += 32) mt = fmaxf(mt, s_p[t]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float mo = s_st[0];
            const float mn = fmaxf(mo, mt);
            float add = 0.f;
            for (int t = lane; t < n; t += 32) {
                const float e = exp2f(s_p[t] - mn);
                s_p[t] = e;
                add += e;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) add += __shfl_xor_sync(0xffffffffu, add, off);
            if (lane == 0) {
                const float a = exp2f(mo - mn);         // 0 while the max was -inf
                s_st[1] = s_st[1] * a + add;
                s_st[0] = mn;
                s_st[2] = a;
            }
        }
        __syncthreads();
        // P.V: the tile's tokens split among `parts` threads per output value
        // (token t to part t % parts), four partial sums each, then summed
        // into the running value by the part-0 threads
        {
            const int part = tid / D, d = tid - part * D;
            if (part < parts) {
                float ac[4] = {0.f, 0.f, 0.f, 0.f};
                int t = part;
                for (; t + 3 * parts < n; t += 4 * parts)
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        ac[u] = fmaf(s_p[t + u * parts],
                                     bf16_bits_to_f32(s_v[(t + u * parts) * D + d]), ac[u]);
                for (; t < n; t += parts) ac[0] = fmaf(s_p[t], bf16_bits_to_f32(s_v[t * D + d]), ac[0]);
                s_red[tid] = (ac[0] + ac[1]) + (ac[2] + ac[3]);
            }
            __syncthreads();
            if (tid < D) {
                float sum = o * s_st[2];
                for (int q = 0; q < parts; ++q) sum += s_red[q * D + tid];
                o = sum;
            }
        }
    }
    __syncthreads();
    // this CTA's INT8 partials: their maximum and weighted sum; empty slots
    // (m = -inf) are dropped by selection (no load behind a branch)
    float M = s_st[0];
    float lsum = 0.f;                                   // relative to M, the window's l not included
    float acc = 0.f;
    const float mw = s_st[0], lw = s_st[1];
    auto rescale = [&](int nj) {                        // the new maximum over nj staged slots
        float Mn = M;
        for (int j = 0; j < nj; ++j) Mn = fmaxf(Mn, s_m8[j]);
        const float a = M == -INFINITY ? 0.f : exp2f(M - Mn);
        acc *= a;
        lsum *= a;
        M = Mn;
    };
    auto add = [&](int j, float value) {                // staged slot j with this thread's value
        const float mj = s_m8[j];
        const bool live = mj != -INFINITY;
        const float w = live ? exp2f(mj - M) : 0.f;
        acc = live ? fmaf(w, value, acc) : acc;
        lsum = live ? fmaf(w, s_l8[j], lsum) : lsum;
    };
    rescale(npre);
#pragma unroll
    for (int u = 0; u < kRecPre; ++u)
        if (u < npre) add(u, ovp[u]);
#pragma unroll 1
    for (int u0 = npre; u0 < nsr; u0 += kRecMaxSlots) {
        const int nj = min(kRecMaxSlots, nsr - u0);
        __syncthreads();                                // s_m8, s_l8 free
        if (tid < nj) {
            s_m8[tid] = m8[r + kRecParts * (u0 + tid)];
            s_l8[tid] = l8[r + kRecParts * (u0 + tid)];
        }
        __syncthreads();
        rescale(nj);
        for (int j = 0; j < nj; ++j) add(j, o8[static_cast<int64_t>(r + kRecParts * (u0 + j)) * D]);
    }
    // this CTA's state, relative to its maximum M
    {
        const float aw = mw == -INFINITY ? 0.f : exp2f(mw - M);
        if (tid == 0) {
            s_fm = M;
            s_fl = lsum + lw * aw;
        }
        if (tid < D) s_fo[tid] = acc + o * aw;
    }
    cluster_sync_all();                                 // every CTA's state is written
    if (r == 0) {
        float fm[kRecParts], fl[kRecParts], fo[kRecParts];
        const uint32_t am = ptx::smem_u32(&s_fm), al = ptx::smem_u32(&s_fl);
        const uint32_t ao = ptx::smem_u32(&s_fo[tid < D ? tid : 0]);
#pragma unroll
        for (int q = 0; q < kRecParts; ++q) {
            fm[q] = ld_peer_f32(am, q);
            fl[q] = ld_peer_f32(al, q);
            fo[q] = tid < D ? ld_peer_f32(ao, q) : 0.f;
        }
        float Mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < kRecParts; ++q) Mx = fmaxf(Mx, fm[q]);
        float tot = 0.f, val = 0.f;
#pragma unroll
        for (int q = 0; q < kRecParts; ++q) {
            const float w = fm[q] == -INFINITY ? 0.f : exp2f(fm[q] - Mx);
            tot = fmaf(w, fl[q], tot);
            val = fmaf(w, fo[q], val);
        }
        if (tid < D) p.out[row * D + tid] = tot > 0.f ? val / tot : 0.f;
    }
    cluster_sync_all();                                 // rank 0 has read every CTA's state
}

}  // namespace

cudaError_t launch_recent_combine(const DecodeParams& p, cudaStream_t s) {
    if (p.recent < 1 || p.recent > kMaxRecent || p.D > 256 || p.qlen != 1 ||
        static_cast<int64_t>(p.B) * p.Hq * kRecParts > 0x7fffffffll)
        return cudaErrorInvalidValue;
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = once_per_device(done, dev, cudaSuccess, [] {
        return cudaFuncSetAttribute(decode_recent_combine,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kRecSmem);
    });
    if (e != cudaSuccess) return e;
    const int tw = recent_tile(p.recent, p.D);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(p.B) * p.Hq * kRecParts), 1, 1);
    cfg.blockDim = dim3(kRecThreads, 1, 1);
    cfg.dynamicSmemBytes = recent_smem(tw, p.D);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_recent_combine, p, tw);
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

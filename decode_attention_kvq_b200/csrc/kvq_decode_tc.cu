// kvq_decode_tc.cu -- decode attention on the INT8 cache for sm_100a:
// a persistent split-K kernel with a TMA-fed shared-memory ring and
// tensor-core Q.K^T and P.V on exact integer operands, the dequantisation
// scales applied outside the MMA.
//
// Method (what is computed): abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
// module doc "Fused approach" -- Q.K^T with K dequantised on the fly,
// softmax, P.V with V dequantised on the fly; combs-models 0.2.2, src/kv.rs,
// attend / repeat_kv -- scale after the dot product, query head h reads kv
// head h / G, a decode query attends to the whole cache.  Split-K with an
// online softmax and the combine are this library's own (flash-decoding).
//
// How (sm_100a):
//  * Work items are (sequence b, kv head, chunk j) with chunk = p.chunk
//    tokens, listed in (b, kv head, j) order.  The grid is persistent (at
//    most one CTA per SM) and CTA c takes the contiguous block
//    [c*T/grid, (c+1)*T/grid) of the T items, found from a prefix sum of the
//    per-sequence chunk counts (sequence lengths cached in shared memory).
//    Consecutive chunks of one (b, kv head) inside a CTA's block form a
//    segment and share one softmax state; a segment that is a whole
//    sequence writes the final rows, any other writes one partial state
//    (o, m, l) into the slot of its first chunk and marks the slots of its
//    other chunks empty for the combine kernel (kvq_decode.cu).
//  * CTA = 8 consumer warps + 1 producer warp.  The producer streams
//    128-token stages into a ring of 3-8 stages (~150-180 KB of shared
//    memory, one CTA per SM): K and V bytes by TMA tile loads (2-D tensor
//    maps over the cache rows, 128-byte swizzle for D=128, 64-byte for
//    D=64), the fp32 scales and, with a segment's first stage, its query
//    rows by cp.async; all complete on the stage's mbarrier.  It refills a
//    slot as soon as all consumers released it, independent of their
//    progress elsewhere.  Every consumer warp takes one 16-token slice of
//    each stage.
//  * Per slice, on mma.sync m16n8k16 (f16 in, f32 accumulate), with the
//    query heads of the GQA group as the N = 8 dimension (two n-tiles when
//    G > 8):  S^T = K . Q^T (M = 16 tokens, K = head_dim) and
//    O^T += V^T . P^T (M = 16 head_dim rows, K = 16 tokens).  The operands
//    are exact: K and V enter as the integers (byte - 128) built in
//    registers (1024 + byte spliced into an f16 mantissa, minus 1152), and Q
//    enters as f16 after a per-head power-of-two prescale (bf16 has 8
//    significant bits, f16 has 11, so q * 2^s is exact).  The K scale (per
//    token, or per 32-value group with one accumulator per group), 2^-s,
//    attn_scale and log2(e) are applied to the f32 scores.
//  * Online softmax in base 2 per head.  The V scale is folded into P:
//    P'' = 2^(z-m) * v_scale(token) * 2^kv (per 32-value group in group-32
//    mode), with a running per-warp power of two 2^kv that keeps P'' inside
//    the f16 normal range.  P'' is split into f16 hi + lo parts (about 22
//    significant bits together); each part is transposed from the score
//    accumulator layout into the P^T operand layout with movmatrix and
//    multiplied with the exact (v - 128) integers.
//  * Token order inside each 16-token slice and the head_dim order of the
//    MMA k-dimension are permuted so that every shared-memory load of the
//    swizzled tiles is free of bank conflicts (sigma below).
//  * A segment's eight warp states are merged in one round through eight
//    shared-memory slots in register order (deterministic: no atomics).
//  * Programmatic dependent launch: the kernel waits for its predecessor in
//    the stream before touching inputs and lets the combine kernel launch
//    early.
//  * mbarrier waits are bounded (KVQ_DEVERR_TIMEOUT when one gives up, after
//    which every wait of the CTA returns at once); barriers are reached by
//    every participating thread unconditionally.
#include <cuda.h>
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

constexpr int NW = 8;                  // consumer warps per CTA
constexpr int NCONS = NW * 32;         // consumer threads
constexpr int NTHREADS = NCONS + 32;   // + the producer warp
constexpr int TT = 16 * NW;            // tokens per stage: one 16-token slice per warp
constexpr int kMaxB = 1024;            // sequences whose lengths are cached in shared memory

// Row (inside an 8-token half of a slice) that holds MMA row r of the K
// operand and MMA k-index r of the V operand: sigma = {0, 2, 4, 6, 3, 1, 7, 5}.
// Under the 128-byte swizzle (16-byte chunk index XOR row % 8) the rows that
// one load instruction touches then differ in bits 1..2, so the K loads
// (rows sigma(g), 8 bytes at 32*G + 8*t) and the V loads (rows sigma(2t),
// sigma(2t+1), 16 bytes at 16*g) of a warp hit distinct banks.
__device__ __forceinline__ int sigma(int x) { return x < 4 ? 2 * x : ((2 * x - 7) ^ 2); }

// (a, b) -> f16x2 hi = rn(a, b) and lo = rn(a - hi, b - hi): hi + lo carries
// about 22 significant bits of each value.
__device__ __forceinline__ void split_f16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 f = __half22float2(h);
    const __half2 l = __floats2half2_rn(a - f.x, b - f.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// 8x8 b16 transpose across the warp (fragment of row lane/4, columns
// 2*(lane%4) and +1, in and out).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// The NG fp32 scales of one token (4, 8 or 16 bytes, aligned to their size
// because the scale array is 16-byte aligned and rows are NG floats apart).
template <int NG>
__device__ __forceinline__ void copy_scales(uint32_t dst, const float* src) {
    static_assert(NG == 1 || NG == 2 || NG == 4, "scales per token");
    if constexpr (NG == 1) ptx::cp_async_4(dst, src);
    else if constexpr (NG == 2) ptx::cp_async_8(dst, src);
    else ptx::cp_async_16(dst, src);
}

// Shared-memory plan (one CTA per SM): a ring of NST stages (K and V bytes of
// 128 tokens, their scales, room for one segment's query rows), the merge
// slots, the cached lengths and chunk prefix sums, the stage mbarriers and
// per-warp head maxima.
template <int D, bool G32, bool G16>
struct Layout {
    static constexpr int NG = G32 ? D / 32 : 1;
    static constexpr int KV_BYTES = TT * D;
    static constexpr int SC_FLOATS = TT * NG;
    static constexpr int Q_OFF = 2 * KV_BYTES + 2 * SC_FLOATS * 4;   // within a stage
    static constexpr int Q_BYTES = (G16 ? 16 : 8) * D * 2;           // bf16 query rows
    static constexpr int STAGE = ((Q_OFF + Q_BYTES) + 1023) / 1024 * 1024;
    static constexpr int NV = (G16 ? 2 : 1) * (D / 16) * 4;        // o floats per lane
    static constexpr int MERGE_BYTES = NW * NV * 32 * 4;
    static constexpr int LENS_BYTES = 2 * (kMaxB + 1) * 4;          // lengths, prefix sums
    static constexpr int MISC_BYTES = 2048;                         // barriers, maxima, flags
    static constexpr int BUDGET = 227 * 1024 - 1024 - MERGE_BYTES - LENS_BYTES - MISC_BYTES;
    static constexpr int NST = (BUDGET / STAGE) > 8 ? 8 : (BUDGET / STAGE);
    static_assert(NST >= 3, "at least three stages");
    static constexpr int MERGE_OFF = NST * STAGE;
    static constexpr int LENS_OFF = MERGE_OFF + MERGE_BYTES;
    static constexpr int MISC_OFF = LENS_OFF + LENS_BYTES;
    static constexpr int SMEM = MISC_OFF + MISC_BYTES + 1024;       // + base alignment slack
    static_assert(SMEM <= 227 * 1024, "fits one SM");
};

// byte offset of (row, byte) inside a swizzled K or V stage tile
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t byte) {
    if constexpr (D == 128) {
        return row * 128u + ((((byte >> 4) ^ row) & 7u) << 4) + (byte & 15u);
    } else {  // D == 64, 64-byte swizzle
        return row * 64u + ((((byte >> 4) ^ (row >> 1)) & 3u) << 4) + (byte & 15u);
    }
}

__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ float ldsf(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

// One work item of a CTA's block: item index -> (b, kv head, chunk j).
struct Item {
    int b, hk, j, ns, L, t0, t1;   // ns = chunks of the sequence (0: empty sequence)
};

// cum[b] = items of sequences < b (each sequence has Hk * max(1, ns_b) items)
__device__ __forceinline__ Item item_at(int64_t i, const int* lens, const int* cum, int B,
                                        int Hk, int chunk) {
    int lo = 0, hi = B;                  // largest b with cum[b] <= i
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= i) lo = mid;
        else hi = mid;
    }
    Item it;
    it.b = lo;
    it.L = lens[lo];
    it.ns = (it.L + chunk - 1) / chunk;
    const int per = it.ns > 0 ? it.ns : 1;
    const int r = static_cast<int>(i - cum[lo]);
    it.hk = r / per;
    it.j = r - it.hk * per;
    it.t0 = it.j * chunk;
    it.t1 = it.ns > 0 ? min(it.t0 + chunk, it.L) : 0;
    return it;
}

template <int D, bool G32, bool PAGED, bool G16>
__global__ void __launch_bounds__(NTHREADS, 1)
decode_split_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                DecodeParams p) {
    using Lay = Layout<D, G32, G16>;
    constexpr int NG = Lay::NG;
    constexpr int NST = Lay::NST;
    constexpr int NV = Lay::NV;
    constexpr int KS = D / 16;          // MMA k-steps over head_dim (QK)
    constexpr int NGRP = D / 32;        // 32-value groups over head_dim
    constexpr int MT = D / 16;          // m-tiles of O^T over head_dim (PV)
    constexpr int NT = G16 ? 2 : 1;     // n-tiles of 8 query heads
    constexpr int NACC = G32 ? NG : 2;  // score accumulators per n-tile (two chains per token)
    constexpr int NGV = G32 ? NG : 1;   // V scales per token

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tid = threadIdx.x;
    const int g = lane >> 2, t = lane & 3;
    const int G = p.G;

    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar_full = sbase + Lay::MISC_OFF;
    const uint32_t bar_empty = bar_full + NST * 8;
    // per-warp head maxima and sums of a segment (read only between the two
    // merge barriers, so the next segment's writes cannot overtake a reader)
    float* mrg_m = reinterpret_cast<float*>(smem + Lay::MISC_OFF + 2 * NST * 8);  // [NW][16]
    float* mrg_l = mrg_m + NW * 16;                                               // [NW][16]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(mrg_l + NW * 16);
    float* mslot = reinterpret_cast<float*>(smem + Lay::MERGE_OFF);               // [NW][NV][32]
    int* lens = reinterpret_cast<int*>(smem + Lay::LENS_OFF);                     // [B]
    int* cum = lens + (kMaxB + 1);                                               // [B + 1]

    if (tid == 0) {
        ptx::prefetch_tensormap(&tm_k);     // kernel parameters: safe before the dependency wait
        ptx::prefetch_tensormap(&tm_v);
        for (int s = 0; s < NST; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 1 + 32);   // expect_tx arrive + 32 cp.async arrivals
            ptx::mbar_init(bar_empty + 8 * s, NW);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    grid_dep_wait();                    // the predecessor's writes (q, cache, lengths) are visible
    grid_dep_launch();                  // the combine kernel may be scheduled now

    // ---- lengths and chunk prefix sums (items per sequence: Hk * max(1, chunks))
    const int64_t cap = PAGED ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t lim = min(cap, static_cast<int64_t>(p.splits) * p.chunk);
    const int B = p.B;
    for (int b = tid; b < B; b += NTHREADS) {
        int L = p.seq_lens[b];
        if (L < 0 || L > lim) {
            if (blockIdx.x == 0) raise_flag(p.d_err, KVQ_DEVERR_LEN);
            L = 0;
        }
        lens[b] = L;
        const int ns = (L + p.chunk - 1) / p.chunk;
        cum[b + 1] = p.Hk * (ns > 0 ? ns : 1);
    }
    __syncthreads();
    if (warp == 0) {                    // inclusive scan of cum[1..B] by one warp
        int carry = 0;
        for (int base = 0; base < B; base += 32) {
            int v = base + lane < B ? cum[base + lane + 1] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, off);
                if (lane >= off) v += u;
            }
            if (base + lane < B) cum[base + lane + 1] = v + carry;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) cum[0] = 0;
    }
    __syncthreads();
    const int64_t T = cum[B];
    const int64_t ibeg = T * blockIdx.x / gridDim.x;
    const int64_t iend = T * (blockIdx.x + 1) / gridDim.x;

    // bounded wait that gives up at once after any earlier timeout of this CTA
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (*abort_flag) return;
        if (!ptx::mbar_wait(bar, parity)) {
            *abort_flag = 1;
            if (lane == 0) raise_flag(p.d_err, KVQ_DEVERR_TIMEOUT);
        }
    };

    // ------------------------------------------------------------ producer
    if (warp == NW) {
        const uint64_t pol = ptx::policy_evict_first();
        int count = 0;                  // tiles issued (ring position)
        int pb = -1, phk = -1;
        for (int64_t i = ibeg; i < iend; ++i) {
            const Item itm = item_at(i, lens, cum, B, p.Hk, p.chunk);
            if (itm.ns == 0) continue;
            const bool seg_first = itm.b != pb || itm.hk != phk;
            pb = itm.b;
            phk = itm.hk;
            const int b = itm.b, hk = itm.hk;
            for (int tt0 = itm.t0; tt0 < itm.t1; tt0 += TT, ++count) {
                const int s = count % NST;
                const uint32_t full = bar_full + 8 * s;
                if (count >= NST) wait(bar_empty + 8 * s, ((count / NST) - 1) & 1);
                const int ntok = min(TT, itm.t1 - tt0);
                const uint32_t sk = sbase + s * Lay::STAGE;
                const uint32_t sv = sk + Lay::KV_BYTES;
                const uint32_t sks = sv + Lay::KV_BYTES;
                const uint32_t svs = sks + Lay::SC_FLOATS * 4;
                if (!PAGED) {
                    const int64_t row0 = (static_cast<int64_t>(b) * p.Hk + hk) * p.max_seq + tt0;
                    if (lane == 0) {
                        ptx::mbar_arrive_expect_tx(full, 2 * Lay::KV_BYTES);
                        ptx::tma_load_2d(sk, &tm_k, 0, static_cast<int>(row0), full, pol);
                        ptx::tma_load_2d(sv, &tm_v, 0, static_cast<int>(row0), full, pol);
                    }
                    for (int k = lane; k < ntok; k += 32) {
                        const int64_t r = row0 + k;
                        copy_scales<NG>(sks + k * NG * 4, p.k_scale + r * NG);
                        copy_scales<NG>(svs + k * NG * 4, p.v_scale + r * NG);
                    }
                } else {
                    constexpr int PPS = TT / 16;                // pages per stage
                    const int np = (ntok + 15) >> 4;
                    int32_t pg = -1;
                    if (lane < np) {
                        // a bad entry is skipped here and reported by the consumers
                        pg = p.table[static_cast<int64_t>(b) * p.max_pages + (tt0 >> 4) + lane];
                        if (pg < 0 || pg >= p.num_pages) pg = -1;
                    }
                    const uint32_t valid = __ballot_sync(0xffffffffu, pg >= 0);
                    if (lane == 0) ptx::mbar_arrive_expect_tx(full, __popc(valid) * 2 * 16 * D);
#pragma unroll
                    for (int q = 0; q < PPS; ++q) {
                        const int pq = __shfl_sync(0xffffffffu, pg, q);
                        if (lane == 0 && pq >= 0) {
                            const int y = (pq * p.Hk + hk) * 16;
                            ptx::tma_load_2d(sk + q * 16 * D, &tm_k, 0, y, full, pol);
                            ptx::tma_load_2d(sv + q * 16 * D, &tm_v, 0, y, full, pol);
                        }
                    }
                    for (int k = lane; k < TT; k += 32) {
                        const int pk = __shfl_sync(0xffffffffu, pg, k >> 4);
                        if (k < ntok && pk >= 0) {
                            const int64_t r = (static_cast<int64_t>(pk) * p.Hk + hk) * 16 + (k & 15);
                            copy_scales<NG>(sks + k * NG * 4, p.k_scale + r * NG);
                            copy_scales<NG>(svs + k * NG * 4, p.v_scale + r * NG);
                        }
                    }
                }
                if (seg_first && tt0 == itm.t0) {
                    // the segment's G query rows (contiguous bf16) ride with its first stage
                    const uint16_t* qsrc = p.q + (static_cast<int64_t>(b) * p.Hq + hk * G) * D;
                    const uint32_t sq = sk + Lay::Q_OFF;
                    for (int c = lane; c < G * D / 8; c += 32)
                        ptx::cp_async_16(sq + c * 16, qsrc + c * 8);
                }
                ptx::cp_async_arrive_noinc(full);
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        // the last tile of every slot has landed (normally long consumed; after a
        // timeout this keeps the CTA alive until its bulk copies are done)
        if (lane == 0)
            for (int c = count - 1; c >= 0 && c >= count - NST; --c)
                ptx::mbar_wait(bar_full + 8 * (c % NST), (c / NST) & 1);
        return;                         // consumers synchronise among themselves (barrier 1)
    }

    // ------------------------------------------------------------ consumers
    const int sig_g = sigma(g);
    const int sig_a = sigma(2 * t), sig_b = sigma(2 * t + 1);
    const int rowA = 16 * warp + sig_g;           // MMA row g     of this warp's slice
    const int rowB = rowA + 8;                    // MMA row g + 8
    const int R0 = 16 * warp + sig_a, R1 = 16 * warp + sig_b;   // V rows of k 2t, 2t+1
    const int R2 = R0 + 8, R3 = R1 + 8;                         // V rows of k 2t+8, 2t+9

    uint32_t qb0[NT][KS], qb1[NT][KS];
    float zs[NT][2];
    float m[NT][2], l[NT][2];
    float o[MT][NT][4];                 // O^T C fragments: rows = head_dim, columns = heads
    int kv = 64;                        // running P'' prescale exponent (per warp)
    int c_count = 0;                    // tiles consumed (ring position)
    bool open = false;                  // a segment's state is live
    int seg_j0 = 0;                     // first chunk of the open segment

    for (int64_t i = ibeg; i < iend; ++i) {
        const Item itm = item_at(i, lens, cum, B, p.Hk, p.chunk);
        const int b = itm.b, hk = itm.hk;
        const int64_t bh0 = static_cast<int64_t>(b) * p.Hq + hk * G;   // first q head of the group
        if (itm.ns == 0) {
            // empty (or rejected) sequence: zero rows
            for (int idx = tid; idx < G * D; idx += NCONS) p.out[bh0 * D + idx] = 0.f;
            continue;
        }
        if (!open) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                m[nt][0] = m[nt][1] = -INFINITY;
                l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
                    o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
            }
            kv = 64;
            seg_j0 = itm.j;
        }
        const int t0 = itm.t0, t1 = itm.t1;
        const int ntiles = (t1 - t0 + TT - 1) / TT;
        for (int it = 0; it < ntiles; ++it, ++c_count) {
            const int s = c_count % NST;
            wait(bar_full + 8 * s, (c_count / NST) & 1);
            const int tt0 = t0 + it * TT;
            const uint32_t sk = sbase + s * Lay::STAGE;
            const uint32_t sv = sk + Lay::KV_BYTES;
            const uint32_t sks = sv + Lay::KV_BYTES;
            const uint32_t svs = sks + Lay::SC_FLOATS * 4;
            if (!open && it == 0) {
                // ---- Q^T operand from the stage: column n = g of n-tile nt is query
                // head 8*nt + g, pre-scaled by 2^sh so max |q| * 2^sh is in [2^14, 2^15).
                // B fragment rows 2t, 2t+1 (qb0) and 2t+8, 2t+9 (qb1) of k-step
                // 2*gi + h2 hold head_dim 32*gi + 8*t + 4*h2 + {0, 1} and {2, 3}.
                const uint32_t sq = sk + Lay::Q_OFF;
                float zsq[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int h = 8 * nt + g;
                    float qf[NGRP][8];
                    float amax = 0.f;
#pragma unroll
                    for (int gi = 0; gi < NGRP; ++gi) {
                        uint4 raw = make_uint4(0u, 0u, 0u, 0u);
                        if (h < G) raw = lds128(sq + (h * D + 32 * gi + 8 * t) * 2);
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            qf[gi][2 * e] = bf16_bits_to_f32(w[e] & 0xffffu);
                            qf[gi][2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(qf[gi][e]));
                    }
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                    int sh = 0;
                    if (amax > 0.f) {
                        const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
                        sh = min(max(14 - e, -100), 100);
                    }
                    const float up = ldexpf(1.f, sh);
                    zsq[nt] = ldexpf(1.f, -sh) * p.scale_log2;
#pragma unroll
                    for (int gi = 0; gi < NGRP; ++gi)
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            qb0[nt][2 * gi + h2] =
                                ptx::pack_f16x2(qf[gi][4 * h2] * up, qf[gi][4 * h2 + 1] * up);
                            qb1[nt][2 * gi + h2] =
                                ptx::pack_f16x2(qf[gi][4 * h2 + 2] * up, qf[gi][4 * h2 + 3] * up);
                        }
                }
                // score factor of the two heads (columns 2t, 2t+1) this thread accumulates
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    zs[nt][0] = __shfl_sync(0xffffffffu, zsq[nt], 4 * (2 * t));
                    zs[nt][1] = __shfl_sync(0xffffffffu, zsq[nt], 4 * (2 * t + 1));
                }
            }
            const int tok0 = tt0 + 16 * warp;             // first token of this warp's slice
            if (tok0 < t1) {
            bool page_ok = true;
            if (PAGED) {
                const int32_t pg = p.table[static_cast<int64_t>(b) * p.max_pages + (tok0 >> 4)];
                page_ok = pg >= 0 && pg < p.num_pages;
                if (!page_ok && lane == 0) raise_flag(p.d_err, KVQ_DEVERR_PAGE);
            }
            const bool okA = page_ok && (tok0 + sig_g < t1);
            const bool okB = page_ok && (tok0 + 8 + sig_g < t1);

            // ---- S^T = K . Q^T: rows tokens (rowA, rowB), columns heads
            float sacc[NT][NACC][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int a = 0; a < NACC; ++a)
                    sacc[nt][a][0] = sacc[nt][a][1] = sacc[nt][a][2] = sacc[nt][a][3] = 0.f;
#pragma unroll
            for (int gi = 0; gi < NGRP; ++gi) {
                const uint2 wa = lds64(sk + swz<D>(rowA, 32 * gi + 8 * t));
                const uint2 wb = lds64(sk + swz<D>(rowB, 32 * gi + 8 * t));
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const uint32_t xa = h2 ? wa.y : wa.x;
                    const uint32_t xb = h2 ? wb.y : wb.x;
                    const uint32_t a0 = ptx::bytes_to_f16x2(xa, 0x4140u);
                    const uint32_t a2 = ptx::bytes_to_f16x2(xa, 0x4342u);
                    const uint32_t a1 = ptx::bytes_to_f16x2(xb, 0x4140u);
                    const uint32_t a3 = ptx::bytes_to_f16x2(xb, 0x4342u);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        ptx::mma_f16(sacc[nt][G32 ? gi : (gi & 1)], a0, a1, a2, a3,
                                     qb0[nt][2 * gi + h2], qb1[nt][2 * gi + h2]);
                }
            }
            // ---- scores z (log2 domain): [nt][0..1] token rowA, [nt][2..3] token rowB
            float z[NT][4];
            if (G32) {
                float ksa[NG], ksb[NG];
#pragma unroll
                for (int a = 0; a < NG; ++a) {
                    ksa[a] = ldsf(sks + (rowA * NG + a) * 4);
                    ksb[a] = ldsf(sks + (rowB * NG + a) * 4);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float za0 = 0.f, za1 = 0.f, zb0 = 0.f, zb1 = 0.f;
#pragma unroll
                    for (int a = 0; a < NACC; ++a) {
                        za0 = fmaf(sacc[nt][a][0], ksa[a], za0);
                        za1 = fmaf(sacc[nt][a][1], ksa[a], za1);
                        zb0 = fmaf(sacc[nt][a][2], ksb[a], zb0);
                        zb1 = fmaf(sacc[nt][a][3], ksb[a], zb1);
                    }
                    z[nt][0] = okA ? za0 * zs[nt][0] : -INFINITY;
                    z[nt][1] = okA ? za1 * zs[nt][1] : -INFINITY;
                    z[nt][2] = okB ? zb0 * zs[nt][0] : -INFINITY;
                    z[nt][3] = okB ? zb1 * zs[nt][1] : -INFINITY;
                }
            } else {
                const float ksa = ldsf(sks + rowA * 4), ksb = ldsf(sks + rowB * 4);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float s0 = sacc[nt][0][0] + sacc[nt][1][0];
                    const float s1 = sacc[nt][0][1] + sacc[nt][1][1];
                    const float s2 = sacc[nt][0][2] + sacc[nt][1][2];
                    const float s3 = sacc[nt][0][3] + sacc[nt][1][3];
                    z[nt][0] = okA ? s0 * ksa * zs[nt][0] : -INFINITY;
                    z[nt][1] = okA ? s1 * ksa * zs[nt][1] : -INFINITY;
                    z[nt][2] = okB ? s2 * ksb * zs[nt][0] : -INFINITY;
                    z[nt][3] = okB ? s3 * ksb * zs[nt][1] : -INFINITY;
                }
            }
            // ---- online softmax per head: max over the slice's 16 tokens
            float pr[NT][4];
            float f[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    float mx = fmaxf(z[nt][c], z[nt][2 + c]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float mn = fmaxf(m[nt][c], mx);
                    const float al = (mn == -INFINITY) ? 1.f : ptx::ex2(m[nt][c] - mn);
                    pr[nt][c] = okA ? ptx::ex2(z[nt][c] - mn) : 0.f;
                    pr[nt][2 + c] = okB ? ptx::ex2(z[nt][2 + c] - mn) : 0.f;
                    l[nt][c] = l[nt][c] * al + pr[nt][c] + pr[nt][2 + c];
                    m[nt][c] = mn;
                    f[nt][c] = al;
                }
            // ---- V scales of the thread's two tokens and the running prescale 2^kv
            float vsa[NGV], vsb[NGV];
            float vmax = 0.f;
#pragma unroll
            for (int gv = 0; gv < NGV; ++gv) {
                vsa[gv] = okA ? ldsf(svs + (rowA * NG + gv) * 4) : 0.f;
                vsb[gv] = okB ? ldsf(svs + (rowB * NG + gv) * 4) : 0.f;
                vmax = fmaxf(vmax, fmaxf(vsa[gv], vsb[gv]));
            }
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 4));
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 8));
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 16));
            if (vmax > 0.f) {
                const int ev = static_cast<int>((__float_as_uint(vmax) >> 23) & 0xffu) - 127;
                const int kn = min(kv, 14 - ev);
                if (kn < kv) {
                    const float drop = ldexpf(1.f, kn - kv);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        f[nt][0] *= drop;
                        f[nt][1] *= drop;
                    }
                    kv = kn;
                }
            }
            const float up = ldexpf(1.f, kv);
            bool unit = true;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) unit = unit && f[nt][0] == 1.f && f[nt][1] == 1.f;
            if (!__all_sync(0xffffffffu, unit)) {       // the running max moved: rescale O
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        o[mt][nt][0] *= f[nt][0];
                        o[mt][nt][1] *= f[nt][1];
                        o[mt][nt][2] *= f[nt][0];
                        o[mt][nt][3] *= f[nt][1];
                    }
            }
            // ---- P^T operand: P'' hi / lo, transposed from the score layout
            // (row = token, column = head) into B fragments (k = token, n = head)
            uint32_t pbh[NGV][NT][2], pbl[NGV][NT][2];
#pragma unroll
            for (int gv = 0; gv < NGV; ++gv)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    uint32_t ha, la, hb, lb;
                    split_f16x2(pr[nt][0] * vsa[gv] * up, pr[nt][1] * vsa[gv] * up, ha, la);
                    split_f16x2(pr[nt][2] * vsb[gv] * up, pr[nt][3] * vsb[gv] * up, hb, lb);
                    pbh[gv][nt][0] = transpose8x8(ha);
                    pbl[gv][nt][0] = transpose8x8(la);
                    pbh[gv][nt][1] = transpose8x8(hb);
                    pbl[gv][nt][1] = transpose8x8(lb);
                }
            // ---- O^T += V^T . P^T.  V^T A fragment of m-tile mt: rows g, g+8 are
            // head_dim d(mt, g), d(mt, g) + 1; columns 2t, 2t+1 / 2t+8, 2t+9 are the
            // V rows R0, R1 / R2, R3.  Byte pairs of two rows are interleaved with
            // prmt and turned into exact (v - 128) f16 pairs.
            auto pv_words = [&](int mt0, int gv, uint32_t w0, uint32_t w1, uint32_t w2,
                                uint32_t w3) {
                const uint32_t xl01 = ptx::prmt(w0, w1, 0x5140u);
                const uint32_t xh01 = ptx::prmt(w0, w1, 0x7362u);
                const uint32_t xl23 = ptx::prmt(w2, w3, 0x5140u);
                const uint32_t xh23 = ptx::prmt(w2, w3, 0x7362u);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t x01 = hh ? xh01 : xl01;
                    const uint32_t x23 = hh ? xh23 : xl23;
                    const uint32_t a0 = ptx::bytes_to_f16x2(x01, 0x4140u);
                    const uint32_t a1 = ptx::bytes_to_f16x2(x01, 0x4342u);
                    const uint32_t a2 = ptx::bytes_to_f16x2(x23, 0x4140u);
                    const uint32_t a3 = ptx::bytes_to_f16x2(x23, 0x4342u);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        ptx::mma_f16(o[mt0 + hh][nt], a0, a1, a2, a3, pbh[gv][nt][0],
                                     pbh[gv][nt][1]);
                        ptx::mma_f16(o[mt0 + hh][nt], a0, a1, a2, a3, pbl[gv][nt][0],
                                     pbl[gv][nt][1]);
                    }
                }
            };
            if (!G32) {
                if constexpr (D == 128) {
                    // thread g owns head_dim [16g, 16g + 16): d(mt, g) = 16g + 2mt
                    const uint4 v0 = lds128(sv + swz<D>(R0, 16 * g));
                    const uint4 v1 = lds128(sv + swz<D>(R1, 16 * g));
                    const uint4 v2 = lds128(sv + swz<D>(R2, 16 * g));
                    const uint4 v3 = lds128(sv + swz<D>(R3, 16 * g));
                    pv_words(0, 0, v0.x, v1.x, v2.x, v3.x);
                    pv_words(2, 0, v0.y, v1.y, v2.y, v3.y);
                    pv_words(4, 0, v0.z, v1.z, v2.z, v3.z);
                    pv_words(6, 0, v0.w, v1.w, v2.w, v3.w);
                } else {
                    // D == 64: thread g owns head_dim [8g, 8g + 8): d(mt, g) = 8g + 2mt
                    const uint2 v0 = lds64(sv + swz<D>(R0, 8 * g));
                    const uint2 v1 = lds64(sv + swz<D>(R1, 8 * g));
                    const uint2 v2 = lds64(sv + swz<D>(R2, 8 * g));
                    const uint2 v3 = lds64(sv + swz<D>(R3, 8 * g));
                    pv_words(0, 0, v0.x, v1.x, v2.x, v3.x);
                    pv_words(2, 0, v0.y, v1.y, v2.y, v3.y);
                }
            } else {
                // group-32: m-tiles 2*gv, 2*gv + 1 stay inside group gv:
                // d(2gv + hh, g) = 32*gv + 4*g + 2*hh
#pragma unroll
                for (int gv = 0; gv < NGRP; ++gv) {
                    const uint32_t cb = 32 * gv + 4 * g;
                    pv_words(2 * gv, gv, lds32(sv + swz<D>(R0, cb)), lds32(sv + swz<D>(R1, cb)),
                             lds32(sv + swz<D>(R2, cb)), lds32(sv + swz<D>(R3, cb)));
                }
            }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_empty + 8 * s);
        }
        open = true;
        // the segment continues if the next item is the next chunk of this (b, kv head)
        if (i + 1 < iend) {
            const Item nx = item_at(i + 1, lens, cum, B, p.Hk, p.chunk);
            if (nx.b == b && nx.hk == hk) continue;
        }
        open = false;

        // ---- merge the eight warps' states of the segment (one round)
        // a segment that is the whole sequence writes the final rows (and,
        // when the sequence has several chunks, a marker l = -1 in slot 0 that
        // tells the combine kernel to leave them alone)
        const bool final_rows = itm.ns == 1 || (seg_j0 == 0 && itm.j == itm.ns - 1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 4);
                l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 8);
                l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 16);
                if (g == 0) {
                    mrg_m[warp * 16 + 8 * nt + 2 * t + c] = m[nt][c];
                    mrg_l[warp * 16 + 8 * nt + 2 * t + c] = l[nt][c];
                }
            }
        ptx::named_bar_sync(1, NCONS);
        // per head of this thread: segment max M, segment sum Ls, and the factor
        // for this warp's o (2^(m - M) undoing the P'' prescale, divided by Ls
        // when the rows are final)
        float fo[NT][2];
        {
            const float down = ldexpf(1.f, -kv);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int h = 8 * nt + 2 * t + c;
                    float mw[NW];
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < NW; ++w) {
                        mw[w] = mrg_m[w * 16 + h];
                        M = fmaxf(M, mw[w]);
                    }
                    float Ls = 0.f;
#pragma unroll
                    for (int w = 0; w < NW; ++w)
                        if (mw[w] != -INFINITY) Ls = fmaf(mrg_l[w * 16 + h], ptx::ex2(mw[w] - M), Ls);
                    const float f = (m[nt][c] == -INFINITY) ? 0.f : ptx::ex2(m[nt][c] - M) * down;
                    fo[nt][c] = final_rows ? (Ls > 0.f ? f / Ls : 0.f) : f;
                    if (warp == 0 && g == 0 && itm.ns > 1 && h < G) {
                        const int64_t row = bh0 + h;
                        if (final_rows) {
                            p.ws_l[row * p.splits] = -1.f;
                        } else {
                            p.ws_m[row * p.splits + seg_j0] = M;
                            p.ws_l[row * p.splits + seg_j0] = Ls;
                            for (int jj = seg_j0 + 1; jj <= itm.j; ++jj) {   // merged into seg_j0
                                p.ws_m[row * p.splits + jj] = -INFINITY;
                                p.ws_l[row * p.splits + jj] = 0.f;
                            }
                        }
                    }
                }
        }
        {
            float* slot = mslot + warp * NV * 32 + lane;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        slot[((mt * NT + nt) * 4 + e) * 32] = o[mt][nt][e] * fo[nt][e & 1];
        }
        ptx::named_bar_sync(1, NCONS);
        // sum the eight slots position by position and write the rows
        for (int pos = tid; pos < NV * 32; pos += NCONS) {
            const int v = pos >> 5, ln = pos & 31;
            const int pg_ = ln >> 2, pt = ln & 3;
            const int mt = v / (NT * 4), nt = (v / 4) % NT, e = v & 3;
            const int h = 8 * nt + 2 * pt + (e & 1);
            if (h >= G) continue;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) sum += mslot[(w * NV + v) * 32 + ln];
            const int d = G32 ? 32 * (mt >> 1) + 4 * pg_ + 2 * (mt & 1) + (e >> 1)
                              : (D == 128 ? 16 : 8) * pg_ + 2 * mt + (e >> 1);
            const int64_t row = bh0 + h;
            if (final_rows) p.out[row * D + d] = sum;
            else p.ws_o[(row * p.splits + seg_j0) * D + d] = sum;
        }
    }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(ptr);
    }
    return fn;
}

// 2-D u8 tensor map over `rows` rows of D bytes, box of box_rows rows.
cudaError_t make_map(CUtensorMap* map, const void* base, int D, int64_t rows, int box_rows) {
    EncodeFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw =
        D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, bool G32, bool PAGED, bool G16>
cudaError_t set_attrs() {
    using Lay = Layout<D, G32, G16>;
    static bool done = false;
    if (done) return cudaSuccess;
    auto kern = decode_split_tc<D, G32, PAGED, G16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) done = true;
    return e;
}

template <int D, bool G32, bool PAGED, bool G16>
cudaError_t launch_tc(const DecodeParams& p, cudaStream_t s) {
    using Lay = Layout<D, G32, G16>;
    cudaError_t e = set_attrs<D, G32, PAGED, G16>();
    if (e != cudaSuccess) return e;
    CUtensorMap mk, mv;
    const int64_t rows = PAGED ? static_cast<int64_t>(p.num_pages) * p.Hk * 16
                               : static_cast<int64_t>(p.B) * p.Hk * p.max_seq;
    const int box = PAGED ? 16 : TT;
    e = make_map(&mk, p.k, D, rows, box);
    if (e == cudaSuccess) e = make_map(&mv, p.v, D, rows, box);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid, 1, 1);
    cfg.blockDim = dim3(NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = Lay::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_split_tc<D, G32, PAGED, G16>, mk, mv, p);
}

template <int D, bool G32, bool PAGED>
cudaError_t pick_g(const DecodeParams& p, cudaStream_t s) {
    return p.G > 8 ? launch_tc<D, G32, PAGED, true>(p, s) : launch_tc<D, G32, PAGED, false>(p, s);
}

template <int D>
cudaError_t pick_layout(const DecodeParams& p, cudaStream_t s) {
    if (p.page_size)
        return p.group32 ? pick_g<D, true, true>(p, s) : pick_g<D, false, true>(p, s);
    return p.group32 ? pick_g<D, true, false>(p, s) : pick_g<D, false, false>(p, s);
}

}  // namespace

cudaError_t launch_decode_split_tc(const DecodeParams& p, cudaStream_t s) {
    if (p.grid < 1) return cudaErrorInvalidValue;
    if (p.D == 128) return pick_layout<128>(p, s);
    if (p.D == 64) return pick_layout<64>(p, s);
    return cudaErrorInvalidValue;
}

}  // namespace kvq

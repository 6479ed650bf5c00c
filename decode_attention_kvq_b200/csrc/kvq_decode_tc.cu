// kvq_decode_tc.cu -- decode attention on the INT8 cache for sm_100a:
// TMA-staged K/V tiles, tensor-core Q.K^T and P.V on exact integer operands
// with the dequantisation scales applied outside the MMA, split-K across the
// CTAs of a thread-block cluster combined through distributed shared memory.
//
// Method (what is computed): abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
// module doc "Fused approach" -- Q.K^T with K dequantised on the fly,
// softmax, P.V with V dequantised on the fly; combs-models 0.2.2, src/kv.rs,
// attend / repeat_kv -- scale after the dot product, query head h reads kv
// head h / G, a decode query attends to the whole cache.  Split-K with an
// online softmax and the combine are this library's own (flash-decoding).
//
// How (sm_100a):
//  * Grid (S, Hk, B): S splits of the KV range per (sequence, kv head).  With
//    2 <= S <= 16 the S CTAs form one thread-block cluster and merge their
//    partial softmax states through distributed shared memory (no global
//    workspace, no second kernel).  Larger S (only on request) writes the
//    partials to a workspace for the combine kernel in kvq_decode.cu.
//  * CTA = 4 warps.  Warp 0 streams 64-token stages of K and V bytes into
//    shared memory with TMA tile loads (2-D tensor maps over the cache rows,
//    128-byte swizzle for D=128, 64-byte for D=64) and the fp32 scales with
//    cp.async; both complete on the stage's mbarrier; 4 stages in flight.
//    Every warp takes one 16-token slice of each stage.
//  * Per slice: S = Q.K^T with mma.sync m16n8k16 (f16 in, f32 accumulate),
//    rows = query heads of the GQA group (padded to 16), columns = tokens.
//    The operands are exact: K enters as the integers (byte - 128) built in
//    registers (1024 + byte spliced into an f16 mantissa, minus 1152), and Q
//    enters as f16 after a per-head power-of-two prescale (bf16 has 8
//    significant bits, f16 has 11, so q * 2^s is exact), so the f32
//    accumulators hold sum_d q_d (k_d - 128) up to accumulation rounding.
//    The K scale (per token, or per 32-value group with one accumulator per
//    group), 2^-s, attn_scale and log2(e) are applied to the accumulator.
//  * Online softmax in base 2 per head row.  The V scale is folded into P:
//    P'' = 2^(z-m) * v_scale(token) * 2^kv (per 32-value group in group-32
//    mode), with a running per-warp power of two 2^kv that keeps P'' inside
//    the f16 normal range.  P'' is split into f16 hi + lo parts (about 22
//    significant bits together) and both are multiplied with the exact
//    integers (v - 128), so P.V carries no f16 rounding of P beyond ~2^-22.
//  * Token order inside each 16-token slice and the d order of the MMA
//    k-dimension are permuted so that every shared-memory load of the
//    swizzled tiles is free of bank conflicts (sigma below).
//  * Every wait on an mbarrier is bounded; a wait that gives up sets
//    KVQ_DEVERR_TIMEOUT and the kernel finishes without hanging.
#include <cuda.h>
#include <math.h>

#include "kvq_internal.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

constexpr int TT = 64;                 // tokens per stage: one 16-token slice per warp
constexpr int NW = 4;                  // warps per CTA
constexpr int NTHREADS = NW * 32;
constexpr int NST = 4;                 // stages in flight
constexpr int kMaxCluster = 16;        // largest cluster the combine supports

// Row (inside an 8-token group) that holds MMA column n of the K operand and
// MMA k-index n of the V operand: sigma = {0, 2, 4, 6, 3, 1, 7, 5}.  Under the
// 128-byte swizzle (16-byte chunk index XOR row % 8) this makes the K loads
// (rows sigma(g), 8 bytes at 32*G + 8*t) and the V loads (rows sigma(2t),
// sigma(2t+1), 16 bytes at 16*g) of a warp hit distinct banks: the rows a
// load instruction touches differ in bits 1..2.
__device__ __forceinline__ int sigma(int x) { return x < 4 ? 2 * x : ((2 * x - 7) ^ 2); }


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

// (a, b) -> f16x2 hi = rn(a, b) and lo = rn(a - hi, b - hi): hi + lo carries
// about 22 significant bits of each value.
__device__ __forceinline__ void split_f16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 f = __half22float2(h);
    const __half2 l = __floats2half2_rn(a - f.x, b - f.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
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

template <int D, bool G32>
struct Layout {
    static constexpr int NG = G32 ? D / 32 : 1;
    static constexpr int KV_BYTES = TT * D;
    static constexpr int SC_FLOATS = TT * NG;
    static constexpr int STAGE = ((2 * KV_BYTES + 2 * SC_FLOATS * 4) + 1023) / 1024 * 1024;
    static constexpr int BAR_OFF = NST * STAGE;
    static constexpr int NBAR = 2 * NST + 2;               // full[], empty[], done, read
    static constexpr int SMEM = BAR_OFF + NBAR * 8 + 1024;  // + base alignment slack
    // epilogue buffers, in floats, reusing the stage area once every stage is consumed
    static constexpr int RS = D + 4;                       // warp-merge row stride
    static constexpr int RED_M = NW * 16 * RS;             // [NW][16] running max
    static constexpr int RED_L = RED_M + NW * 16;          // [NW][16] running sum
    static constexpr int CPS = D + 2;                      // CTA partial row: o[D], m, l
    static constexpr int CP = RED_L + NW * 16;             // [16][CPS]
    static constexpr int CW = CP + 16 * CPS;               // [kMaxCluster][16] peer max / weights
    static constexpr int CL = CW + kMaxCluster * 16;       // [kMaxCluster][16] peer sums
    static constexpr int CSUM = CL + kMaxCluster * 16;     // [16] combined sums
    static constexpr int EPI_FLOATS = CSUM + 16;
    static_assert(EPI_FLOATS * 4 <= BAR_OFF, "epilogue buffers fit in the stage area");
};

__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// Bounded wait with cluster-scope acquire (sees stores released by peers).
__device__ __forceinline__ bool wait_cluster(uint32_t bar, uint32_t parity) {
    for (uint32_t i = 0; i < ptx::kSpinLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}

template <int D, bool G32, bool PAGED, bool G16>
__global__ void __launch_bounds__(NTHREADS, G16 ? 2 : 3)
decode_split_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                DecodeParams p) {
    using Lay = Layout<D, G32>;
    constexpr int NG = Lay::NG;
    constexpr int KS = D / 16;          // MMA k-steps over head_dim
    constexpr int NGRP = D / 32;        // 32-value groups over head_dim
    constexpr int NTD = D / 8;          // output n-tiles over head_dim
    constexpr int NACC = G32 ? NG : 1;  // score accumulators per n-tile
    constexpr int NGV = G32 ? NG : 1;   // V scales per token

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int j = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tid = threadIdx.x;
    const int G = p.G;
    const int S = p.cluster;            // CTAs in this kernel's cluster (1: none)

    const int64_t cap = PAGED ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int64_t lim = min(cap, static_cast<int64_t>(p.splits) * p.chunk);
    int L = p.seq_lens[b];
    if (L < 0 || L > lim) {
        if (j == 0 && hk == 0 && tid == 0) raise_flag(p.d_err, KVQ_DEVERR_LEN);
        L = 0;
    }
    // No CTA leaves early: in a cluster every CTA takes part in the combine.
    const int t0 = j * p.chunk;
    const bool active = t0 < L;
    const int t1 = active ? min(t0 + p.chunk, L) : t0;
    const int nsplit = (L + p.chunk - 1) / p.chunk;
    const int ntiles = active ? (t1 - t0 + TT - 1) / TT : 0;

    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar_full = sbase + Lay::BAR_OFF;
    const uint32_t bar_empty = bar_full + NST * 8;
    const uint32_t bar_done = bar_empty + NST * 8;     // all peers' partials are ready
    const uint32_t bar_read = bar_done + 8;             // all peers finished reading ours
    if (tid == 0) {
        for (int s = 0; s < NST; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 1 + 32);   // expect_tx arrive + 32 cp.async arrivals
            ptx::mbar_init(bar_empty + 8 * s, NW);
        }
        ptx::mbar_init(bar_done, S);
        ptx::mbar_init(bar_read, S);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    // peers arrive on our barriers only after every CTA has initialised them
    if (S > 1) cluster_sync_all();

    // ---- warp 0 issues stage i: TMA for K/V bytes, cp.async for the scales
    const uint64_t pol = ptx::policy_evict_first();
    auto issue = [&](int i) {
        const int s = i % NST;
        const uint32_t full = bar_full + 8 * s;
        const int tt0 = t0 + i * TT;
        const int ntok = min(TT, t1 - tt0);
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
            const int np = (ntok + 15) >> 4;
            int32_t pg = -1;
            if (lane < np) {
                pg = p.table[static_cast<int64_t>(b) * p.max_pages + (tt0 >> 4) + lane];
                if (pg < 0 || pg >= p.num_pages) {
                    raise_flag(p.d_err, KVQ_DEVERR_PAGE);
                    pg = -1;
                }
            }
            const uint32_t valid = __ballot_sync(0xffffffffu, pg >= 0);
            int pgs[TT / 16];
#pragma unroll
            for (int q = 0; q < TT / 16; ++q) pgs[q] = __shfl_sync(0xffffffffu, pg, q);
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(full, __popc(valid) * 2 * 16 * D);
                for (int q = 0; q < np; ++q) {
                    const int pq = pgs[q];
                    if (pq < 0) continue;
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
        ptx::cp_async_arrive_noinc(full);
    };
    if (warp == 0) {
        if (lane == 0 && ntiles > 0) {
            ptx::prefetch_tensormap(&tm_k);
            ptx::prefetch_tensormap(&tm_v);
        }
        for (int i = 0; i < min(NST, ntiles); ++i) issue(i);
    }

    const int g = lane >> 2, t = lane & 3;
    // Q fragments: rows = heads g (lo) and g + 8 (hi), pre-scaled by 2^s
    uint32_t qa0[KS], qa2[KS], qa1[KS], qa3[KS];
    float zs_lo = 0.f, zs_hi = 0.f;
    const float sc_log2 = p.scale_log2;
    auto load_q = [&](int h, uint32_t* f0, uint32_t* f2, float& zs) {
        float qf[NGRP][8];
        float amax = 0.f;
        if (h < G) {
            const uint16_t* qrow = p.q + (static_cast<int64_t>(b) * p.Hq + hk * G + h) * D;
#pragma unroll
            for (int gi = 0; gi < NGRP; ++gi) {
                const uint4 raw = *reinterpret_cast<const uint4*>(qrow + 32 * gi + 8 * t);
                const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    qf[gi][2 * e] = bf16_bits_to_f32(w[e] & 0xffffu);
                    qf[gi][2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(qf[gi][e]));
            }
        } else {
#pragma unroll
            for (int gi = 0; gi < NGRP; ++gi)
#pragma unroll
                for (int e = 0; e < 8; ++e) qf[gi][e] = 0.f;
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        // power-of-two prescale: max |q| * 2^s in [2^14, 2^15)
        int sh = 0;
        if (amax > 0.f) {
            const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
            sh = min(max(14 - e, -100), 100);
        }
        const float up = ldexpf(1.f, sh);
        zs = ldexpf(1.f, -sh) * sc_log2;
#pragma unroll
        for (int gi = 0; gi < NGRP; ++gi)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                f0[2 * gi + h2] = ptx::pack_f16x2(qf[gi][4 * h2] * up, qf[gi][4 * h2 + 1] * up);
                f2[2 * gi + h2] = ptx::pack_f16x2(qf[gi][4 * h2 + 2] * up, qf[gi][4 * h2 + 3] * up);
            }
    };
#pragma unroll
    for (int k = 0; k < KS; ++k) qa0[k] = qa1[k] = qa2[k] = qa3[k] = 0u;
    if (ntiles > 0) {
        load_q(g, qa0, qa2, zs_lo);
        if (G16) load_q(g + 8, qa1, qa3, zs_hi);
    }

    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    float o_lo[NTD][2], o_hi[NTD][2];
#pragma unroll
    for (int n = 0; n < NTD; ++n) o_lo[n][0] = o_lo[n][1] = o_hi[n][0] = o_hi[n][1] = 0.f;

    int kv = 64;                         // running P'' prescale exponent (per warp)
    const int sig_g = sigma(g);
    const int sig_a = sigma(2 * t), sig_b = sigma(2 * t + 1);

    for (int i = 0; i < ntiles; ++i) {
        const int s = i % NST;
        if (!ptx::mbar_wait(bar_full + 8 * s, (i / NST) & 1)) {
            if (lane == 0) raise_flag(p.d_err, KVQ_DEVERR_TIMEOUT);
            break;
        }
        const int tt0 = t0 + i * TT;
        const uint32_t sk = sbase + s * Lay::STAGE;
        const uint32_t sv = sk + Lay::KV_BYTES;
        const uint32_t sks = sv + Lay::KV_BYTES;
        const uint32_t svs = sks + Lay::SC_FLOATS * 4;
        const int tok0 = tt0 + 16 * warp;             // this warp's 16-token slice
        if (tok0 < t1) {
            bool page_ok = true;
            if (PAGED) {
                const int32_t pg = p.table[static_cast<int64_t>(b) * p.max_pages + (tok0 >> 4)];
                page_ok = pg >= 0 && pg < p.num_pages;
            }
            // ---- S = Q.K^T on 16 tokens: two n-tiles of 8
            float sacc[2][NACC][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int a = 0; a < NACC; ++a)
                    sacc[nt][a][0] = sacc[nt][a][1] = sacc[nt][a][2] = sacc[nt][a][3] = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const uint32_t row = 16 * warp + 8 * nt + sig_g;
                uint2 kw[NGRP];
#pragma unroll
                for (int gi = 0; gi < NGRP; ++gi) kw[gi] = lds64(sk + swz<D>(row, 32 * gi + 8 * t));
#pragma unroll
                for (int gi = 0; gi < NGRP; ++gi)
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const uint32_t w = h2 ? kw[gi].y : kw[gi].x;
                        const uint32_t b0 = ptx::bytes_to_f16x2(w, 0x4140u);
                        const uint32_t b1 = ptx::bytes_to_f16x2(w, 0x4342u);
                        const int ks = 2 * gi + h2;
                        ptx::mma_f16(sacc[nt][G32 ? gi : 0], qa0[ks], qa1[ks], qa2[ks], qa3[ks],
                                     b0, b1);
                    }
            }
            // ---- scores (log2 domain), masked
            float z_lo[2][2], z_hi[2][2];
            bool ok[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int r = 16 * warp + 8 * nt + (c ? sig_b : sig_a);
                    ok[nt][c] = page_ok && (tt0 + r < t1);
                    float zl, zh;
                    if (G32) {
                        zl = 0.f;
                        zh = 0.f;
#pragma unroll
                        for (int a = 0; a < NACC; ++a) {
                            const float ksc = ldsf(sks + (r * NG + a) * 4);
                            zl = fmaf(sacc[nt][a][c], ksc, zl);
                            zh = fmaf(sacc[nt][a][2 + c], ksc, zh);
                        }
                    } else {
                        const float ksc = ldsf(sks + r * 4);
                        zl = sacc[nt][0][c] * ksc;
                        zh = sacc[nt][0][2 + c] * ksc;
                    }
                    z_lo[nt][c] = ok[nt][c] ? zl * zs_lo : -INFINITY;
                    z_hi[nt][c] = ok[nt][c] ? zh * zs_hi : -INFINITY;
                }
            // ---- online softmax, rows g (lo) and g + 8 (hi)
            float mx_lo = fmaxf(fmaxf(z_lo[0][0], z_lo[0][1]), fmaxf(z_lo[1][0], z_lo[1][1]));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
            const float mn_lo = fmaxf(m_lo, mx_lo);
            const float al_lo = (mn_lo == -INFINITY) ? 1.f : ptx::ex2(m_lo - mn_lo);
            float pr_lo[2][2], pr_hi[2][2];
            float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    pr_lo[nt][c] = ok[nt][c] ? ptx::ex2(z_lo[nt][c] - mn_lo) : 0.f;
                    pr_hi[nt][c] = 0.f;
                    ps_lo += pr_lo[nt][c];
                }
            l_lo = l_lo * al_lo + ps_lo;
            m_lo = mn_lo;
            float al_hi = 1.f;
            if (G16) {
                float mx_hi = fmaxf(fmaxf(z_hi[0][0], z_hi[0][1]), fmaxf(z_hi[1][0], z_hi[1][1]));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
                const float mn_hi = fmaxf(m_hi, mx_hi);
                al_hi = (mn_hi == -INFINITY) ? 1.f : ptx::ex2(m_hi - mn_hi);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        pr_hi[nt][c] = ok[nt][c] ? ptx::ex2(z_hi[nt][c] - mn_hi) : 0.f;
                        ps_hi += pr_hi[nt][c];
                    }
                l_hi = l_hi * al_hi + ps_hi;
                m_hi = mn_hi;
            }

            // ---- V scales of this slice and the running power-of-two prescale:
            // P'' = p * v_scale * 2^kv with kv chosen so that the largest
            // v_scale * 2^kv seen by this warp lies in [2^14, 2^15); when kv
            // drops, the accumulated O is rescaled by the same power of two.
            const int R0 = 16 * warp + sig_a, R1 = 16 * warp + sig_b;
            const int R2 = R0 + 8, R3 = R1 + 8;
            const int rr[2][2] = {{R0, R1}, {R2, R3}};
            float vsc[2][2][NGV];
            float vmax = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c)
#pragma unroll
                    for (int gv = 0; gv < NGV; ++gv) {
                        vsc[nt][c][gv] = ok[nt][c] ? ldsf(svs + (rr[nt][c] * NG + gv) * 4) : 0.f;
                        vmax = fmaxf(vmax, vsc[nt][c][gv]);
                    }
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 1));
            vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 2));
            float f_lo = al_lo, f_hi = al_hi;     // factors applied to O
            if (vmax > 0.f) {
                const int ev = static_cast<int>((__float_as_uint(vmax) >> 23) & 0xffu) - 127;
                const int kn = min(kv, 14 - ev);
                if (kn < kv) {
                    const float drop = ldexpf(1.f, kn - kv);
                    f_lo *= drop;
                    f_hi *= drop;
                    kv = kn;
                }
            }
            const float up = ldexpf(1.f, kv);
#pragma unroll
            for (int n = 0; n < NTD; ++n) {
                o_lo[n][0] *= f_lo;
                o_lo[n][1] *= f_lo;
                if (G16) {
                    o_hi[n][0] *= f_hi;
                    o_hi[n][1] *= f_hi;
                }
            }
            // A fragments of P'' split into f16 hi + lo (P'' = hi + lo to ~2^-22)
            uint32_t ah[NGV][4], al[NGV][4];
#pragma unroll
            for (int gv = 0; gv < NGV; ++gv) {
                split_f16x2(pr_lo[0][0] * vsc[0][0][gv] * up, pr_lo[0][1] * vsc[0][1][gv] * up,
                            ah[gv][0], al[gv][0]);
                split_f16x2(pr_lo[1][0] * vsc[1][0][gv] * up, pr_lo[1][1] * vsc[1][1][gv] * up,
                            ah[gv][2], al[gv][2]);
                if (G16) {
                    split_f16x2(pr_hi[0][0] * vsc[0][0][gv] * up, pr_hi[0][1] * vsc[0][1][gv] * up,
                                ah[gv][1], al[gv][1]);
                    split_f16x2(pr_hi[1][0] * vsc[1][0][gv] * up, pr_hi[1][1] * vsc[1][1][gv] * up,
                                ah[gv][3], al[gv][3]);
                } else {
                    ah[gv][1] = ah[gv][3] = al[gv][1] = al[gv][3] = 0u;
                }
            }
            auto pv = [&](int n, int gv, uint32_t b0, uint32_t b1) {
                float acc[4] = {o_lo[n][0], o_lo[n][1], o_hi[n][0], o_hi[n][1]};
                ptx::mma_f16(acc, ah[gv][0], ah[gv][1], ah[gv][2], ah[gv][3], b0, b1);
                ptx::mma_f16(acc, al[gv][0], al[gv][1], al[gv][2], al[gv][3], b0, b1);
                o_lo[n][0] = acc[0];
                o_lo[n][1] = acc[1];
                o_hi[n][0] = acc[2];
                o_hi[n][1] = acc[3];
            };
            // B fragments from two pairs of V words: rows (R0, R1) give b0,
            // rows (R2, R3) give b1; byte e of the words is n-tile offset e.
            auto pv_words = [&](int n0, int gv, uint32_t w0, uint32_t w1, uint32_t w2,
                                uint32_t w3) {
                const uint32_t xl01 = ptx::prmt(w0, w1, 0x5140u);
                const uint32_t xh01 = ptx::prmt(w0, w1, 0x7362u);
                const uint32_t xl23 = ptx::prmt(w2, w3, 0x5140u);
                const uint32_t xh23 = ptx::prmt(w2, w3, 0x7362u);
                pv(n0 + 0, gv, ptx::bytes_to_f16x2(xl01, 0x4140u), ptx::bytes_to_f16x2(xl23, 0x4140u));
                pv(n0 + 1, gv, ptx::bytes_to_f16x2(xl01, 0x4342u), ptx::bytes_to_f16x2(xl23, 0x4342u));
                pv(n0 + 2, gv, ptx::bytes_to_f16x2(xh01, 0x4140u), ptx::bytes_to_f16x2(xh23, 0x4140u));
                pv(n0 + 3, gv, ptx::bytes_to_f16x2(xh01, 0x4342u), ptx::bytes_to_f16x2(xh23, 0x4342u));
            };
            if (!G32) {
                if constexpr (D == 128) {
                    // thread g owns head_dim bytes [16g, 16g + 16): n-tile n, MMA column c
                    // is head_dim 16c + n
                    const uint32_t col = 16 * g;
                    const uint4 v0 = lds128(sv + swz<D>(R0, col));
                    const uint4 v1 = lds128(sv + swz<D>(R1, col));
                    const uint4 v2 = lds128(sv + swz<D>(R2, col));
                    const uint4 v3 = lds128(sv + swz<D>(R3, col));
                    pv_words(0, 0, v0.x, v1.x, v2.x, v3.x);
                    pv_words(4, 0, v0.y, v1.y, v2.y, v3.y);
                    pv_words(8, 0, v0.z, v1.z, v2.z, v3.z);
                    pv_words(12, 0, v0.w, v1.w, v2.w, v3.w);
                } else {
                    // D == 64: thread g owns bytes [8g, 8g + 8): column c is 8c + n
                    const uint32_t col = 8 * g;
                    const uint2 v0 = lds64(sv + swz<D>(R0, col));
                    const uint2 v1 = lds64(sv + swz<D>(R1, col));
                    const uint2 v2 = lds64(sv + swz<D>(R2, col));
                    const uint2 v3 = lds64(sv + swz<D>(R3, col));
                    pv_words(0, 0, v0.x, v1.x, v2.x, v3.x);
                    pv_words(4, 0, v0.y, v1.y, v2.y, v3.y);
                }
            } else {
                // group-32: n-tile 4*gv + e covers head_dim 32*gv + 4*c + e (c = MMA
                // column), so thread g reads 4 bytes at 32*gv + 4*g of each row
#pragma unroll
                for (int gv = 0; gv < NGRP; ++gv) {
                    const uint32_t cb = 32 * gv + 4 * g;
                    pv_words(4 * gv, gv, lds32(sv + swz<D>(R0, cb)), lds32(sv + swz<D>(R1, cb)),
                             lds32(sv + swz<D>(R2, cb)), lds32(sv + swz<D>(R3, cb)));
                }
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_empty + 8 * s);
        if (warp == 0 && i + NST < ntiles) {
            // refill slot s once all four warps have released it
            if (!ptx::mbar_wait(bar_empty + 8 * s, (i / NST) & 1)) {
                if (lane == 0) raise_flag(p.d_err, KVQ_DEVERR_TIMEOUT);
                break;
            }
            issue(i + NST);
        }
    }
    if (warp == 0) asm volatile("cp.async.wait_all;" ::: "memory");

    // ---- merge the four warps' (m, l, o) into the CTA partial
    {
        const float down = ldexpf(1.f, -kv);         // undo the P'' prescale
#pragma unroll
        for (int n = 0; n < NTD; ++n) {
            o_lo[n][0] *= down;
            o_lo[n][1] *= down;
            o_hi[n][0] *= down;
            o_hi[n][1] *= down;
        }
    }
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    __syncthreads();                              // every stage consumed: reuse shared memory
    float* red = reinterpret_cast<float*>(smem);  // [NW][16][RS]
    float* red_m = red + Lay::RED_M;
    float* red_l = red + Lay::RED_L;
    // head_dim index of output n-tile n, column c (0/1) of this thread
    auto dcol = [&](int n, int c) -> int {
        if (G32) return 32 * (n >> 2) + 4 * (2 * t + c) + (n & 3);
        return (D == 128 ? 16 : 8) * (2 * t + c) + n;
    };
#pragma unroll
    for (int n = 0; n < NTD; ++n)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            red[(warp * 16 + g) * Lay::RS + dcol(n, c)] = o_lo[n][c];
            if (G16) red[(warp * 16 + g + 8) * Lay::RS + dcol(n, c)] = o_hi[n][c];
        }
    if (t == 0) {
        red_m[warp * 16 + g] = m_lo;
        red_l[warp * 16 + g] = l_lo;
        red_m[warp * 16 + g + 8] = G16 ? m_hi : -INFINITY;
        red_l[warp * 16 + g + 8] = G16 ? l_hi : 0.f;
    }
    __syncthreads();
    float* cp = red + Lay::CP;                    // [16][CPS]: o (unnormalised), m, l
    for (int idx = tid; idx < G * D; idx += NTHREADS) {
        const int h = idx / D, d = idx - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * 16 + h]);
        float acc = 0.f, lsum = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float mw = red_m[w * 16 + h];
            const float f = (mw == -INFINITY) ? 0.f : ptx::ex2(mw - M);
            acc = fmaf(f, red[(w * 16 + h) * Lay::RS + d], acc);
            lsum = fmaf(f, red_l[w * 16 + h], lsum);
        }
        cp[h * Lay::CPS + d] = acc;
        if (d == 0) {
            cp[h * Lay::CPS + D] = M;
            cp[h * Lay::CPS + D + 1] = lsum;
        }
    }
    __syncthreads();

    const int64_t bh0 = static_cast<int64_t>(b) * p.Hq + hk * G;   // first q head of the group
    if (S > 1) {
        // ---- cluster combine: partial j lives in CTA j's shared memory
        const uint32_t cp_addr = ptx::smem_u32(cp);
        if (tid < S) arrive_remote(mapa(bar_done, tid));
        if (!wait_cluster(bar_done, 0) && tid == 0) raise_flag(p.d_err, KVQ_DEVERR_TIMEOUT);
        float* cw = red + Lay::CW;                // [S][16] peer max, then weights
        float* cl = red + Lay::CL;                // [S][16] peer sums
        float* csum = red + Lay::CSUM;            // [16]
        for (int idx = tid; idx < S * G; idx += NTHREADS) {
            const int r = idx / G, h = idx - r * G;
            const uint32_t a = mapa(cp_addr + (h * Lay::CPS + D) * 4, r);
            cw[r * 16 + h] = ld_cluster_f32(a);
            cl[r * 16 + h] = ld_cluster_f32(a + 4);
        }
        __syncthreads();
        if (tid < G) {
            float M = -INFINITY;
            for (int r = 0; r < S; ++r) M = fmaxf(M, cw[r * 16 + tid]);
            float lsum = 0.f;
            for (int r = 0; r < S; ++r) {
                const float mr = cw[r * 16 + tid];
                const float w = (mr == -INFINITY) ? 0.f : ptx::ex2(mr - M);
                cw[r * 16 + tid] = w;
                lsum = fmaf(w, cl[r * 16 + tid], lsum);
            }
            csum[tid] = lsum;
        }
        __syncthreads();
        // this CTA writes outputs j*128 + tid, stepping by S*128
        for (int idx = j * NTHREADS + tid; idx < G * D; idx += S * NTHREADS) {
            const int h = idx / D, d = idx - h * D;
            const uint32_t a = cp_addr + (h * Lay::CPS + d) * 4;
            float acc = 0.f;
            for (int r = 0; r < S; ++r) acc = fmaf(cw[r * 16 + h], ld_cluster_f32(mapa(a, r)), acc);
            const float lsum = csum[h];
            p.out[(bh0 + h) * D + d] = lsum > 0.f ? acc / lsum : 0.f;
        }
        __syncthreads();
        // keep this CTA's shared memory alive until every peer has read it
        if (tid < S) arrive_remote(mapa(bar_read, tid));
        if (!wait_cluster(bar_read, 0) && tid == 0) raise_flag(p.d_err, KVQ_DEVERR_TIMEOUT);
    } else if (nsplit <= 1) {
        // single split (or empty sequence): the final row
        if (j == 0)
            for (int idx = tid; idx < G * D; idx += NTHREADS) {
                const int h = idx / D, d = idx - h * D;
                const float lsum = cp[h * Lay::CPS + D + 1];
                p.out[(bh0 + h) * D + d] = lsum > 0.f ? cp[h * Lay::CPS + d] / lsum : 0.f;
            }
    } else if (active) {
        // many splits without a cluster: partials for the combine kernel
        for (int idx = tid; idx < G * D; idx += NTHREADS) {
            const int h = idx / D, d = idx - h * D;
            p.ws_o[((bh0 + h) * p.splits + j) * D + d] = cp[h * Lay::CPS + d];
            if (d == 0) {
                p.ws_m[(bh0 + h) * p.splits + j] = cp[h * Lay::CPS + D];
                p.ws_l[(bh0 + h) * p.splits + j] = cp[h * Lay::CPS + D + 1];
            }
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
    using Lay = Layout<D, G32>;
    static bool done = false;
    if (done) return cudaSuccess;
    auto kern = decode_split_tc<D, G32, PAGED, G16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess) done = true;
    return e;
}

template <int D, bool G32, bool PAGED, bool G16>
cudaError_t launch_tc(const DecodeParams& p, cudaStream_t s) {
    using Lay = Layout<D, G32>;
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
    cfg.gridDim = dim3(p.splits, p.Hk, p.B);
    cfg.blockDim = dim3(NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = Lay::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (p.cluster > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = p.cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
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
    if (p.cluster > kMaxCluster || (p.cluster > 1 && p.cluster != p.splits))
        return cudaErrorInvalidValue;
    if (p.D == 128) return pick_layout<128>(p, s);
    if (p.D == 64) return pick_layout<64>(p, s);
    return cudaErrorInvalidValue;
}

int decode_max_cluster() {
    static int cached = 0;
    if (cached) return cached;
    // the most demanding variant (registers, shared memory) bounds every other
    auto kern = decode_split_tc<128, true, true, true>;
    int n = 0;
    if (set_attrs<128, true, true, true>() == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(kMaxCluster, 1, 1);
        cfg.blockDim = dim3(NTHREADS, 1, 1);
        cfg.dynamicSmemBytes = Layout<128, true>::SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kMaxCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxPotentialClusterSize(&n, kern, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();                           // a failed query leaves no sticky error
    n = n < 1 ? 1 : (n > kMaxCluster ? kMaxCluster : n);
    cached = n;
    return n;
}

}  // namespace kvq

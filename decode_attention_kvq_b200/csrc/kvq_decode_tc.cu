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
//    most one CTA per SM).  When the items fit the grid, CTA c takes item c
//    (one item per CTA); otherwise CTA c takes a contiguous block of items
//    whose weight (items, plus W per (b, kv head) started) is an equal share
//    of the total, found from prefix sums of the per-sequence chunk counts
//    (lengths cached in shared memory).  The items of one (b, kv head)
//    inside a CTA's block form a segment: one token range, one softmax
//    state.  A segment that is a whole (b, kv head) writes the final rows;
//    any other writes one partial state (o, m, l) into the workspace slot of
//    its first chunk, and with blocks of several items m = -inf into the
//    other slots it covers, so the combine kernel (kvq_decode.cu) finds a
//    unit's partials from its m slots.
//  * CTA = 1 producer warp (2 for the paged cache) + 8 consumer warps.  One
//    producer lane streams 128-token stages into a ring of 3-8 stages
//    (~150-220 KB of shared memory, one CTA per SM): K and V bytes by TMA
//    tile loads (2-D tensor maps over the cache rows, 128-byte swizzle for
//    D=128, 64-byte for D=64), the fp32 scales and, with a segment's first
//    two stages, its query rows by 1-D bulk copies; all complete on the
//    stage's mbarrier.  It refills a slot as soon as its consumers released
//    it.  The consumers form two groups of four warps that take alternate
//    stages (with 9 to 16 heads: every stage, group g taking heads 8g ..
//    8g + 7); a warp takes 32 tokens of its group's stage as two 16-token
//    MMA tiles.
//  * S^T = K . Q^T on the integer MMA (mma.sync m16n8k32, s32 accumulate),
//    with 8 query heads of the GQA group as the N = 8 dimension: the K
//    bytes are the A operand as loaded, and Q is
//    a per-head power-of-two prescaled 16-bit integer in two byte digits, so
//    S = 256 S_hi + S_lo - 128 sum(Qi) is exact.  The K scale (per token, or
//    per 32-value group with one fold per group), the prescale, attn_scale
//    and log2(e) are applied to the f32 scores.
//  * Online softmax in base 2 per head.  The V scale is folded into P:
//    P'' = 2^(z-m) * v_scale(token) * 2^kv (per 32-value group in group-32
//    mode), with a running per-warp power of two 2^kv that keeps P'' inside
//    the f16 normal range.  P'' is split into f16 hi + lo parts (about 22
//    significant bits together); each part is transposed from the score
//    accumulator layout into the P^T operand layout with movmatrix and
//    multiplied on mma.sync m16n8k16 (f32 accumulate) with the exact
//    (v - 128) integers, O^T += V^T . P^T (M = 16 head_dim rows, K = 16
//    tokens).
//  * Token order inside each 16-token MMA tile and the head_dim order of the
//    MMA k-dimension are permuted so that every shared-memory load of the
//    swizzled tiles is free of bank conflicts (sigma below).
//  * A segment's eight warp states are merged behind one named barrier
//    through head-major shared-memory rows (deterministic: no atomics).
//  * Programmatic dependent launch: the kernel waits for its predecessor in
//    the stream before touching inputs and lets the combine kernel launch
//    early.
//  * mbarrier waits are bounded (KVQ_DEVERR_TIMEOUT when one gives up, after
//    which every wait of the CTA returns at once); barriers are reached by
//    every participating thread unconditionally.
#include <cuda.h>
#include <cuda_fp8.h>
#include <math.h>

#include <atomic>
#include <climits>
#include <type_traits>
#include <unordered_map>

#include "kvq_devonce.h"
#include "kvq_internal.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

constexpr int NW = 8;                  // consumer warps per CTA
constexpr int NCONS = NW * 32;         // consumer threads
// producer warps: one; two for paged caches (K pages and V pages), whose
// stages take sixteen page copies
constexpr int nprod(bool paged) { return paged ? 2 : 1; }
constexpr int nthreads(bool paged) { return NCONS + 32 * nprod(paged); }
constexpr int WPG = 4;                 // consumer warps per group (a group works one stage)
constexpr int TT = 32 * WPG;           // tokens per stage: one 32-token slice per warp of a group
constexpr int kMaxB = kMaxBatch;       // sequences whose lengths are cached in shared memory

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

// Two FP8 bytes of w (bytes 0, 1 when hi == 0, bytes 2, 3 when hi == 1) ->
// f16x2 holding their exact values.  F8 == 2 (E5M2): the byte is the top
// byte of the f16 of the same value.  F8 == 1 (E4M3): the hardware fp8x2 ->
// f16x2 conversion.
template <int F8>
__device__ __forceinline__ uint32_t fp8x2_to_f16x2(uint32_t w, int hi) {
    if constexpr (F8 == 2) {
        return ptx::prmt(w, 0u, hi ? 0x3424u : 0x1404u);
    } else {
        // the two bytes as an fp8x2 value (first byte in the low half), one
        // hardware conversion to f16x2 (exact: E4M3 values are f16 values)
        const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((w >> (hi ? 16 : 0)) & 0xffffu), __NV_E4M3);
        return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
    }
}

// 8x8 b16 transpose across the warp (fragment of row lane/4, columns
// 2*(lane%4) and +1, in and out).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Shared-memory plan (one CTA per SM): a ring of NST stages (K and V bytes of
// 128 tokens, their scales, room for one segment's query rows), the merge
// slots, the cached lengths and chunk prefix sums, the stage mbarriers and
// per-warp head maxima.
template <int D, bool G32, bool G16>
struct Layout {
    static constexpr int NG = G32 ? D / 32 : 1;
    static constexpr int KV_BYTES = TT * D;
    static constexpr int SC_FLOATS = TT * NG + 4;   // + room for a 16-byte alignment offset
    static constexpr int Q_OFF = 2 * KV_BYTES + 2 * SC_FLOATS * 4;   // within a stage
    static constexpr int Q_BYTES = (G16 ? 16 : 8) * D * 2;           // bf16 query rows
    static constexpr int MASK_OFF = Q_OFF + Q_BYTES;                 // paged: valid-page bits
    static constexpr int STAGE = ((MASK_OFF + 16) + 1023) / 1024 * 1024;
    static constexpr int NV = (D / 16) * 4;                         // o floats per lane
    static constexpr int MERGE_BYTES = NW * NV * 32 * 4;
    static constexpr int LENS_BYTES = (3 * kMaxB + 1) * 4;          // lengths, chunks, prefix sums
    static constexpr int PARAM_BYTES = 256;                         // the kernel parameters
    static constexpr int MISC_BYTES = 1536;                         // barriers, maxima, flags
    static constexpr int BUDGET =
        227 * 1024 - 1024 - MERGE_BYTES - LENS_BYTES - PARAM_BYTES - MISC_BYTES;
    static constexpr int NST = (BUDGET / STAGE) > 8 ? 8 : (BUDGET / STAGE);
    static_assert(NST >= 3, "at least three stages");
    static constexpr int MERGE_OFF = NST * STAGE;
    static constexpr int LENS_OFF = MERGE_OFF + MERGE_BYTES;
    static constexpr int PARAM_OFF = (LENS_OFF + LENS_BYTES + 15) / 16 * 16;
    static constexpr int MISC_OFF = PARAM_OFF + PARAM_BYTES;
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
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ float ldsf(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

// The run of work items of one (sequence, kv head) that starts at item i and
// stays inside [i, iend): chunks j0..j1 of sequence b, kv head hk, i.e.
// tokens [t0, t1).  Items are listed in (b, kv head, chunk) order and
// cum[b] counts the items of sequences before b (Hk * max(1, ns) each).
// 2^e for -126 <= e <= 127, exact.
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// Merge-slot swizzle: chunk k (16 bytes) of head h's row is stored at
// k ^ mswz(h).  The eight lanes of a quarter warp store chunks of heads
// 2t + c (t = lane % 4) whose unswizzled indices differ only in one bit
// (bit 2 per-token at D = 128, bit 1 at D = 64, bit 0 in group-32 mode);
// XOR-ing t into the two other low bits makes the eight chunks fall into
// eight different bank quads.  mswz(h) < 8, so an aligned run of eight
// chunks of one row stays a run of eight distinct quads for the readers.
template <int D, bool G32>
__device__ __forceinline__ int mswz(int h) {
    const int t = (h >> 1) & 3;
    if constexpr (G32) return t << 1;
    else if constexpr (D == 128) return t;
    else return (t & 1) | ((t & 2) << 1);
}

struct Seg {
    int b, hk, ns, j0, j1, t0, t1;
    int next;                      // first item after the run
};

__device__ __forceinline__ Seg seg_at(int i, int iend, const int* lens, const int* nsv,
                                      const int* cum, int B, int chunk) {
    int lo = 0, hi = B;            // largest b with cum[b] <= i
#pragma unroll 1
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= i) lo = mid;
        else hi = mid;
    }
    Seg sg;
    sg.b = lo;
    sg.ns = nsv[lo];
    const int per = sg.ns > 0 ? sg.ns : 1;
    const int r = i - cum[lo];
    sg.hk = r / per;
    sg.j0 = r - sg.hk * per;
    sg.next = min(iend, cum[lo] + (sg.hk + 1) * per);
    sg.j1 = sg.j0 + (sg.next - i) - 1;
    sg.t0 = sg.j0 * chunk;
    sg.t1 = sg.ns > 0 ? min((sg.j1 + 1) * chunk, lens[lo]) : 0;
    return sg;
}

// PK (group-32, G <= 4): the 8 columns of an MMA n-tile carry the G heads
// twice, columns 4*par + h for the two parities par of the 32-value groups.
// A Q.K^T k-step over group gi fills only the columns of parity gi % 2 (the
// others' Q digits are zero), so groups 2a and 2a + 1 share one accumulator
// and one fold; lanes t and t ^ 2 (the two parities) add their scores.  P''
// is built once per group pair, each column with its own parity's V scale;
// the P.V output columns of the other parity are not used.
// CAUSAL (a chunk of T = p.qlen queries per sequence and q head, or a
// sliding window): the G columns are (head, query i) rows, query fastest, and
// column i of a sequence of length L sees the positions <= L - T + i (L
// counts the chunk's tokens) and, with a window w, >= L - T + i - w + 1.
// With a window the tokens are counted from the sequence's window base.
// Fused append: the warp whose 32-token slice of a landed stage holds the
// new token (position tok of unit (b, hk), stage row r) quantises it -- the
// append kernels' quantiser -- into the stage's K and V rows and scales (sk,
// sv, sks, svs: shared-memory addresses) and, if to_cache, into the cache,
// before any of its MMA operands are read.  (G16: the slice's warp of each
// group does this; both write the same bits into the stage, and only group
// 0's writes the cache.)  Lane l takes head_dim values [l * VPL,
// (l + 1) * VPL) of k_new and v_new.  Only the fused instantiation of the
// split kernel (VAR == 2) contains it.
template <int D, bool G32, bool PAGED>
__device__ __forceinline__ void patch_new_token(const DecodeParams& p, uint32_t sk, uint32_t sv,
                                             uint32_t sks, uint32_t svs, int r, int tok, int b,
                                             int hk, bool to_cache) {
    constexpr int VPL = D / 32;          // values per lane
    constexpr int NG = G32 ? D / 32 : 1;
    const int lane = threadIdx.x & 31;
    uint32_t kx[2] = {0u, 0u}, vx[2] = {0u, 0u};
    const int64_t nrow = (static_cast<int64_t>(b) * p.Hk + hk) * D + lane * VPL;
    if constexpr (VPL == 4) {
        const uint2 a = *reinterpret_cast<const uint2*>(p.k_new + nrow);
        const uint2 c = *reinterpret_cast<const uint2*>(p.v_new + nrow);
        kx[0] = a.x; kx[1] = a.y;
        vx[0] = c.x; vx[1] = c.y;
    } else {
        kx[0] = *reinterpret_cast<const uint32_t*>(p.k_new + nrow);
        vx[0] = *reinterpret_cast<const uint32_t*>(p.v_new + nrow);
    }
    float xk[VPL], xv[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
        xk[e] = bf16_bits_to_f32((kx[e >> 1] >> (16 * (e & 1))) & 0xffffu);
        xv[e] = bf16_bits_to_f32((vx[e >> 1] >> (16 * (e & 1))) & 0xffffu);
    }
    float ak = 0.f, av = 0.f;
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
        ak = fmaxf(ak, fabsf(xk[e]));
        av = fmaxf(av, fabsf(xv[e]));
    }
    // per token: over the warp; group-32: over the 32 / VPL lanes of a group
    constexpr int RED = G32 ? 32 / VPL : 32;
#pragma unroll
    for (int off = 1; off < RED; off <<= 1) {
        ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
        av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
    }
    const float sck = q8_scale(ak), scv = q8_scale(av);
    const float ik = __frcp_rn(sck), iv = __frcp_rn(scv);
    uint32_t bk = 0u, bv = 0u;
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
        bk |= q8_byte(xk[e], sck, ik) << (8 * e);
        bv |= q8_byte(xv[e], scv, iv) << (8 * e);
    }
    const int gidx = G32 ? (lane * VPL) >> 5 : 0;
    const bool lead = G32 ? ((lane * VPL) & 31) == 0 : lane == 0;
    const uint32_t off = swz<D>(static_cast<uint32_t>(r), static_cast<uint32_t>(lane * VPL));
    int64_t crow;
    if constexpr (PAGED) {
        const int32_t pg = p.table[static_cast<int64_t>(b) * p.max_pages + (tok >> 4)];
        crow = (static_cast<int64_t>(pg) * p.Hk + hk) * 16 + (tok & 15);
    } else {
        crow = (static_cast<int64_t>(b) * p.Hk + hk) * p.max_seq + tok;
    }
    if constexpr (VPL == 4) {
        sts_u32(sk + off, bk);
        sts_u32(sv + off, bv);
        if (to_cache) {
            *reinterpret_cast<uint32_t*>(p.k_w + crow * D + lane * VPL) = bk;
            *reinterpret_cast<uint32_t*>(p.v_w + crow * D + lane * VPL) = bv;
        }
    } else {
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(sk + off), "h"(static_cast<uint16_t>(bk)) : "memory");
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(sv + off), "h"(static_cast<uint16_t>(bv)) : "memory");
        if (to_cache) {
            *reinterpret_cast<uint16_t*>(p.k_w + crow * D + lane * VPL) = static_cast<uint16_t>(bk);
            *reinterpret_cast<uint16_t*>(p.v_w + crow * D + lane * VPL) = static_cast<uint16_t>(bv);
        }
    }
    if (lead) {
        sts_f32(sks + (r * NG + gidx) * 4, sck);
        sts_f32(svs + (r * NG + gidx) * 4, scv);
        if (to_cache) {
            p.ks_w[crow * NG + gidx] = sck;
            p.vs_w[crow * NG + gidx] = scv;
        }
    }
    // the slot is refilled by TMA (async proxy) after these generic writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
}


template <int D, bool G32, bool PAGED, bool G16, bool PK, int VAR, int F8, bool ST>
__global__ void __launch_bounds__(nthreads(PAGED), 1)
decode_split_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ DecodeParams prm) {
    // VAR: 0 decode, 1 masked (chunks of queries, sliding windows), 2 decode
    // with the fused append of the step's new token
    constexpr bool CAUSAL = VAR == 1;
    constexpr bool FUSED = VAR == 2;
    using Lay = Layout<D, G32, G16>;
    constexpr int NG = Lay::NG;
    constexpr int NST = Lay::NST;
    constexpr int NV = Lay::NV;
    constexpr int NGRP = D / 32;        // 32-value groups over head_dim
    constexpr int MT = D / 16;          // m-tiles of O^T over head_dim (PV)
    // n-tiles of 8 query heads per warp.  G16 (9 to 16 heads): the two groups
    // split the heads (group grp takes heads 8 grp .. 8 grp + 7) and both work
    // every stage, so a warp still holds one n-tile of state
    constexpr int NT = 1;
    constexpr int NGV = G32 ? NG : 1;   // V scales per token
    static_assert(!PK || (G32 && !G16), "packing: group-32 scales, at most 4 heads");
    static_assert(!(PK && CAUSAL), "chunk queries: unpacked columns");
    static_assert(F8 == 0 || !G32, "FP8 caches have no scales");
    static_assert(!ST || (F8 == 0 && !G32), "per-head / per-channel scales: INT8, no groups");
    static_assert(!FUSED || (F8 == 0 && !ST), "fused append: INT8 per token / group-32");
    // no scale rows in the ring: FP8 (no scales) and per-head / per-channel
    // scales (one set per (sequence, kv head), folded into Q and the output)
    constexpr bool NOSC = F8 != 0 || ST;
    constexpr int NVS = PK ? NGRP / 2 : NGV;   // P'' operand sets (PK: group pairs)

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tid = threadIdx.x;
    const int g = lane >> 2, t = lane & 3;
    const int par = PK ? (t >> 1) : 0;  // PK: parity of this thread's MMA columns

    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar_full = sbase + Lay::MISC_OFF;
    const uint32_t bar_empty = bar_full + NST * 8;
    // per-warp head maxima and sums of a segment (read after the merge
    // barrier; the next segment's writers first wait on bar_mfree, which
    // completes once every consumer warp has read them and the slots)
    float* mrg_m = reinterpret_cast<float*>(smem + Lay::MISC_OFF + 2 * NST * 8);  // [16][NW]
    float* mrg_l = mrg_m + 16 * NW;                                               // [16][NW]
    // completes when all consumer warps have read a segment's maxima and slots
    const uint32_t bar_mfree = ptx::smem_u32(mrg_l + 16 * NW);
    // one item per CTA: the query rows' own barrier (they land ahead of stage 0)
    const uint32_t bar_q = bar_mfree + 8;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(mrg_l + 16 * NW + 4);
    static_assert(2 * NST * 8 + 2 * 16 * NW * 4 + 16 + 4 <= Lay::MISC_BYTES,
                  "barriers, maxima, flag");
    float* mslot = reinterpret_cast<float*>(smem + Lay::MERGE_OFF);   // [NW][8 heads][D]
    int* lens = reinterpret_cast<int*>(smem + Lay::LENS_OFF);                     // [B]
    int* nsv = lens + kMaxB;                                                     // [B] chunks
    int* cum = nsv + kMaxB;                                                      // [B + 1]
    DecodeParams* sprm = reinterpret_cast<DecodeParams*>(smem + Lay::PARAM_OFF);

    // the parameters are copied to shared memory in one parallel round of
    // parameter-space reads (their latency overlaps the dependency wait);
    // every later use is a shared-memory load
    static_assert(sizeof(DecodeParams) % 4 == 0 && sizeof(DecodeParams) <= Lay::PARAM_BYTES,
                  "the parameters fit their shared-memory copy");
    if (tid < static_cast<int>(sizeof(DecodeParams) / 4))
        reinterpret_cast<uint32_t*>(sprm)[tid] = reinterpret_cast<const uint32_t*>(&prm)[tid];
    if (tid == 0) {
        ptx::prefetch_tensormap(&tm_k);     // kernel parameters: safe before the dependency wait
        ptx::prefetch_tensormap(&tm_v);
#pragma unroll 1
        for (int s = 0; s < NST; ++s) {
            // the producer's expect_tx arrival (paged: one per producer warp, plus
            // one cp.async arrival per lane of producer warp 0 for the scales)
            ptx::mbar_init(bar_full + 8 * s, PAGED ? 2 + 32 : 1);
            ptx::mbar_init(bar_empty + 8 * s, G16 ? 2 * WPG : WPG);
        }
        ptx::mbar_init(bar_mfree, NW);
        ptx::mbar_init(bar_q, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (!PAGED && prm.one_item && !prm.window && tid == 32) {
        // one item per CTA, contiguous cache: the item's first two stages of K
        // and V rows (and their scales) do not depend on the length, so they
        // are prefetched into L2 while the predecessor finishes (more than two
        // stages holds up the CTA's own first loads behind the prefetch).  A prefetch moves
        // nothing into this SM: the loads after the dependency wait still see
        // every write the predecessor makes.
        const int c = blockIdx.x;
        const int pb = c / max(prm.Hk * prm.splits, 1);
        const int pr = c - pb * prm.Hk * prm.splits;
        const int phk = pr / prm.splits;
        const int64_t pt0 = static_cast<int64_t>(pr - phk * prm.splits) * prm.chunk;
        const int64_t prow = static_cast<int64_t>(pb * prm.Hk + phk) * prm.max_seq;
        const int64_t nrow = min(static_cast<int64_t>(min(prm.chunk, 2 * TT)), prm.max_seq - pt0);
        if (nrow > 0) {
            const uint32_t kvb = static_cast<uint32_t>(nrow * D);
            ptx::prefetch_l2(prm.k + (prow + pt0) * D, kvb);
            ptx::prefetch_l2(prm.v + (prow + pt0) * D, kvb);
            // scales: the 16-byte aligned span that covers the rows' floats
            // and stays inside the scale arrays
            const int64_t f0 = (prow + pt0) * Lay::NG;
            const int64_t f1 = min((prow + pt0 + nrow) * Lay::NG + 3,
                                   static_cast<int64_t>(prm.B) * prm.Hk * prm.max_seq * Lay::NG) &
                               ~static_cast<int64_t>(3);
            const int64_t a0 = f0 & ~static_cast<int64_t>(3);
            if (!NOSC && f1 > a0) {
                ptx::prefetch_l2(prm.k_scale + a0, static_cast<uint32_t>((f1 - a0) * 4));
                ptx::prefetch_l2(prm.v_scale + a0, static_cast<uint32_t>((f1 - a0) * 4));
            }
        }
    }
    // the predecessor's writes (q, cache, lengths) are visible after the
    // dependency wait.  One item per CTA: nothing before the roles reads
    // them, so each role waits just before its first global access and the
    // producer's set-up overlaps the predecessor's tail.
    if (!prm.one_item) grid_dep_wait();
    grid_dep_launch();                  // the combine kernel may be scheduled now

    // one item per CTA (the plan's items fit the grid): CTA c takes item c of
    // the plan, (b, kv head, chunk j) = c in (b, kv head, j) order, whatever the
    // lengths; the producer issues its first stage before the length arrives
    const bool one = prm.one_item != 0;
    // ---- lengths and chunk prefix sums (items per sequence: Hk * max(1, chunks))
    if (!one) {
        const int64_t cap = PAGED ? static_cast<int64_t>(prm.max_pages) * prm.page_size : prm.max_seq;
        const int64_t plan = static_cast<int64_t>(prm.splits) * prm.chunk;
#pragma unroll 1
        for (int b = tid; b < prm.B; b += nthreads(PAGED)) {
            const int Lraw = prm.seq_lens[b];
            // tokens walked from the window base (all of them without a window)
            int L = walked_len(Lraw, cap, plan, prm.qlen, prm.window, prm.recent);
            // (a chunk of queries needs its own tokens in the cache: L >= T)
            if (L < 0 || (CAUSAL && Lraw > 0 && Lraw < prm.qlen)) {
                if (blockIdx.x == 0) raise_flag(prm.d_err, KVQ_DEVERR_LEN);
                L = 0;
            }
            lens[b] = L;
            const int ns = (L + prm.chunk - 1) / prm.chunk;
            nsv[b] = ns;
            cum[b + 1] = prm.Hk * (ns > 0 ? ns : 1);
        }
    }
    __syncthreads();
    const DecodeParams& p = *sprm;
    const int B = p.B;
    const int G = p.G;
    if (!one && warp == 0) {            // inclusive scan of cum[1..B] by one warp
        int carry = 0;
#pragma unroll 1
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
    if (!one) __syncthreads();
    // CTA c takes items [c*q + min(c, r), ...) with q = T / grid, r = T % grid
    // (the first r CTAs one item more); T < 2^31 is checked by the host
    // ---- the CTA's block of items.  Every (sequence, kv head) unit weighs its
    // items plus W, the cost of starting it; CTA c takes the equal share
    // [c * TW / grid, (c + 1) * TW / grid) of the total weight TW (the first
    // TW % grid CTAs one more), mapped back to items.
    const int T = cum[B];
    const int W = p.seg_w;
    const int HkW = p.Hk * W;
    const int TW = T + HkW * B;
    auto item_of = [&](int x) {          // first item at or after weight position x
        if (x >= TW) return T;
        int lo = 0, hi = B;              // largest b with wcum(b) <= x
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cum[mid] + HkW * mid <= x) lo = mid;
            else hi = mid;
        }
        const int per = max(nsv[lo], 1);
        const int r = x - (cum[lo] + HkW * lo);
        const int hk = r / (per + W);
        const int jw = r - hk * (per + W);
        return cum[lo] + hk * per + max(jw - W, 0);
    };
    const int grid = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
    int ibeg = c, iend = c + 1;
    if (!one) {
        const int wq = TW / grid, wr = TW % grid;
        ibeg = W ? item_of(c * wq + min(c, wr)) : c * wq + min(c, wr);
        iend = W ? item_of((c + 1) * wq + min(c + 1, wr)) : (c + 1) * wq + min(c + 1, wr);
    }
    // one item per CTA: the item, and its length read straight from the caller
    const int one_b = c / max(p.Hk * p.splits, 1);
    const int one_r = c - one_b * p.Hk * p.splits;
    const int one_hk = one_r / p.splits, one_j = one_r - one_hk * p.splits;
    // the length as read, and as used: a length beyond the capacity or the
    // planned window reads as 0 (flagged once, by the first consumer thread of
    // the sequence's first CTA)
    auto one_raw = [&]() { return p.seq_lens[one_b]; };
    auto one_valid = [&](int Lraw) {
        const int64_t cap = PAGED ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
        int L = walked_len(Lraw, cap, static_cast<int64_t>(p.splits) * p.chunk, p.qlen, p.window,
                           p.recent);
        if (L < 0 || (CAUSAL && Lraw > 0 && Lraw < p.qlen)) {
            if (one_j == 0 && one_hk == 0 && tid == 32 * nprod(PAGED)) raise_flag(p.d_err, KVQ_DEVERR_LEN);
            L = 0;
        }
        return L;
    };
    auto one_seg = [&](int L) {
        Seg sg;
        sg.b = one_b;
        sg.hk = one_hk;
        sg.j0 = sg.j1 = one_j;
        sg.ns = (L + p.chunk - 1) / p.chunk;
        sg.t0 = one_j * p.chunk;
        sg.t1 = max(sg.t0, min(sg.t0 + p.chunk, L));
        sg.next = iend;
        return sg;
    };
    // bounded wait that gives up at once after any earlier timeout of this CTA
    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (*abort_flag) return;
        if (!ptx::mbar_wait(bar, parity)) {
            *abort_flag = 1;
            if (lane == 0) raise_flag(p.d_err, KVQ_DEVERR_TIMEOUT);
        }
    };

    // ------------------------------------------------------------ producer
    if (warp < nprod(PAGED)) {
        const int pw = warp;            // producer warp index
        // one lane issues every copy of a stage (TMA tiles for K and V, 1-D bulk
        // copies for the scales and the query rows); all complete on the stage's
        // mbarrier, whose single arrival is the expect_tx below
        const uint64_t pol = ptx::policy_evict_first();
        // the parameters this loop uses live in registers: the asm statements
        // below clobber memory, so reads through p would be repeated after each
        // of them (shared-memory loads queued behind the consumers' traffic)
        const int Hk = p.Hk, Hq = p.Hq, chunk = p.chunk, max_seq = p.max_seq;
        const int max_pages = p.max_pages, num_pages = p.num_pages;
        const float* const k_scale = p.k_scale;
        const float* const v_scale = p.v_scale;
        const uint16_t* const qg = p.q;
        const int32_t* const table = p.table;
        int32_t* const d_err = p.d_err;
        // sliding window: rows are addressed from the sequence's window base
        const int window = p.window, qlen = p.qlen;
        const int32_t* const seq_lens = p.seq_lens;
        const int64_t cap_tok = PAGED ? static_cast<int64_t>(max_pages) * p.page_size : max_seq;
        // floats in each scale array (contiguous layout)
        const int64_t sc_total = static_cast<int64_t>(B) * Hk * max_seq * NG;
        const uint32_t q_bytes = static_cast<uint32_t>(G * D * 2);
        // the issue loop is compiled once for blocks of items and once for one
        // item per CTA, so the former carries none of the latter's bookkeeping
        auto produce = [&](auto one_tag) {
            constexpr bool ONE = decltype(one_tag)::value;
            int count = 0;                  // tiles issued (ring position)
            if (ONE) grid_dep_wait();       // before the length, table, q and cache reads
#pragma unroll 1
            for (int i = ibeg; i < iend;) {
                // one item per CTA: the length load is issued first and used only
                // after the first stage is on its way (the chunk's end stands in)
                int Lone = 0;
                if (ONE) Lone = one_raw();
                const Seg sg = ONE ? one_seg((one_j + 1) * chunk) : seg_at(i, iend, lens, nsv, cum, B, chunk);
                i = sg.next;
                if (sg.ns == 0) continue;
                int t1 = sg.t1;
                uint32_t spec_valid = ~0u;      // paged, ONE item: the first stage's loaded pages
                const int b = sg.b, hk = sg.hk;
                int wb = 0;                     // the window base (a multiple of 16)
                if (CAUSAL && window > 0) {
                    const int Lr = ONE ? Lone : seq_lens[b];
                    wb = (Lr >= 0 && Lr <= cap_tok) ? window_base(Lr, qlen, window) : 0;
                }
                const uint16_t* qsrc = qg + (static_cast<int64_t>(b) * Hq + hk * G) * D;
                int seg_tiles = 0;          // tiles issued for this segment
                if (ONE && pw == 0 && lane == 0) {
                    // one item per CTA: the query rows go first, on their own
                    // barrier, into stage 0's query area (no stage carries them), so
                    // the consumers build their Q operand while K and V are in flight
                    ptx::mbar_arrive_expect_tx(bar_q, q_bytes);
                    ptx::bulk_load(sbase + Lay::Q_OFF, qsrc, q_bytes, bar_q);
                }
                // paged: the segment's page ids, 32 pages (4 stages) per register,
                // loaded ONE group of 4 stages ahead so the table read is off the
                // issue path; lane i holds page pbase + i (-1: none or out of range)
                int pbase = sg.t0 >> 4;
                int32_t pg_cur = -1, pg_nxt = -1;
                auto load_pages = [&](int first) {
                    const int idx = first + lane;           // counted from the window base
                    const int ia = (wb >> 4) + idx;         // the logical page
                    int32_t v = -1;
                    if (16 * idx < t1 && ia < max_pages) {
                        v = table[static_cast<int64_t>(b) * max_pages + ia];
                        if (v < 0 || v >= num_pages) v = -1;
                    }
                    return v;
                };
                if (PAGED) {
                    pg_cur = load_pages(pbase);
                    pg_nxt = load_pages(pbase + 32);
                }
#pragma unroll 1
                for (int tt0 = sg.t0; tt0 < t1; tt0 += TT, ++count, ++seg_tiles,
                         t1 = (ONE && seg_tiles == 1) ? max(sg.t0, min(sg.t0 + chunk, one_valid(Lone))) : t1) {
                    const int s = count % NST;
                    const uint32_t full = bar_full + 8 * s;
                    if (count >= NST && lane == 0) wait(bar_empty + 8 * s, ((count / NST) - 1) & 1);
                    __syncwarp();
                    const int ntok = min(TT, t1 - tt0);
                    const uint32_t sk = sbase + s * Lay::STAGE;
                    const uint32_t sv = sk + Lay::KV_BYTES;
                    const uint32_t sks = sv + Lay::KV_BYTES;
                    const uint32_t svs = sks + Lay::SC_FLOATS * 4;
                    // the segment's G query rows (contiguous bf16) ride with its first
                    // two stages: each consumer group builds its Q operand from the
                    // first stage it works in the segment (one item per CTA: they
                    // came first, on their own barrier)
                    const bool with_q = !ONE && seg_tiles < 2;
                    if (!PAGED) {
                        if (lane == 0) {
                            const int64_t row0 = (static_cast<int64_t>(b) * Hk + hk) * max_seq + wb + tt0;
                            // scales: whole 16-byte chunks from the aligned float at or
                            // below the tile's first ONE; where the last chunk would run
                            // past the end of the scale array its 1-3 floats are copied
                            // by plain loads (before the arrival that publishes them)
                            int nb = 0;             // 16-byte chunks of scales (none for FP8)
                            int64_t c0 = 0;
                            if constexpr (!NOSC) {
                                const int64_t f0 = row0 * NG;
                                const int off = static_cast<int>(f0 & 3);
                                c0 = f0 - off;
                                const int nf = ntok * NG + off;
                                nb = (nf + 3) & ~3;
                                if (c0 + nb > sc_total) {
                                    nb = nf & ~3;
#pragma unroll 1
                                    for (int e = nb; e < nf; ++e) {
                                        sts_f32(sks + 4 * e, k_scale[c0 + e]);
                                        sts_f32(svs + 4 * e, v_scale[c0 + e]);
                                    }
                                }
                            }
                            ptx::mbar_arrive_expect_tx(
                                full, 2 * Lay::KV_BYTES + 8 * nb + (with_q ? q_bytes : 0u));
                            ptx::tma_load_2d(sk, &tm_k, 0, static_cast<int>(row0), full, pol);
                            ptx::tma_load_2d(sv, &tm_v, 0, static_cast<int>(row0), full, pol);
                            if (!NOSC && nb > 0) {
                                ptx::bulk_load(sks, k_scale + c0, 4 * nb, full);
                                ptx::bulk_load(svs, v_scale + c0, 4 * nb, full);
                            }
                            if (with_q) ptx::bulk_load(sk + Lay::Q_OFF, qsrc, q_bytes, full);
                        }
                    } else {
                        constexpr uint32_t PAGE_BYTES = 16 * D;   // TMA bytes of K (or V) per page
                        const int np = (ntok + 15) >> 4;
                        if ((tt0 >> 4) >= pbase + 32) {
                            pbase += 32;
                            pg_cur = pg_nxt;
                            pg_nxt = load_pages(pbase + 32);
                        }
                        // a bad entry is skipped (its tokens are masked)
                        int32_t pg = __shfl_sync(0xffffffffu, pg_cur, (tt0 >> 4) - pbase + (lane & 7));
                        if (lane >= np) pg = -1;
                        const uint32_t valid = __ballot_sync(0xffffffffu, pg >= 0);
                        if (pw == 1) {
                            // producer warp 1: the V rows of the pages (lane q < 8 loads
                            // page q: 16 rows of this kv head), its own byte count
                            if (lane == 0) ptx::mbar_arrive_expect_tx(full, __popc(valid) * PAGE_BYTES);
                            __syncwarp();
                            if (pg >= 0)
                                ptx::tma_load_2d(sv + lane * 16 * D, &tm_v, 0, (pg * Hk + hk) * 16, full,
                                                 pol);
                            continue;
                        }
                        if (lane == 0) {
                            // the consumers mask the tokens of pages that were not
                            // loaded; a bad table entry is reported here
                            // (one item per CTA: the first stage's range is the chunk's, not
                            // yet the length's; its pages are checked once the length is known)
                            if (ONE && seg_tiles == 0) spec_valid = valid;
                            else if (valid != (1u << np) - 1u) raise_flag(d_err, KVQ_DEVERR_PAGE);
                            sts_u32(sk + Lay::MASK_OFF, valid);
                            ptx::mbar_arrive_expect_tx(
                                full, __popc(valid) * PAGE_BYTES + (with_q ? q_bytes : 0u));
                            if (with_q) ptx::bulk_load(sk + Lay::Q_OFF, qsrc, q_bytes, full);
                        }
                        __syncwarp();
                        // producer warp 0: lane q < 8 loads page q's K rows; every lane
                        // copies 16-byte chunks of the pages' scales (16 * NG aligned
                        // floats per page), chunk c of the stage being page c / (4 NG)
                        if (pg >= 0)
                            ptx::tma_load_2d(sk + lane * 16 * D, &tm_k, 0, (pg * Hk + hk) * 16, full, pol);
#pragma unroll
                        for (int it = 0; it < (NOSC ? 0 : NG); ++it) {
                            const int c = lane + 32 * it;
                            const int q = c / (4 * NG), cc = c % (4 * NG);
                            const int pq = __shfl_sync(0xffffffffu, pg, q);
                            if (pq >= 0) {
                                const int64_t fc = static_cast<int64_t>((pq * Hk + hk) * 16) * NG + 4 * cc;
                                ptx::cp_async_16(sks + 16 * c, k_scale + fc);
                                ptx::cp_async_16(svs + 16 * c, v_scale + fc);
                            }
                        }
                        ptx::cp_async_arrive_noinc(full);
                    }
                }
                if (PAGED && ONE && lane == 0) {
                    // the first stage's pages inside the sequence must all have loaded
                    const int nreal = min(max(t1 - sg.t0, 0), TT);
                    const uint32_t need = nreal >= 16 * 32 ? ~0u : (1u << ((nreal + 15) >> 4)) - 1u;
                    if ((spec_valid & need) != need) raise_flag(d_err, KVQ_DEVERR_PAGE);
                }
            }
            // the last tile of every slot has landed (normally long consumed; after a
            // timeout this keeps the CTA alive until its bulk copies are done)
            if (PAGED) asm volatile("cp.async.wait_all;" ::: "memory");
            if (lane == 0)
#pragma unroll 1
                for (int c = count - 1; c >= 0 && c >= count - NST; --c)
                    ptx::mbar_wait(bar_full + 8 * (c % NST), (c / NST) & 1);
            if (ONE && pw == 0 && lane == 0) ptx::mbar_wait(bar_q, 0);
        };
        if (one) produce(std::true_type{});
        else produce(std::false_type{});
        return;                         // consumers synchronise among themselves (barrier 1)
    }

    // ------------------------------------------------------------ consumers
    // Two groups of four warps take alternate stages (tile c of the CTA goes
    // to group c % 2), so two stages are in work at once.  Inside a stage,
    // warp wg of the group owns rows [32 wg, 32 wg + 32) as two 16-token MMA
    // tiles u = 0, 1 that share one online-softmax step.
    const int cw = warp - nprod(PAGED);            // consumer warp index
    const int ctid = tid - 32 * nprod(PAGED);      // consumer thread index
    if (one) grid_dep_wait();           // before the length read and any global write
    const int grp = cw / WPG, wg = cw % WPG;
    const int hofs = G16 ? 8 * grp : 0;          // the warp's first query head (column)
    const int sig_g = sigma(g);
    const int sig_a = sigma(2 * t), sig_b = sigma(2 * t + 1);

    constexpr int NCG = G32 ? NGRP : 1;   // offset terms per head (per 32-value group)
    uint32_t qh0[NT][NGRP], qh1[NT][NGRP], ql0[NT][NGRP], ql1[NT][NGRP];   // Q digits
    int qc[NT][2][NCG];                   // 128 * sum(Qi) of the thread's two heads
    float zs[NT][2];
    float m[NT][2], l[NT][2];
    float o[MT][NT][4];                 // O^T C fragments: rows = head_dim, columns = heads
    int kv = 64;                        // running P'' prescale exponent (per warp)
    int c_count = 0;                    // tiles of the CTA seen so far (ring position)
    int merges = 0;                     // segment merges of the CTA so far

    // ---- Q^T operand from the segment's query rows at sq (they ride with its
    // first two stages; one item per CTA: they come ahead of stage 0).
    // Column n = g of n-tile nt is query head 8*nt + g.
    // Each head is scaled by 2^sh so max |q| * 2^sh is in [2^14, 2^15)
    // and rounded to a 16-bit integer Qi = 256 * hi + lo (hi signed,
    // lo unsigned byte); the relative error per element is at most
    // 2^-15 of the head's max |q|.  B fragment rows 4t..4t+3 (b0) and
    // 16+4t..16+4t+3 (b1) of k-step gi hold head_dim 32*gi + 8*t +
    // {0..3} and {4..7}: the same permutation of head_dim as the
    // K operand's bytes, so the dot products are unchanged.
    // ksc: per-head / per-channel K scales of the segment's (sequence, kv
    // head), folded into Q (q_d * s_d) before the fixed-point digits
    auto build_q = [&](uint32_t sq, const float* ksc) {
        float zsq[NT];
        int csq[NT][NCG];              // sum of the head's Qi (per 32-value group)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = PK ? (g & 3) : hofs + 8 * nt + g;
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
                if constexpr (ST) {
                    if (p.static_ns > 1) {
                        const float4 s0 = *reinterpret_cast<const float4*>(ksc + 32 * gi + 8 * t);
                        const float4 s1 = *reinterpret_cast<const float4*>(ksc + 32 * gi + 8 * t + 4);
                        qf[gi][0] *= s0.x; qf[gi][1] *= s0.y; qf[gi][2] *= s0.z; qf[gi][3] *= s0.w;
                        qf[gi][4] *= s1.x; qf[gi][5] *= s1.y; qf[gi][6] *= s1.z; qf[gi][7] *= s1.w;
                    } else {
                        const float s0 = ksc[0];
#pragma unroll
                        for (int e = 0; e < 8; ++e) qf[gi][e] *= s0;
                    }
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
            const float up = pow2i(sh);                  // |sh| <= 100
            zsq[nt] = pow2i(-sh) * p.scale_log2;
#pragma unroll
            for (int c = 0; c < NCG; ++c) csq[nt][c] = 0;
            if constexpr (F8 != 0) {
                // FP8 keys: Q^T as f16 (the prescaled bf16 values are exact in
                // f16 down to 2^-14 of the head's max): b0 / b1 of k-step 2 gi
                // are head_dim 32 gi + 8 t + {0,1} / {2,3}, of k-step 2 gi + 1
                // {4,5} / {6,7}, matching the K operand's byte pairs
#pragma unroll
                for (int gi = 0; gi < NGRP; ++gi) {
                    qh0[nt][gi] = ptx::pack_f16x2(qf[gi][0] * up, qf[gi][1] * up);
                    qh1[nt][gi] = ptx::pack_f16x2(qf[gi][2] * up, qf[gi][3] * up);
                    ql0[nt][gi] = ptx::pack_f16x2(qf[gi][4] * up, qf[gi][5] * up);
                    ql1[nt][gi] = ptx::pack_f16x2(qf[gi][6] * up, qf[gi][7] * up);
                }
            } else {
#pragma unroll
            for (int gi = 0; gi < NGRP; ++gi) {
                uint32_t qi[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    // PK: column g carries group parity g / 4 only
                    const int v = (PK && (g >> 2) != (gi & 1))
                                      ? 0
                                      : min(max(__float2int_rn(qf[gi][e] * up), -32767), 32767);
                    csq[nt][G32 ? gi : 0] += v;
                    qi[e] = static_cast<uint32_t>(v);
                }
                // byte 1 (hi digit) and byte 0 (lo digit) of four values each
                auto pick4 = [&](int e0, uint32_t sel2) {
                    return ptx::prmt(ptx::prmt(qi[e0], qi[e0 + 1], sel2),
                                     ptx::prmt(qi[e0 + 2], qi[e0 + 3], sel2), 0x5410u);
                };
                qh0[nt][gi] = pick4(0, 0x0051u);
                qh1[nt][gi] = pick4(4, 0x0051u);
                ql0[nt][gi] = pick4(0, 0x0040u);
                ql1[nt][gi] = pick4(4, 0x0040u);
            }
#pragma unroll
            for (int c = 0; c < NCG; ++c) {
                csq[nt][c] += __shfl_xor_sync(0xffffffffu, csq[nt][c], 1);
                csq[nt][c] += __shfl_xor_sync(0xffffffffu, csq[nt][c], 2);
            }
            }
        }
        // per-head factors of the two heads (columns 2t, 2t+1) this thread
        // accumulates: score scale, and the offset term 128 * sum(Qi) of
        // sum Qi * (byte - 128) = sum Qi * byte - 128 * sum Qi
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                zs[nt][c] = __shfl_sync(0xffffffffu, zsq[nt], 4 * (2 * t + c));
#pragma unroll
                for (int k = 0; k < NCG; ++k)
                    qc[nt][c][k] = 128 * __shfl_sync(0xffffffffu, csq[nt][k], 4 * (2 * t + c));
            }
    };

    // ---- in-kernel combine (flash-decoding): fold a split unit's partial
    // states, slots j < ns of rows bh0 .. bh0 + G - 1 (a slot whose m is -inf
    // holds none), into its output rows:
    //   M = max_j m_j,  w_j = 2^(m_j - M),  out = sum_j w_j o_j / sum_j w_j l_j.
    // tpi adjacent threads share the slots of one (row, 16-byte chunk), each
    // folding batches of eight slots per round of L2 loads, then merge their
    // states by shuffles.
    // ---- fused append (decode, INT8 per token / group-32): patch_new_token

#pragma unroll 1
    for (int i = ibeg; i < iend;) {
        const int Lone = one ? one_valid(one_raw()) : 0;
        const Seg sg = one ? one_seg(Lone) : seg_at(i, iend, lens, nsv, cum, B, p.chunk);
        i = sg.next;
        const int b = sg.b, hk = sg.hk;
        const int64_t bh0 = static_cast<int64_t>(b) * p.Hq + hk * G;   // first q head of the group
        // chunk of queries: the last position column 8 nt + 2 t + c may see;
        // sliding window: the first (both counted from the window base)
        int lim_col[NT][2], lo_col[NT][2];
        if constexpr (CAUSAL) {
            const int Lseq = one ? Lone : lens[b];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    lim_col[nt][c] = Lseq - p.qlen + (hofs + 8 * nt + 2 * t + c) % p.qlen;
                    lo_col[nt][c] = p.window > 0 ? lim_col[nt][c] - p.window + 1 : INT_MIN;
                }
        }
        if (!one && sg.ns == 0) {
            // empty (or rejected) sequence: zero rows
#pragma unroll 1
            for (int idx = ctid; idx < G * D; idx += NCONS) p.out[bh0 * D + idx] = 0.f;
            continue;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
                o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
        }
        kv = 64;
        bool have_q = false;            // Q fragments of this segment are built
        const float* ksc = ST ? p.k_scale + (static_cast<int64_t>(b) * p.Hk + hk) * p.static_ns
                              : nullptr;
        if (one) {                      // the query rows came ahead of stage 0
            wait(bar_q, 0);
            build_q(sbase + Lay::Q_OFF, ksc);
            have_q = true;
        }
        // contiguous layout: the stage's scales start sc_off bytes in (the copies
        // start at the 16-byte aligned float at or below the tile's first; tiles
        // start at multiples of 16 tokens, so the offset is the segment's)
        const uint32_t sc_off =
            PAGED ? 0u
                  : ((static_cast<uint32_t>(b * p.Hk + hk) * static_cast<uint32_t>(p.max_seq) *
                      static_cast<uint32_t>(NG)) & 3u) * 4u;
        const int t0 = sg.t0, t1 = sg.t1;
        // one item per CTA: at least the one stage the producer issued before
        // it knew the length
        const int ntiles = max(one ? 1 : 0, (t1 - t0 + TT - 1) / TT);
        // fused append: the new token (position L - 1, fa_tok) lies in one
        // stage of this segment, in the slice of one warp of the group that
        // takes that stage; that warp quantises it there (-1: not this warp)
        int fa_tok = -1;
        if constexpr (FUSED) {
            if (p.k_new != nullptr) {
                const int tok = (one ? Lone : lens[b]) - 1;
                if (tok >= t0 && tok < t1) {
                    const int itn = (tok - t0) / TT;
                    if ((G16 || ((c_count + itn) & 1) == grp) && ((tok - t0 - itn * TT) >> 5) == wg)
                        fa_tok = tok;
                }
            }
        }
#pragma unroll 1
        for (int it = 0; it < ntiles; ++it, ++c_count) {
            if (!G16 && (c_count & 1) != grp) continue;   // the other group's stage
            const int s = c_count % NST;
            wait(bar_full + 8 * s, (c_count / NST) & 1);
            const int tt0 = t0 + it * TT;
            const uint32_t sk = sbase + s * Lay::STAGE;
            const uint32_t sv = sk + Lay::KV_BYTES;
            const uint32_t sks = sv + Lay::KV_BYTES + sc_off;
            const uint32_t svs = sv + Lay::KV_BYTES + Lay::SC_FLOATS * 4 + sc_off;
            if (!have_q) {
                have_q = true;
                build_q(sk + Lay::Q_OFF, ksc);
            }
            const int tok0 = tt0 + 32 * wg;               // first token of this warp's slice
            if (tok0 < t1) {
                // stage rows of MMA tile u: K rows g, g + 8; V rows of k 2t, 2t+1, 2t+8, 2t+9
                int rA[2], rB[2], V0[2], V1[2];
                bool okA[2], okB[2];
                const uint32_t pmask = PAGED ? lds32(sk + Lay::MASK_OFF) : 0u;
                if constexpr (FUSED) {
                    // (paged: only into a page that was loaded; a missing one
                    // was flagged by the producer and its tokens are masked)
                    if (fa_tok >= tt0 && fa_tok < tt0 + TT &&
                        (!PAGED || ((pmask >> ((fa_tok - tt0) >> 4)) & 1u)))
                        patch_new_token<D, G32, PAGED>(p, sk, sv, sks, svs, fa_tok - tt0, fa_tok,
                                                       b, hk, !G16 || grp == 0);
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int base = 32 * wg + 16 * u;
                    rA[u] = base + sig_g;
                    rB[u] = rA[u] + 8;
                    V0[u] = base + sig_a;
                    V1[u] = base + sig_b;
                    const int tk = tok0 + 16 * u;
                    bool page_ok = tk < t1;
                    // paged: page 2 wg + u of the stage was loaded (the producer
                    // checked the table entry)
                    if (PAGED) page_ok = page_ok && ((pmask >> (2 * wg + u)) & 1u);
                    okA[u] = page_ok && (tk + sig_g < t1);
                    okB[u] = page_ok && (tk + 8 + sig_g < t1);
                }

                // ---- S^T = K . Q^T per MMA tile on the integer MMA: the K bytes
                // are the A operand as loaded (rows tokens rA, rB; 8 bytes at
                // 32*gi + 8*t are k = 4t..4t+3 and 16+4t..16+4t+3), times the two
                // Q digits; S = 256 * S_hi + S_lo - 128 * sum(Qi) is exact in s32.
                // ---- scores z (log2 domain): [u][nt][0..1] token rA[u], [u][nt][2..3] token rB[u]
                float z[2][NT][4];
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        z[u][nt][0] = z[u][nt][1] = z[u][nt][2] = z[u][nt][3] = 0.f;
                int ah[2][NT][4], al[2][NT][4];
                // accumulators of fold kg (a head_dim group; PK: a group pair,
                // whose lo digit starts at the pair's offset term -128 * sum(Qi))
                auto zero_acc = [&](int kg) {
#pragma unroll
                    for (int u = 0; u < 2; ++u)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                ah[u][nt][e] = 0;
                                al[u][nt][e] =
                                    PK ? -(qc[nt][e & 1][2 * kg] + qc[nt][e & 1][2 * kg + 1]) : 0;
                            }
                };
                // fold the integer scores of fold kg into z, times the K scale of
                // the token and of the column's group (per token: kg = 0, once
                // after all groups; PK: group 2 kg + par)
                auto fold = [&](int kg) {
                    const int cg = PK ? 2 * kg + par : kg;
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float ksa = ST ? 1.f : ldsf(sks + (rA[u] * NG + cg) * 4);
                        const float ksb = ST ? 1.f : ldsf(sks + (rB[u] * NG + cg) * 4);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int S = ah[u][nt][e] * 256 + al[u][nt][e] -
                                              (PK ? 0 : qc[nt][e & 1][kg]);
                                z[u][nt][e] = fmaf(static_cast<float>(S), e < 2 ? ksa : ksb, z[u][nt][e]);
                            }
                    }
                };
                if constexpr (F8 != 0) {
                    // FP8 keys: byte pairs to exact f16, two m16n8k16 k-steps per
                    // 32 head_dim values (A rows: tokens rA, rB; k as in build_q)
#pragma unroll
                    for (int gi = 0; gi < NGRP; ++gi)
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const uint2 wa = lds64(sk + swz<D>(rA[u], 32 * gi + 8 * t));
                            const uint2 wb = lds64(sk + swz<D>(rB[u], 32 * gi + 8 * t));
                            const uint32_t a0 = fp8x2_to_f16x2<F8>(wa.x, 0);
                            const uint32_t a1 = fp8x2_to_f16x2<F8>(wb.x, 0);
                            const uint32_t a2 = fp8x2_to_f16x2<F8>(wa.x, 1);
                            const uint32_t a3 = fp8x2_to_f16x2<F8>(wb.x, 1);
                            const uint32_t c0 = fp8x2_to_f16x2<F8>(wa.y, 0);
                            const uint32_t c1 = fp8x2_to_f16x2<F8>(wb.y, 0);
                            const uint32_t c2 = fp8x2_to_f16x2<F8>(wa.y, 1);
                            const uint32_t c3 = fp8x2_to_f16x2<F8>(wb.y, 1);
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                ptx::mma_f16(z[u][nt], a0, a1, a2, a3, qh0[nt][gi], qh1[nt][gi]);
                                ptx::mma_f16(z[u][nt], c0, c1, c2, c3, ql0[nt][gi], ql1[nt][gi]);
                            }
                        }
                } else {
                zero_acc(0);
#pragma unroll
                for (int gi = 0; gi < NGRP; ++gi) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint2 wa = lds64(sk + swz<D>(rA[u], 32 * gi + 8 * t));
                        const uint2 wb = lds64(sk + swz<D>(rB[u], 32 * gi + 8 * t));
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            ptx::mma_u8<true>(ah[u][nt], wa.x, wb.x, wa.y, wb.y, qh0[nt][gi],
                                              qh1[nt][gi]);
                            ptx::mma_u8<false>(al[u][nt], wa.x, wb.x, wa.y, wb.y, ql0[nt][gi],
                                               ql1[nt][gi]);
                        }
                    }
                    if constexpr (G32) {
                        if (!PK || (gi & 1)) {
                            const int kg = PK ? gi >> 1 : gi;
                            fold(kg);
                            if (gi + 1 < NGRP) zero_acc(kg + 1);
                        }
                    }
                }
                if constexpr (!G32) fold(0);
                }
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if constexpr (PK) {
                            // this parity's groups, then the other parity's (lane t ^ 2)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float zz = z[u][nt][e] * zs[nt][e & 1];
                                z[u][nt][e] = zz + __shfl_xor_sync(0xffffffffu, zz, 2);
                            }
                            z[u][nt][0] = okA[u] ? z[u][nt][0] : -INFINITY;
                            z[u][nt][1] = okA[u] ? z[u][nt][1] : -INFINITY;
                            z[u][nt][2] = okB[u] ? z[u][nt][2] : -INFINITY;
                            z[u][nt][3] = okB[u] ? z[u][nt][3] : -INFINITY;
                        } else {
                            z[u][nt][0] = okA[u] ? z[u][nt][0] * zs[nt][0] : -INFINITY;
                            z[u][nt][1] = okA[u] ? z[u][nt][1] * zs[nt][1] : -INFINITY;
                            z[u][nt][2] = okB[u] ? z[u][nt][2] * zs[nt][0] : -INFINITY;
                            z[u][nt][3] = okB[u] ? z[u][nt][3] * zs[nt][1] : -INFINITY;
                        }
                        if constexpr (CAUSAL) {
                            // positions past the column's query, or older than its
                            // sliding window, are masked
                            const int ta = tt0 + rA[u], tb = tt0 + rB[u];
                            if (ta > lim_col[nt][0] || ta < lo_col[nt][0]) z[u][nt][0] = -INFINITY;
                            if (ta > lim_col[nt][1] || ta < lo_col[nt][1]) z[u][nt][1] = -INFINITY;
                            if (tb > lim_col[nt][0] || tb < lo_col[nt][0]) z[u][nt][2] = -INFINITY;
                            if (tb > lim_col[nt][1] || tb < lo_col[nt][1]) z[u][nt][3] = -INFINITY;
                        }
                    }
                // ---- online softmax per head: max over the slice's 32 tokens
                float pr[2][NT][4];
                float f[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        float mx = fmaxf(fmaxf(z[0][nt][c], z[0][nt][2 + c]),
                                         fmaxf(z[1][nt][c], z[1][nt][2 + c]));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                        const float mn = fmaxf(m[nt][c], mx);
                        const float al = (mn == -INFINITY) ? 1.f : ptx::ex2(m[nt][c] - mn);
                        float add = 0.f;
                        // (a chunk query, or a windowed one, can have seen no
                        // position yet: its masked scores then give 2^-inf = 0,
                        // not NaN)
                        const float mb = (CAUSAL && mn == -INFINITY) ? 0.f : mn;
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            pr[u][nt][c] = okA[u] ? ptx::ex2(z[u][nt][c] - mb) : 0.f;
                            pr[u][nt][2 + c] = okB[u] ? ptx::ex2(z[u][nt][2 + c] - mb) : 0.f;
                            add += pr[u][nt][c] + pr[u][nt][2 + c];
                        }
                        l[nt][c] = l[nt][c] * al + add;
                        m[nt][c] = mn;
                        f[nt][c] = al;
                    }
                // ---- V scales of the thread's four tokens and the running prescale 2^kv
                // (PK: set gv is group pair gv, this thread's column group 2 gv + par)
                float vsa[2][NVS], vsb[2][NVS];
                float vmax = 0.f;
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int gv = 0; gv < NVS; ++gv) {
                        const int cg = PK ? 2 * gv + par : gv;
                        vsa[u][gv] = okA[u] ? (NOSC ? 1.f : ldsf(svs + (rA[u] * NG + cg) * 4)) : 0.f;
                        vsb[u][gv] = okB[u] ? (NOSC ? 1.f : ldsf(svs + (rB[u] * NG + cg) * 4)) : 0.f;
                        vmax = fmaxf(vmax, fmaxf(vsa[u][gv], vsb[u][gv]));
                    }
                if constexpr (PK) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 2));
                vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 4));
                vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 8));
                vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 16));
                if (vmax > 0.f) {
                    const int ev = static_cast<int>((__float_as_uint(vmax) >> 23) & 0xffu) - 127;
                    const int kn = max(min(kv, 14 - ev), -120);   // kv stays in [-120, 64]
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
                const float up = pow2i(kv);
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
                // ---- O^T += V^T . P^T, one k-step of 16 tokens per MMA tile u.  P^T
                // operand: P'' hi / lo transposed from the score layout (row = token,
                // column = head) into B fragments (k = token, n = head).  V^T A
                // fragment of m-tile mt: rows g, g+8 are head_dim d(mt, g),
                // d(mt, g) + 1; columns 2t, 2t+1 / 2t+8, 2t+9 are the V rows
                // V0, V1 / V0 + 8, V1 + 8.  Byte pairs of two rows are interleaved
                // with prmt and turned into exact (v - 128) f16 pairs.
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    uint32_t pbh[NVS][NT][2], pbl[NVS][NT][2];
#pragma unroll
                    for (int gv = 0; gv < NVS; ++gv)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            uint32_t ha, la, hb, lb;
                            split_f16x2(pr[u][nt][0] * vsa[u][gv] * up,
                                        pr[u][nt][1] * vsa[u][gv] * up, ha, la);
                            split_f16x2(pr[u][nt][2] * vsb[u][gv] * up,
                                        pr[u][nt][3] * vsb[u][gv] * up, hb, lb);
                            pbh[gv][nt][0] = transpose8x8(ha);
                            pbl[gv][nt][0] = transpose8x8(la);
                            pbh[gv][nt][1] = transpose8x8(hb);
                            pbl[gv][nt][1] = transpose8x8(lb);
                        }
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
                            uint32_t a0, a1, a2, a3;
                            if constexpr (F8 != 0) {     // FP8 values, exact in f16
                                a0 = fp8x2_to_f16x2<F8>(x01, 0);
                                a1 = fp8x2_to_f16x2<F8>(x01, 1);
                                a2 = fp8x2_to_f16x2<F8>(x23, 0);
                                a3 = fp8x2_to_f16x2<F8>(x23, 1);
                            } else {                     // offset-128 bytes as exact integers
                                a0 = ptx::bytes_to_f16x2(x01, 0x4140u);
                                a1 = ptx::bytes_to_f16x2(x01, 0x4342u);
                                a2 = ptx::bytes_to_f16x2(x23, 0x4140u);
                                a3 = ptx::bytes_to_f16x2(x23, 0x4342u);
                            }
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                ptx::mma_f16(o[mt0 + hh][nt], a0, a1, a2, a3, pbh[gv][nt][0],
                                             pbh[gv][nt][1]);
                                ptx::mma_f16(o[mt0 + hh][nt], a0, a1, a2, a3, pbl[gv][nt][0],
                                             pbl[gv][nt][1]);
                            }
                        }
                    };
                    const int R0 = V0[u], R1 = V1[u], R2 = V0[u] + 8, R3 = V1[u] + 8;
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
                            pv_words(2 * gv, PK ? gv >> 1 : gv, lds32(sv + swz<D>(R0, cb)),
                                     lds32(sv + swz<D>(R1, cb)), lds32(sv + swz<D>(R2, cb)),
                                     lds32(sv + swz<D>(R3, cb)));
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_empty + 8 * s);
        }

        // ---- merge the eight warps' states of the segment (one barrier); a
        // segment that is the whole (b, kv head) writes the final rows
        // (one item per CTA: the final rows of a one-chunk or empty sequence come
        // from its chunk 0; chunks past the length write nothing)
        // (mixed cache: partials only, the window kernel writes the rows)
        const bool final_rows =
            !p.recent && (one ? sg.j0 == 0 && sg.ns <= 1 : sg.j0 == 0 && sg.j1 == sg.ns - 1);
        const bool part_rows = p.recent ? (one ? sg.j0 < sg.ns : true)
                                        : (one ? sg.ns > 1 && sg.j0 < sg.ns : !final_rows);
        const int seg_j0 = sg.j0;
        // the previous segment's readers are done with the maxima and the slots
        if (merges > 0) wait(bar_mfree, (merges - 1) & 1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 4);
                l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 8);
                l[nt][c] += __shfl_xor_sync(0xffffffffu, l[nt][c], 16);
                if (g == 0) {
                    const int hm = PK ? 2 * (t & 1) + c : hofs + 8 * nt + 2 * t + c;
                    mrg_m[hm * NW + cw] = m[nt][c];
                    mrg_l[hm * NW + cw] = l[nt][c];
                }
            }
        // this warp's o, prescale 2^kv undone, into its slot: one row of D
        // floats per head, stored as 16-byte chunks, chunk k of head h at
        // k ^ mswz(h).  A thread holds four consecutive head_dim values of a
        // head in o[2a][nt][c], o[2a][nt][c+2], o[2a+1][nt][c], o[2a+1][nt][c+2]
        // (one chunk), and the swizzle puts the eight chunks of a quarter warp
        // in eight different bank quads.
        {
            const float down = pow2i(-kv);
            float* slot = mslot + cw * NV * 32;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int h = PK ? 2 * (t & 1) + c : 8 * nt + 2 * t + c;
#pragma unroll
                    for (int a = 0; a < D / 32; ++a) {
                        if (PK && (a & 1) != par) continue;   // the other parity's group
                        const int k = G32 ? 8 * a + g : (D / 32) * g + a;
                        *reinterpret_cast<float4*>(slot + h * D + 4 * (k ^ mswz<D, G32>(h))) =
                            make_float4(o[2 * a][nt][c] * down, o[2 * a][nt][c + 2] * down,
                                        o[2 * a + 1][nt][c] * down, o[2 * a + 1][nt][c + 2] * down);
                    }
                }
        }
        ptx::named_bar_sync(1, NCONS);
        // one thread per (head, 16-byte chunk of its row): the head's segment
        // max M and sum Ls over the warps that hold the head (all eight; G16:
        // the four of its group), the weights 2^(m_w - M) (over Ls when the
        // rows are final), and the weighted sum of their slots
        constexpr int NCH = D / 4;
        constexpr int NWH = G16 ? WPG : NW;           // warps holding one head
        constexpr int NITEM = (G16 ? 16 : 8) * NCH;
        static_assert(NW == 8 && NWH % 4 == 0, "16-byte loads of per-warp maxima and sums");
#pragma unroll
        for (int it = 0; it < (NITEM + NCONS - 1) / NCONS; ++it) {
            const int idx = ctid + it * NCONS;
            const int h = idx / NCH, k = idx % NCH;
            if (idx >= NITEM || h >= G) continue;
            const int wb = G16 ? WPG * (h >> 3) : 0;   // the head's first warp
            const int hl = G16 ? (h & 7) : h;           // its row in a warp's slot
            float mw[NWH], fw[NWH], lw[NWH];
#pragma unroll
            for (int x = 0; x < NWH / 4; ++x) {
                *reinterpret_cast<float4*>(mw + 4 * x) =
                    *reinterpret_cast<const float4*>(mrg_m + h * NW + wb + 4 * x);
                *reinterpret_cast<float4*>(lw + 4 * x) =
                    *reinterpret_cast<const float4*>(mrg_l + h * NW + wb + 4 * x);
            }
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NWH; ++w) M = fmaxf(M, mw[w]);
            float Ls = 0.f;
#pragma unroll
            for (int w = 0; w < NWH; ++w) {
                fw[w] = mw[w] == -INFINITY ? 0.f : ptx::ex2(mw[w] - M);
                Ls += lw[w] * fw[w];
            }
            if (final_rows) {
                const float r = Ls > 0.f ? __frcp_rn(Ls) : 0.f;
#pragma unroll
                for (int w = 0; w < NWH; ++w) fw[w] *= r;
            }
            float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
            const float* src = mslot + hl * D + 4 * (k ^ mswz<D, G32>(hl)) + wb * NV * 32;
#pragma unroll
            for (int w = 0; w < NWH; ++w) {
                const float4 v = *reinterpret_cast<const float4*>(src + w * NV * 32);
                s0 = fmaf(fw[w], v.x, s0);
                s1 = fmaf(fw[w], v.y, s1);
                s2 = fmaf(fw[w], v.z, s2);
                s3 = fmaf(fw[w], v.w, s3);
            }
            if constexpr (ST) {         // per-head / per-channel V scales on the output
                const float* vsc = p.v_scale + (static_cast<int64_t>(b) * p.Hk + hk) * p.static_ns;
                if (p.static_ns > 1) {
                    const float4 w4 = *reinterpret_cast<const float4*>(vsc + 4 * k);
                    s0 *= w4.x; s1 *= w4.y; s2 *= w4.z; s3 *= w4.w;
                } else {
                    const float w1 = vsc[0];
                    s0 *= w1; s1 *= w1; s2 *= w1; s3 *= w1;
                }
            }
            const int64_t row = bh0 + h;
            if (final_rows) {
                *reinterpret_cast<float4*>(p.out + row * D + 4 * k) = make_float4(s0, s1, s2, s3);
            } else if (part_rows) {
                // the partial, with its (m, l) in the slot of the segment's first chunk
                *reinterpret_cast<float4*>(p.ws_o + (row * p.splits + seg_j0) * D + 4 * k) =
                    make_float4(s0, s1, s2, s3);
                if (k == 0) {
                    p.ws_m[row * p.splits + seg_j0] = M;
                    p.ws_l[row * p.splits + seg_j0] = Ls;
                }
            }
            // blocks of several items: every other chunk slot the segment covers
            // gets m = -inf ("no partial here"), so the combine kernel finds a
            // unit's partials from its m slots alone (one item per CTA: every
            // chunk below the chunk count holds a partial)
            if (!one && p.splits > 1 && sg.ns > 1) {
#pragma unroll 1
                for (int j = seg_j0 + (part_rows ? 1 : 0) + k; j <= sg.j1; j += NCH)
                    p.ws_m[row * p.splits + j] = -INFINITY;
            }
        }
        // this warp has read the maxima and the slots
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_mfree);
        ++merges;
    }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn query_encode_fn() {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<EncodeFn>(ptr);
    return nullptr;
}

// The driver's tensor-map encoder, looked up once per process (a
// function-local static is initialised exactly once even when several host
// threads get here together; the entry point is the same for every device).
EncodeFn encode_fn() {
    static const EncodeFn fn = query_encode_fn();
    return fn;
}

// The inputs a tensor map is encoded from (everything else is fixed).
struct MapKey {
    uintptr_t base;
    int64_t rows;
    int D, box_rows;
    bool operator==(const MapKey& o) const {
        return base == o.base && rows == o.rows && D == o.D && box_rows == o.box_rows;
    }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        uint64_t h = k.base * 0x9E3779B97F4A7C15ull;
        h ^= static_cast<uint64_t>(k.rows) + 0x7F4A7C15ull + (h << 6) + (h >> 2);
        h ^= static_cast<uint64_t>(k.D * 1031 + k.box_rows) + (h << 6) + (h >> 2);
        return static_cast<size_t>(h);
    }
};

// 2-D u8 tensor map over `rows` rows of D bytes, box of box_rows rows.  The
// encoded maps are kept per host thread, keyed by every input of the
// encoding, so a cached map is the one the encoder would produce again.
cudaError_t make_map(CUtensorMap* map, const void* base, int D, int64_t rows, int box_rows) {
    thread_local std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
    const MapKey key{reinterpret_cast<uintptr_t>(base), rows, D, box_rows};
    const auto it = cache.find(key);
    if (it != cache.end()) {
        *map = it->second;
        return cudaSuccess;
    }
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
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    if (cache.size() >= 4096) cache.clear();
    cache.emplace(key, *map);
    return cudaSuccess;
}

// Function attributes belong to the current device's context, so they are
// set once per device ordinal.
template <int D, bool G32, bool PAGED, bool G16, bool PK, int VAR, int F8, bool ST>
cudaError_t set_attrs() {
    using Lay = Layout<D, G32, G16>;
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    return once_per_device(done, dev, cudaSuccess, [] {
        auto kern = decode_split_tc<D, G32, PAGED, G16, PK, VAR, F8, ST>;
        cudaError_t r =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     cudaSharedmemCarveoutMaxShared);
        return r;
    });
}

template <int D, bool G32, bool PAGED, bool G16, bool PK, int VAR, int F8 = 0, bool ST = false>
cudaError_t launch_tc(const DecodeParams& p, cudaStream_t s) {
    using Lay = Layout<D, G32, G16>;
    cudaError_t e = set_attrs<D, G32, PAGED, G16, PK, VAR, F8, ST>();
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
    cfg.blockDim = dim3(nthreads(PAGED), 1, 1);
    cfg.dynamicSmemBytes = Lay::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_split_tc<D, G32, PAGED, G16, PK, VAR, F8, ST>, mk, mv,
                              p);
}

template <int D, bool G32, bool PAGED>
cudaError_t pick_g(const DecodeParams& p, cudaStream_t s) {
    // a chunk of queries (causal columns) or a sliding window: the masked
    // instantiation (for one decode query the causal mask keeps every position)
    if (p.qlen > 1 || p.window > 0)
        return p.G > 8 ? launch_tc<D, G32, PAGED, true, false, 1>(p, s)
                       : launch_tc<D, G32, PAGED, false, false, 1>(p, s);
    // the step's new token quantised inside the kernel (kvq_append_decode):
    // its own instantiation, so the plain decode code carries none of it
    if (p.k_new != nullptr) {
        if (p.G > 8) return launch_tc<D, G32, PAGED, true, false, 2>(p, s);
        if constexpr (G32)
            if (p.G <= 4) return launch_tc<D, G32, PAGED, false, true, 2>(p, s);
        return launch_tc<D, G32, PAGED, false, false, 2>(p, s);
    }
    if (p.G > 8) return launch_tc<D, G32, PAGED, true, false, 0>(p, s);
    if constexpr (G32)
        if (p.G <= 4) return launch_tc<D, G32, PAGED, false, true, 0>(p, s);
    return launch_tc<D, G32, PAGED, false, false, 0>(p, s);
}

// FP8 caches (no scales): E4M3 (F8 = 1) or E5M2 (F8 = 2)
template <int D, bool PAGED, int F8>
cudaError_t pick_g_fp8(const DecodeParams& p, cudaStream_t s) {
    const bool masked = p.qlen > 1 || p.window > 0;
    if (p.G > 8)
        return masked ? launch_tc<D, false, PAGED, true, false, 1, F8>(p, s)
                      : launch_tc<D, false, PAGED, true, false, 0, F8>(p, s);
    return masked ? launch_tc<D, false, PAGED, false, false, 1, F8>(p, s)
                  : launch_tc<D, false, PAGED, false, false, 0, F8>(p, s);
}

// per-head / per-channel scales (one set per (sequence, kv head))
template <int D, bool PAGED>
cudaError_t pick_g_static(const DecodeParams& p, cudaStream_t s) {
    const bool masked = p.qlen > 1 || p.window > 0;
    if (p.G > 8)
        return masked ? launch_tc<D, false, PAGED, true, false, 1, 0, true>(p, s)
                      : launch_tc<D, false, PAGED, true, false, 0, 0, true>(p, s);
    return masked ? launch_tc<D, false, PAGED, false, false, 1, 0, true>(p, s)
                  : launch_tc<D, false, PAGED, false, false, 0, 0, true>(p, s);
}

template <int D, bool PAGED>
cudaError_t pick_fmt(const DecodeParams& p, cudaStream_t s) {
    if (p.static_ns) return pick_g_static<D, PAGED>(p, s);
    if (p.fp8 == 1) return pick_g_fp8<D, PAGED, 1>(p, s);
    if (p.fp8 == 2) return pick_g_fp8<D, PAGED, 2>(p, s);
    return p.group32 ? pick_g<D, true, PAGED>(p, s) : pick_g<D, false, PAGED>(p, s);
}

template <int D>
cudaError_t pick_layout(const DecodeParams& p, cudaStream_t s) {
    return p.page_size ? pick_fmt<D, true>(p, s) : pick_fmt<D, false>(p, s);
}

}  // namespace

cudaError_t make_tile_map(CUtensorMap* map, const void* base, int D, int64_t rows, int box_rows) {
    return make_map(map, base, D, rows, box_rows);
}

cudaError_t launch_decode_split_tc(const DecodeParams& p, cudaStream_t s) {
    if (p.grid < 1) return cudaErrorInvalidValue;
    if (p.D == 128) return pick_layout<128>(p, s);
    if (p.D == 64) return pick_layout<64>(p, s);
    return cudaErrorInvalidValue;
}

}  // namespace kvq

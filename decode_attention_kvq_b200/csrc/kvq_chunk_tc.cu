// kvq_chunk_tc.cu -- attention of a dense chunk of queries on the INT8 cache
// (chunked prefill: many (query, head) rows per kv head) on the tcgen05
// tensor cores, accumulators in tensor memory.
//
// Method (what is computed): abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs,
// CudaQuantizedKvCache::forward_attention with q_len > 1 -- the chunk's
// queries sit at positions L - T + i and see the keys up to their own
// position, K and V dequantised on the fly ((byte - 128) * scale); combs-
// models 0.2.2, src/kv.rs, attend (scale after the dot product, GQA: query
// head h reads kv head h / G).
//
// How (sm_100a):
//  * CTA = one kv head of one sequence and 128 (query, head) rows, row
//    r = i * G + h (query i, head h of the group), so the rows share K and V
//    and their causal limits lie within 128 / G positions.  It walks the KV
//    positions up to its last row's limit in tiles of 128 tokens.
//  * Warp 8 (one lane) streams K and V tiles (TMA 2-D, 128-byte swizzle) and
//    their fp32 scales (bulk copies) through a two-stage ring.
//  * Warp 9 (one lane) issues the tensor-core work: S = Q K^T on tcgen05
//    kind::i8 -- Q as a per-row power-of-two prescaled 16-bit integer in two
//    byte digits (signed hi, unsigned lo), the K bytes as loaded, so
//    S = 256 S_hi + S_lo - 128 sum(Qi) is exact in int32 -- into two 128-
//    column TMEM accumulators; then P V on kind::f16 into a third (fp32, a
//    fresh one per tile), with P'' = 2^(z - m) * v_scale * 2^kv split into f16
//    hi + lo parts and V as the exact f16 integers byte - 128.  The next
//    tile's Q K^T is issued as soon as the rows hold this tile's scores in
//    registers, ahead of this tile's P V.
//  * Warps 0-7 own the rows, two warps per row: warp w reads TMEM lanes
//    32 (w % 4) .. + 31 (row i = TMEM lane i) and takes half h = w / 4 of the
//    row's 128 columns -- tokens 64 h .. 64 h + 63 of a tile and head_dim
//    64 h .. 64 h + 63 of the output -- so two row warps share each
//    scheduler.  They read the scores with tcgen05.ld into registers, apply
//    the K scale, the row's prescale, attn_scale and log2(e), mask causally,
//    exchange the halves' maxima through shared memory, keep the online
//    softmax per row, fold the P V of tiles into a running sum in TMEM (fp32,
//    with the row's rescale), write P'' into shared memory in the canonical
//    swizzled layout, and finally read the sum back and write the row.
//  * Warps 10 and 11 help ahead of the rows: per tile, warp 10 copies the K
//    scales and the V scales times the P'' prescale into aligned shared-
//    memory vectors (with the prescale's drop), and both write the tile's V
//    as exact f16 into the MN-major B tile once the previous P V has read
//    it.
//  * Every mbarrier wait is bounded; a timeout sets KVQ_DEVERR_TIMEOUT, every
//    role then skips its remaining work (the row warps still pass every
//    named barrier of every tile, so none waits for another that left), and
//    the CTA frees its tensor memory.
#include <cuda.h>
#include <math.h>

#include <atomic>

#include "kvq_devonce.h"
#include "kvq_internal.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

constexpr int kRows = 128;                 // (query, head) rows per CTA: the MMA M
constexpr int kTok = 128;                  // KV tokens per tile
constexpr int kDim = 128;                  // head_dim handled here
constexpr int kThreads = 384;              // warps 0-7 rows, 8 producer, 9 MMA, 10-11 helpers
constexpr int kRowThreads = 256;
constexpr int kProdWarp = 8, kMmaWarp = 9, kAuxWarp = 10;   // helpers: warps 10 and 11
constexpr int kTmemCols = 512;             // S_hi 128 | S_lo 128 | O tile 128 | O run 128
// The tensor cores add each P.V k-step into O; over a long key range that is
// tens of thousands of accumulations into one fp32 accumulator, and the error
// they leave grows with the count.  Each tile's P.V therefore starts a fresh
// accumulator (O tile: 16 k-steps), which the row threads fold into the
// running sum (O run) in fp32 with the tile's rescale.
constexpr uint32_t kColShi = 0, kColSlo = 128, kColO = 256, kColRun = 384;

// shared memory (offsets from a 1024-byte aligned base)
constexpr int kQhi = 0;                    // Q hi digits [128 rows][128 B], K-major SW128
constexpr int kQlo = 16384;
constexpr int kStage0 = 32768;             // stage s: K [128][128 B], V, K scales, V scales
constexpr int kStageBytes = 34816;
constexpr int kStK = 0, kStV = 16384, kStKs = 32768, kStVs = 33792;
constexpr int kV16 = kStage0 + 2 * kStageBytes;   // V as f16 [2 atoms][128 tok][128 B], MN-major
constexpr int kPhi = kV16 + 32768;                // P'' hi [2 atoms][128 rows][128 B], K-major
constexpr int kPlo = kPhi + 32768;
constexpr int kMisc = kPlo + 32768;               // barriers, tensor-memory address, flags
// row-warp vectors: K scales [2][128], V scales x 2^kv [2][128] (by tile
// parity), the halves' maxima [2][128] and a spare pair [2][128]
constexpr int kAux = kMisc + 256;
constexpr int kSmem = kAux + 4096 + 1024;         // + base alignment slack

struct ChunkParams {
    const uint16_t* q;        // [B, Hq, T, D] bf16
    const float* k_scale;     // [B, Hk, max_seq, 1]
    const float* v_scale;
    const int32_t* seq_lens;  // [B], the chunk's T tokens included
    float* out;               // [B, Hq, T, D]
    int32_t* d_err;
    int B, Hq, Hk, G, T, max_seq;
    int tiles_per_head;       // ceil(G * T / 128)
    float scale_log2;
};

// ---- tcgen05 wrappers -------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// one MMA: D[tmem] (+)= A[desc] * B[desc]
template <bool I8>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
    const uint32_t z = 0;
    if constexpr (I8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(z), "r"(z), "r"(z), "r"(z)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
            ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(z), "r"(z), "r"(z), "r"(z)
            : "memory");
    }
}
// 32 consecutive 32-bit columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(addr)
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};"
        ::"r"(addr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
          "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]),
          "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
          "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
// 16 consecutive 32-bit columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(addr)
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};"
        ::"r"(addr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
          "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm100 version field.
// lbo / sbo in bytes: K-major -- sbo = stride of 8-row groups (lbo unused);
// MN-major -- lbo = stride of 128-byte atoms along M/N, sbo = stride of
// 8-row groups along K.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((addr & 0x3ffffu) >> 4) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptors (M = 128, N = 128): c format (bits 4-5), a / b
// formats (7-9, 10-12), b major (16), N >> 3 (17-22), M >> 4 (24-28).
constexpr uint32_t kIdescShape = (16u << 17) | (8u << 24);
constexpr uint32_t kIdescQkHi = (2u << 4) | (1u << 7) | (0u << 10) | kIdescShape;   // s32 = s8 * u8
constexpr uint32_t kIdescQkLo = (2u << 4) | (0u << 7) | (0u << 10) | kIdescShape;   // s32 = u8 * u8
constexpr uint32_t kIdescPv = (1u << 4) | (1u << 16) | kIdescShape;   // f32 = f16 * f16, B MN-major

__device__ __forceinline__ float pow2i_f(int e) { return __int_as_float((e + 127) << 23); }

__global__ void __launch_bounds__(kThreads, 1)
chunk_attn_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const __grid_constant__ ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sb = ptx::smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const uint32_t bar_full = sb + kMisc;            // [2]
    const uint32_t bar_empty = bar_full + 16;        // [2]
    const uint32_t bar_sfull = bar_full + 32;
    const uint32_t bar_sfree = bar_full + 40;
    const uint32_t bar_pfull = bar_full + 48;
    const uint32_t bar_odone = bar_full + 56;
    const uint32_t bar_qready = bar_full + 64;
    const uint32_t bar_aready = bar_full + 72;       // [2] by tile parity: the tile's vectors
    const uint32_t bar_afree = bar_full + 88;        // [2] by tile parity: rows done with them
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kMisc + 104);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMisc + 108);
    // [8] per-warp "a row's maximum grew this tile"; [2] by tile parity: P.V of
    // the tile adds onto the O tile (1) or starts it afresh (0); [2] by tile
    // parity: the prescale's drop factor and exponent after the tile
    volatile int* grew = reinterpret_cast<volatile int*>(smem + kMisc + 160);
    volatile int* pv_acc = reinterpret_cast<volatile int*>(smem + kMisc + 192);
    volatile float* tdrop = reinterpret_cast<volatile float*>(smem + kMisc + 208);
    volatile int* tkv = reinterpret_cast<volatile int*>(smem + kMisc + 216);
    float* kal = reinterpret_cast<float*>(smem + kAux);          // [2][128] K scales
    float* vsu = kal + 256;                                      // [2][128] V scales * 2^kv
    float* xch = vsu + 256;                                      // [2][128] halves' maxima
    float* lx = xch + 256;                                       // [2][128] spare pair

    // ---- the CTA's (sequence, kv head, row tile) and its KV range
    const int tph = p.tiles_per_head;
    const int b = blockIdx.x / (p.Hk * tph);
    const int rem = blockIdx.x - b * p.Hk * tph;
    const int hk = rem / tph, mt = rem - hk * tph;
    const int G = p.G, T = p.T;
    int L = p.seq_lens[b];
    if (L < T || L > p.max_seq) {                    // (L = 0: zero rows, no flag)
        if (L != 0 && tid == 0 && mt == 0 && hk == 0) raise_flag(p.d_err, KVQ_DEVERR_LEN);
        L = -1;
    }
    const int r_first = mt * kRows;
    const int i_last = min(T - 1, (r_first + kRows - 1) / G);     // last query of the tile
    const int t_hi = L < 0 ? 0 : L - T + i_last + 1;              // keys 0 .. t_hi - 1
    const int ntile = (t_hi + kTok - 1) / kTok;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 1);
            // K: the MMA commit; V and the scales: the two helper warps
            ptx::mbar_init(bar_empty + 8 * s, 1 + 2);
            ptx::mbar_init(bar_aready + 8 * s, 1);
            ptx::mbar_init(bar_afree + 8 * s, 8);
        }
        ptx::mbar_init(bar_sfull, 1);
        ptx::mbar_init(bar_sfree, 8);
        ptx::mbar_init(bar_pfull, 8 + 2);           // P'' by the rows, V16 by the helpers
        ptx::mbar_init(bar_odone, 1);
        ptx::mbar_init(bar_qready, 8);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
    }
    if (warp == 0) {                                 // tensor memory for S_hi, S_lo, O
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         ptx::smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto wait = [&](uint32_t bar, uint32_t parity) {
        if (*abort_flag) return false;
        if (!ptx::mbar_wait(bar, parity)) {
            *abort_flag = 1;
            raise_flag(p.d_err, KVQ_DEVERR_TIMEOUT);
            return false;
        }
        return true;
    };
    // scale rows of tile j start sc_off floats into the stage's copy (the copy
    // starts at the 16-byte aligned float at or below the tile's first)
    const int64_t unit_row = (static_cast<int64_t>(b) * p.Hk + hk) * p.max_seq;
    const int sc_off = static_cast<int>(unit_row & 3);
    const int64_t sc_total = static_cast<int64_t>(p.B) * p.Hk * p.max_seq;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = ptx::policy_evict_first();
            for (int j = 0; j < ntile; ++j) {
                const int s = j & 1;
                if (j >= 2 && !wait(bar_empty + 8 * s, ((j >> 1) - 1) & 1)) break;
                const uint32_t st = sb + kStage0 + s * kStageBytes;
                const int64_t row0 = unit_row + static_cast<int64_t>(j) * kTok;
                const int64_t c0 = row0 - sc_off;
                int nb = (kTok + sc_off + 3) & ~3;
                const int nf = kTok + sc_off;
                if (c0 + nb > sc_total) {            // the tail floats by plain loads
                    nb = nf & ~3;
                    for (int e = nb; e < nf; ++e) {
                        const int64_t gi = c0 + e;
                        const float ks = gi < sc_total ? p.k_scale[gi] : 0.f;
                        const float vs = gi < sc_total ? p.v_scale[gi] : 0.f;
                        asm volatile("st.shared.f32 [%0], %1;" ::"r"(st + kStKs + 4 * e), "f"(ks) : "memory");
                        asm volatile("st.shared.f32 [%0], %1;" ::"r"(st + kStVs + 4 * e), "f"(vs) : "memory");
                    }
                }
                ptx::mbar_arrive_expect_tx(bar_full + 8 * s, 2 * 16384 + 8 * nb);
                ptx::tma_load_2d(st + kStK, &tm_k, 0, static_cast<int>(row0), bar_full + 8 * s, pol);
                ptx::tma_load_2d(st + kStV, &tm_v, 0, static_cast<int>(row0), bar_full + 8 * s, pol);
                if (nb > 0) {
                    ptx::bulk_load(st + kStKs, p.k_scale + c0, 4 * nb, bar_full + 8 * s);
                    ptx::bulk_load(st + kStVs, p.v_scale + c0, 4 * nb, bar_full + 8 * s);
                }
            }
            // the last copies have landed before the CTA can leave
            for (int j = max(ntile - 2, 0); j < ntile; ++j)
                ptx::mbar_wait(bar_full + 8 * (j & 1), (j >> 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        // Order on the tensor pipe: S(0), then per tile j: S(j + 1) as soon as
        // the rows hold tile j's scores in registers (sfree, after their first
        // pass) and its K has landed, and P.V(j) once P'' and V16 are written
        // (pfull).  So the next tile's scores are computed while the rows
        // finish tile j, and P.V(j) runs during their first pass over j + 1.
        if (lane == 0 && ntile > 0 && wait(bar_qready, 0)) {
            const uint64_t dq_hi = smem_desc(sb + kQhi, 16, 1024);
            const uint64_t dq_lo = smem_desc(sb + kQlo, 16, 1024);
            // S = Q K^T of tile j: four k-steps of 32 bytes per digit
            // (descriptor start addresses advance in 16-byte units)
            auto issue_s = [&](int j) {
                const int s = j & 1;
                if (!wait(bar_full + 8 * s, (j >> 1) & 1)) return false;
                tc_fence_after();
                const uint64_t dk = smem_desc(sb + kStage0 + s * kStageBytes + kStK, 16, 1024);
                for (int k = 0; k < 4; ++k)
                    tc_mma<true>(tmem + kColShi, dq_hi + 2 * k, dk + 2 * k, kIdescQkHi, k > 0);
                for (int k = 0; k < 4; ++k)
                    tc_mma<true>(tmem + kColSlo, dq_lo + 2 * k, dk + 2 * k, kIdescQkLo, k > 0);
                tc_commit(bar_sfull);
                tc_commit(bar_empty + 8 * s);       // K consumed
                return true;
            };
            if (issue_s(0)) {
                for (int j = 0; j < ntile; ++j) {
                    if (j + 1 < ntile) {
                        // the rows have read S_hi and S_lo of tile j
                        if (!wait(bar_sfree, j & 1)) break;
                        tc_fence_after();
                        if (!issue_s(j + 1)) break;
                    }
                    if (!wait(bar_pfull, j & 1)) break;
                    tc_fence_after();
                    // O (+)= P'' V: eight k-steps of 16 tokens per part; P rows are
                    // two 64-token atoms, V16 k-steps advance 16 rows of 128 bytes.
                    // The tile's first k-step starts the O tile afresh unless the
                    // rows left it unfolded (then the tile adds onto it)
                    const bool onto = j > 0 && pv_acc[j & 1] != 0;
                    for (int part = 0; part < 2; ++part) {
                        const uint32_t pb = sb + (part ? kPlo : kPhi);
                        for (int k = 0; k < 8; ++k) {
                            const uint64_t da = smem_desc(pb + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                            const uint64_t dv = smem_desc(sb + kV16 + k * 2048, 16384, 1024);
                            tc_mma<false>(tmem + kColO, da, dv, kIdescPv, (onto || part > 0 || k > 0));
                        }
                    }
                    tc_commit(bar_odone);
                }
            }
        }
    } else if (warp >= kAuxWarp) {
        // ------------------------------------------------------------ helpers
        // Per tile j, ahead of the rows: warp 10 copies the K scales and the
        // V scales times the P'' prescale 2^kv into the aligned vectors of the
        // tile's parity (tokens 4 lane .. 4 lane + 3; 0 past the keys), with the
        // largest V scale over the tile: 2^kv only drops, and a drop rescales
        // O.  Then both warps write the tile's V rows as exact f16 (byte - 128)
        // into the MN-major B tile (warp 10 + a: rows 64 a .. 64 a + 63), once
        // the previous P.V has read it.
        const int a = warp - kAuxWarp;
        int kv = 64;
        auto vectors = [&](int j) {
            const int s = j & 1;
            if (!wait(bar_full + 8 * s, (j >> 1) & 1)) return false;
            if (j >= 2 && !wait(bar_afree + 8 * s, ((j >> 1) - 1) & 1)) return false;
            const float* ksc = reinterpret_cast<const float*>(smem + kStage0 + s * kStageBytes + kStKs) + sc_off;
            const float* vsc = reinterpret_cast<const float*>(smem + kStage0 + s * kStageBytes + kStVs) + sc_off;
            float ks[4], vs[4];
            float vm = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int tok = 4 * lane + e;
                const bool real = j * kTok + tok < t_hi;
                ks[e] = real ? ksc[tok] : 0.f;
                vs[e] = real ? vsc[tok] : 0.f;
                vm = fmaxf(vm, vs[e]);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, off));
            float drop = 1.f;
            if (vm > 0.f) {
                const int ev = static_cast<int>((__float_as_uint(vm) >> 23) & 0xffu) - 127;
                const int kn = max(min(kv, 14 - ev), -120);
                if (kn < kv) {
                    drop = pow2i_f(kn - kv);
                    kv = kn;
                }
            }
            const float up = pow2i_f(kv);
            *reinterpret_cast<float4*>(kal + 128 * s + 4 * lane) = make_float4(ks[0], ks[1], ks[2], ks[3]);
            *reinterpret_cast<float4*>(vsu + 128 * s + 4 * lane) =
                make_float4(vs[0] * up, vs[1] * up, vs[2] * up, vs[3] * up);
            if (lane == 0) {
                tdrop[s] = drop;
                tkv[s] = kv;
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_aready + 8 * s);
            return true;
        };
        auto v16 = [&](int j) {
            const int s = j & 1;
            if (a == 1 && !wait(bar_full + 8 * s, (j >> 1) & 1)) return false;
            if (j >= 1 && !wait(bar_odone, (j - 1) & 1)) return false;   // P.V(j - 1) read V16
#pragma unroll 1
            for (int r2 = 0; r2 < 2; ++r2) {
                const int row = 64 * a + 32 * r2 + lane;             // token of the tile
                const uint8_t* vrow = smem + kStage0 + s * kStageBytes + kStV + row * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {            // 16 head_dim values per source chunk
                    const uint4 raw = *reinterpret_cast<const uint4*>(vrow + ((c ^ (row & 7)) << 4));
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                    uint32_t f[8];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        f[2 * w] = ptx::bytes_to_f16x2(w4[w], 0x4140u);
                        f[2 * w + 1] = ptx::bytes_to_f16x2(w4[w], 0x4342u);
                    }
                    const int k0 = 2 * (c & 3);          // chunks (d % 64) / 8 and + 1 of atom c / 4
                    const uint32_t base = kV16 + (c >> 2) * 16384 + row * 128;
                    *reinterpret_cast<uint4*>(smem + base + ((k0 ^ (row & 7)) << 4)) =
                        make_uint4(f[0], f[1], f[2], f[3]);
                    *reinterpret_cast<uint4*>(smem + base + (((k0 + 1) ^ (row & 7)) << 4)) =
                        make_uint4(f[4], f[5], f[6], f[7]);
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(bar_pfull);
                ptx::mbar_arrive(bar_empty + 8 * s);    // V and scales consumed
            }
            return true;
        };
        bool ok = ntile > 0 && (a != 0 || vectors(0));
        for (int j = 0; ok && j < ntile; ++j) {
            if (a == 0 && j + 1 < ntile && !vectors(j + 1)) break;
            ok = v16(j);
        }
    } else {
        // ------------------------------------------------------------ rows
        const int i_row = 32 * (warp & 3) + lane;       // TMEM lane
        const int hf = warp >> 2;                       // half of the row's columns
        const int r = r_first + i_row;
        const int qi = r / G, h = r - qi * G;
        const bool valid = L >= 0 && qi < T;
        const int pos = L - T + qi;                     // the query's position
        const int64_t orow = (static_cast<int64_t>(b) * p.Hq + hk * G + h) * T + qi;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        auto row_sync = [] { ptx::named_bar_sync(1, kRowThreads); };
        // ---- Q digits of this row (this half's 64 head_dim values) into the
        // swizzled A tiles; the row's max |q| and digit sum over both halves
        float zs = 0.f;
        int cq = 0;
        {
            float qf[64];
            float amax = 0.f;
            if (valid) {
                const uint4* src = reinterpret_cast<const uint4*>(p.q + orow * kDim + 64 * hf);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 raw = src[c];
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        qf[8 * c + 2 * e] = bf16_bits_to_f32(w4[e] & 0xffffu);
                        qf[8 * c + 2 * e + 1] = bf16_bits_to_f32(w4[e] >> 16);
                    }
                }
#pragma unroll
                for (int d = 0; d < 64; ++d) amax = fmaxf(amax, fabsf(qf[d]));
            } else {
#pragma unroll
                for (int d = 0; d < 64; ++d) qf[d] = 0.f;
            }
            lx[128 * hf + i_row] = amax;
            row_sync();
            amax = fmaxf(lx[i_row], lx[128 + i_row]);
            int sh = 0;
            if (amax > 0.f) {
                const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
                sh = min(max(14 - e, -100), 100);
            }
            const float up = pow2i_f(sh);
            zs = pow2i_f(-sh) * p.scale_log2;
            int qsum = 0;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {            // 16 values = one 16-byte chunk per digit
                const int c = 4 * hf + cc;
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t hw = 0, lw = 0;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int v = min(max(__float2int_rn(qf[16 * cc + 4 * w + e] * up), -32767), 32767);
                        qsum += v;
                        hw |= ((static_cast<uint32_t>(v) >> 8) & 0xffu) << (8 * e);
                        lw |= (static_cast<uint32_t>(v) & 0xffu) << (8 * e);
                    }
                    hi[w] = hw;
                    lo[w] = lw;
                }
                const uint32_t off = i_row * 128 + ((c ^ (i_row & 7)) << 4);
                *reinterpret_cast<uint4*>(smem + kQhi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(smem + kQlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            xch[128 * hf + i_row] = __int_as_float(qsum);
            row_sync();
            cq = 128 * (__float_as_int(xch[i_row]) + __float_as_int(xch[128 + i_row]));
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_qready);

        float m_run = -INFINITY, l_run = 0.f;            // l_run: this half's tokens
        int kv = 64;                                     // P'' prescale exponent (CTA-uniform)
        // Lazy fold: the O tile adds up the P.V of consecutive tiles while no
        // row's maximum grows and the prescale stays (they share one scale),
        // up to kFoldEvery tiles; it is folded into the running sum (O run)
        // before the P.V of a tile that changes the scale, or at the limit:
        // run = run * f_run + tile, f_run the factor from the running sum's
        // scale to the O tile's (one factor per fold: between folds every
        // factor is 1)
        constexpr int kFoldEvery = 8;
        float f_run = 1.f;
        bool has_run = false;                            // O run holds a sum
        int n_acc = 0;                                   // tiles summed in the O tile
        bool live = true;                                // no wait has given up
        for (int j = 0; j < ntile; ++j) {
            const int s = j & 1;
            const int t0 = j * kTok;
            const float* kal_j = kal + 128 * s;
            const float* vsu_j = vsu + 128 * s;
            // the tile's K scales, V scales * 2^kv and prescale drop (helpers)
            live = live && wait(bar_aready + 8 * s, (j >> 1) & 1);
            const float drop = live ? tdrop[s] : 1.f;
            if (live) kv = tkv[s];
            live = live && wait(bar_sfull, j & 1);
            tc_fence_after();
            // ---- pass 1: x = S * k_scale over this half's tokens (-inf where the
            // causal mask drops the key) and its maximum; x stays in registers
            // (xr), so pass 2 needs no mask, no integer reconstruction and no
            // tensor memory, and S is free for the next tile's Q K^T at once
            // (a warp whose rows all see the whole half skips the mask test)
            const int tb = t0 + 64 * hf;                 // this half's first token
            const bool unmasked = valid && tb + 63 <= pos;
            const bool warp_unmasked = __all_sync(0xffffffffu, unmasked);
            float xmax = -INFINITY;
            uint32_t xr[2][32];
            if (live) {
#pragma unroll
                for (int cl = 0; cl < 2; ++cl) {
                    const int c = 2 * hf + cl;
                    uint32_t sl_[32];
                    tmem_ld32(lane_base + kColShi + 32 * c, xr[cl]);
                    tmem_ld32(lane_base + kColSlo + 32 * c, sl_);
                    tmem_wait_ld();
                    if (warp_unmasked) {
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const float4 k4 = *reinterpret_cast<const float4*>(kal_j + 32 * c + 4 * e4);
                            const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int e = 4 * e4 + u;
                                const int S = static_cast<int>(xr[cl][e]) * 256 + static_cast<int>(sl_[e]) - cq;
                                const float x = static_cast<float>(S) * kk[u];
                                xmax = fmaxf(xmax, x);
                                xr[cl][e] = __float_as_uint(x);
                            }
                        }
                    } else {
#pragma unroll
                        for (int e4 = 0; e4 < 8; ++e4) {
                            const float4 k4 = *reinterpret_cast<const float4*>(kal_j + 32 * c + 4 * e4);
                            const float kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int e = 4 * e4 + u;
                                const int S = static_cast<int>(xr[cl][e]) * 256 + static_cast<int>(sl_[e]) - cq;
                                const bool on = valid && t0 + 32 * c + e <= pos;
                                const float x = on ? static_cast<float>(S) * kk[u] : -INFINITY;
                                xmax = fmaxf(xmax, x);
                                xr[cl][e] = __float_as_uint(x);
                            }
                        }
                    }
                }
            }
            // S_hi / S_lo read into registers: the next Q K^T may start
            tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_sfree);
            xch[128 * hf + i_row] = xmax;
            {
                const bool g = __any_sync(0xffffffffu, xmax * zs > m_run);
                if (lane == 0) grew[warp] = g ? 1 : 0;
            }
            row_sync();
            const float xm = fmaxf(xch[i_row], xch[128 + i_row]);
            const float m_new = fmaxf(m_run, xm * zs);
            const float mb = m_new == -INFINITY ? 0.f : m_new;
            const float alpha = (m_run == -INFINITY || m_new <= m_run) ? 1.f : ptx::ex2(m_run - mb);
            bool any_grew = false;
#pragma unroll
            for (int w = 0; w < 8; ++w) any_grew = any_grew || grew[w] != 0;
            // fold the O tile into the running sum before this tile's P.V (a
            // CTA-wide decision: every row reads the same flags)
            const bool fold_now = j >= 1 && (any_grew || drop != 1.f || n_acc >= kFoldEvery);
            // the previous P.V is done: P, V16 free, O stable
            if (j >= 1) live = live && wait(bar_odone, (j - 1) & 1);
            tc_fence_after();
            // the fold (this half's head_dim columns, in 16-column pieces)
            if (live && fold_now) {
#pragma unroll 1
                for (int cl = 0; cl < 4; ++cl) {
                    const int c = 4 * hf + cl;           // 16-column pieces
                    uint32_t ot[16], orn[16];
                    tmem_ld16(lane_base + kColO + 16 * c, ot);
                    if (has_run) tmem_ld16(lane_base + kColRun + 16 * c, orn);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        orn[e] = __float_as_uint(has_run ? fmaf(__uint_as_float(orn[e]), f_run,
                                                                __uint_as_float(ot[e]))
                                                         : __uint_as_float(ot[e]));
                    tmem_st16(lane_base + kColRun + 16 * c, orn);
                }
                tmem_wait_st();
            }
            if (fold_now) {
                has_run = true;
                f_run = alpha * drop;                    // the running sum's scale -> this tile's
                n_acc = 0;
            }
            ++n_acc;
            if (tid == 0) pv_acc[s] = (j >= 1 && !fold_now) ? 1 : 0;   // read after pfull
            // ---- pass 2: P'' = 2^(x zs - m) * v_scale * 2^kv as f16 hi + lo for
            // this half's tokens (P atom hf); x = -inf (masked) gives 0
            float lsum = 0.f;
            if (live) {
#pragma unroll
                for (int cl = 0; cl < 2; ++cl) {
                    const int c = 2 * hf + cl;
                    const uint32_t (&xs)[32] = xr[cl];
                    uint32_t ph[16], pl[16];
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 v4 = *reinterpret_cast<const float4*>(vsu_j + 32 * c + 4 * e4);
                        const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
                        float pp[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float pe = ptx::ex2(fmaf(__uint_as_float(xs[4 * e4 + u]), zs, -mb));
                            lsum += pe;
                            pp[u] = pe * vv[u];
                        }
#pragma unroll
                        for (int u = 0; u < 4; u += 2) {
                            const __half2 hh = __floats2half2_rn(pp[u], pp[u + 1]);
                            const float2 hfl = __half22float2(hh);
                            const __half2 ll = __floats2half2_rn(pp[u] - hfl.x, pp[u + 1] - hfl.y);
                            ph[2 * e4 + (u >> 1)] = *reinterpret_cast<const uint32_t*>(&hh);
                            pl[2 * e4 + (u >> 1)] = *reinterpret_cast<const uint32_t*>(&ll);
                        }
                    }
                    // tokens 32c .. 32c + 31: atom c / 2 = hf, chunks 4 cl .. + 3
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int kc = 4 * cl + x;
                        const uint32_t off = hf * 16384 + i_row * 128 + ((kc ^ (i_row & 7)) << 4);
                        *reinterpret_cast<uint4*>(smem + kPhi + off) =
                            make_uint4(ph[4 * x], ph[4 * x + 1], ph[4 * x + 2], ph[4 * x + 3]);
                        *reinterpret_cast<uint4*>(smem + kPlo + off) =
                            make_uint4(pl[4 * x], pl[4 * x + 1], pl[4 * x + 2], pl[4 * x + 3]);
                    }
                }
            }
            l_run = l_run * alpha + lsum;
            m_run = m_new;
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(bar_afree + 8 * s);    // this parity's vectors read
                ptx::mbar_arrive(bar_pfull);
            }
        }
        // ---- the row: (run * f_run + O tile) * 2^-kv / l, l over both halves
        lx[128 * hf + i_row] = l_run;
        row_sync();
        const float l_tot = lx[i_row] + lx[128 + i_row];
        if (ntile > 0 && live && wait(bar_odone, (ntile - 1) & 1)) {
            tc_fence_after();
            const float f = (valid && l_tot > 0.f) ? pow2i_f(-kv) / l_tot : 0.f;
#pragma unroll 1
            for (int cl = 0; cl < 2; ++cl) {
                const int c = 2 * hf + cl;
                uint32_t ot[32], orn[32];
                tmem_ld32(lane_base + kColO + 32 * c, ot);
                if (has_run) tmem_ld32(lane_base + kColRun + 32 * c, orn);
                tmem_wait_ld();
                float o_[32];
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    o_[e] = (has_run ? fmaf(__uint_as_float(orn[e]), f_run, __uint_as_float(ot[e]))
                                     : __uint_as_float(ot[e])) * f;
                if (valid) {
                    float4* dst = reinterpret_cast<float4*>(p.out + orow * kDim + 32 * c);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        dst[x] = make_float4(o_[4 * x], o_[4 * x + 1], o_[4 * x + 2], o_[4 * x + 3]);
                }
            }
        } else if (ntile == 0 && (valid || (L < 0 && qi < T))) {
            // no key (an empty or rejected sequence): a zero row
            float4* dst = reinterpret_cast<float4*>(p.out + orow * kDim + 64 * hf);
            for (int x = 0; x < 16; ++x) dst[x] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

bool chunk_tc_supported(int D, int G, int T, int group32, int fp8, int static_ns, int page_size,
                        int window, int recent) {
    return D == kDim && G * T > 16 && !group32 && !fp8 && !static_ns && page_size == 0 &&
           window == 0 && recent == 0;
}

cudaError_t launch_chunk_tc(const DecodeParams& dp, int Hq, int G, int T, cudaStream_t s) {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = once_per_device(done, dev, cudaSuccess, [] {
        return cudaFuncSetAttribute(chunk_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kSmem);
    });
    if (e != cudaSuccess) return e;
    CUtensorMap mk, mv;
    const int64_t rows = static_cast<int64_t>(dp.B) * dp.Hk * dp.max_seq;
    e = make_tile_map(&mk, dp.k, kDim, rows, kTok);
    if (e == cudaSuccess) e = make_tile_map(&mv, dp.v, kDim, rows, kTok);
    if (e != cudaSuccess) return e;
    ChunkParams p{};
    p.q = dp.q; p.k_scale = dp.k_scale; p.v_scale = dp.v_scale; p.seq_lens = dp.seq_lens;
    p.out = dp.out; p.d_err = dp.d_err;
    p.B = dp.B; p.Hq = Hq; p.Hk = dp.Hk; p.G = G; p.T = T; p.max_seq = dp.max_seq;
    p.tiles_per_head = (G * T + kRows - 1) / kRows;
    p.scale_log2 = dp.scale_log2;
    const int64_t grid = static_cast<int64_t>(dp.B) * dp.Hk * p.tiles_per_head;
    if (grid < 1 || grid > 0x7fffffffll) return cudaErrorInvalidValue;
    chunk_attn_tc<<<static_cast<unsigned>(grid), kThreads, kSmem, s>>>(mk, mv, p);
    return cudaGetLastError();
}

}  // namespace kvq

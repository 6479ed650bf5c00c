// kvq_decode_simt.cu -- decode, chunk and sliding-window attention on the
// quantised cache for the shapes the tensor-core kernels do not take: head
// dims other than 64 and 128 (any D % 16 == 0 up to 256), more than 16
// (head, query) rows per kv head outside the dense kernel's shapes, and
// batches above the split kernel's cached lengths.  Plain FP32 arithmetic
// on the CUDA cores, with the same split plan, the same workspace of o / m / l
// partials and the same combine kernel as the split kernel.
//
// Method: abaddon 0.2.0-rc.1, src/kv_cache_quant_cuda.rs, module doc
// "Fused approach" -- scores from K dequantised on the fly, softmax, P.V
// with V dequantised on the fly; combs-models 0.2.2, src/kv.rs, attend /
// repeat_kv -- query head h reads kv head h / G; chunk rows and windows as
// in the split kernel (row i of a chunk of T sees positions <= L - T + i and,
// with a window w, >= L - T + i - w + 1).  Dequantisation per cache format:
// (byte - 128) * scale for INT8 (scale per token, per 32-value group, per
// head or per channel), the exact FP8 value for E4M3 / E5M2.
//
// Mapping: CTA = (sequence b, kv head, chunk j) x (block of up to kRB rows);
// four warps take the chunk's tokens round robin.  For a token, lane l holds
// head_dim d = l + 32 i (i < VPL = ceil(D / 32)) of the dequantised K and V
// rows; the kRB scores are warp all-reductions of q . k; each warp keeps an
// online softmax (base 2) and its o rows in registers; the four warps merge
// through shared memory into the chunk's partial (or the final rows when the
// sequence is one chunk).
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include <climits>

#include "kvq_internal.cuh"
#include "kvq_ptx.cuh"

namespace kvq {
namespace {

constexpr int kSW = 4;                  // warps per CTA
constexpr int kST = 32 * kSW;           // threads per CTA
constexpr int kRB = 8;                  // rows per CTA
constexpr int kDMax = 256;

// the exact value of an FP8 byte (fmt 1: E4M3, 2: E5M2)
__device__ __forceinline__ float fp8_val(uint32_t byte, int fmt) {
    if (fmt == 2) return __half2float(__ushort_as_half(static_cast<unsigned short>(byte << 8)));
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(byte), __NV_E4M3);
    return __half2float(__half(h));
}

template <int VPL>
__global__ void __launch_bounds__(kST)
decode_simt(DecodeParams p) {
    __shared__ float q_s[kRB][kDMax];                       // q rows, times scale_log2
    __shared__ float o_s[kSW][kRB][kDMax];                  // per-warp o rows
    __shared__ float m_s[kSW][kRB], l_s[kSW][kRB];
    grid_dep_wait();                    // inputs written by the preceding grid
    grid_dep_launch();
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int D = p.D, G = p.G, Hk = p.Hk, splits = p.splits;
    const int item = static_cast<int>(blockIdx.x);
    const int b = item / (Hk * splits);
    const int rr = item - b * Hk * splits;
    const int hk = rr / splits, j = rr - (rr / splits) * splits;
    const int row0 = static_cast<int>(blockIdx.y) * kRB;
    const int nr = min(kRB, G - row0);
    const bool paged = p.page_size != 0;

    // the walked length (from the window base) and this chunk's tokens
    const int64_t cap = paged ? static_cast<int64_t>(p.max_pages) * p.page_size : p.max_seq;
    const int Lraw = p.seq_lens[b];
    int L = walked_len(Lraw, cap, static_cast<int64_t>(splits) * p.chunk, p.qlen, p.window,
                       p.recent);
    if (L < 0 || (p.qlen > 1 && Lraw > 0 && Lraw < p.qlen)) {
        if (j == 0 && hk == 0 && blockIdx.y == 0 && tid == 0) raise_flag(p.d_err, KVQ_DEVERR_LEN);
        L = 0;
    }
    const int Lint = Lraw > p.recent ? Lraw - p.recent : 0;      // the INT8 part
    const int wb = L > 0 ? window_base(Lint, p.qlen, p.window) : 0;
    const int ns = (L + p.chunk - 1) / p.chunk;
    if (j >= (ns > 0 ? ns : 1)) return;  // past the chunk count: no partial
    const int t0 = j * p.chunk, t1 = min(t0 + p.chunk, L);
    const int64_t bh0 = static_cast<int64_t>(b) * p.Hq + static_cast<int64_t>(hk) * G + row0;
    const int64_t bhk = static_cast<int64_t>(b) * Hk + hk;
    const int NG = p.group32 ? D / 32 : 1;

    // query rows: bf16 -> fp32, times attn_scale * log2(e)
    for (int x = tid; x < nr * D; x += kST) {
        const int r = x / D, d = x - r * D;
        q_s[r][d] = bf16_bits_to_f32(p.q[(bh0 + r) * D + d]) * p.scale_log2;
    }
    // causal / window limits of the rows (counted from the window base)
    int lim[kRB], lo[kRB];
#pragma unroll
    for (int r = 0; r < kRB; ++r) {
        const int col = row0 + r;
        lim[r] = (p.qlen > 1 || p.window > 0) ? L - p.qlen + col % p.qlen : INT_MAX;
        lo[r] = p.window > 0 ? lim[r] - p.window + 1 : INT_MIN;
    }
    __syncthreads();

    // ---- fused append (INT8 per token / group-32, decode): the chunk that
    // holds position L - 1 quantises the new token itself -- the append
    // kernels' quantiser, in every CTA of the chunk alike -- and uses its
    // dequantised values for that position; the first row block's CTA also
    // writes the bytes and scales into the cache
    int tok = -1;
    float kn[VPL], vn[VPL];
    if (p.k_new != nullptr && L > 0 && L - 1 >= t0 && L - 1 < t1) {
        tok = L - 1;
        float xk[VPL], xv[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int d = lane + 32 * i;
            xk[i] = d < D ? bf16_bits_to_f32(p.k_new[bhk * D + d]) : 0.f;
            xv[i] = d < D ? bf16_bits_to_f32(p.v_new[bhk * D + d]) : 0.f;
        }
        float sk[VPL], sv[VPL];
        if (p.group32) {                 // group i = head_dim [32 i, 32 i + 32): lanes
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                float ak = fabsf(xk[i]), av = fabsf(xv[i]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
                    av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
                }
                sk[i] = q8_scale(ak);
                sv[i] = q8_scale(av);
            }
        } else {                         // per token: the whole row
            float ak = 0.f, av = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                ak = fmaxf(ak, fabsf(xk[i]));
                av = fmaxf(av, fabsf(xv[i]));
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
                av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
            }
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                sk[i] = q8_scale(ak);
                sv[i] = q8_scale(av);
            }
        }
        int64_t crow = -1;               // the cache row (paged: a valid page only)
        if (paged) {
            const int32_t pg = p.table[static_cast<int64_t>(b) * p.max_pages + ((wb + tok) >> 4)];
            if (pg >= 0 && pg < p.num_pages)
                crow = (static_cast<int64_t>(pg) * Hk + hk) * p.page_size + ((wb + tok) & 15);
        } else {
            crow = bhk * p.max_seq + wb + tok;
        }
        const bool writer = blockIdx.y == 0 && w == 0 && crow >= 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int d = lane + 32 * i;
            const uint32_t bk = q8_byte(xk[i], sk[i], __frcp_rn(sk[i]));
            const uint32_t bv = q8_byte(xv[i], sv[i], __frcp_rn(sv[i]));
            kn[i] = static_cast<float>(static_cast<int>(bk) - 128) * sk[i];
            vn[i] = static_cast<float>(static_cast<int>(bv) - 128) * sv[i];
            if (writer && d < D) {
                p.k_w[crow * D + d] = static_cast<uint8_t>(bk);
                p.v_w[crow * D + d] = static_cast<uint8_t>(bv);
                if (lane == 0 && (p.group32 || i == 0)) {
                    p.ks_w[crow * NG + (p.group32 ? i : 0)] = sk[i];
                    p.vs_w[crow * NG + (p.group32 ? i : 0)] = sv[i];
                }
            }
        }
    }

    float m[kRB], l[kRB], o[kRB][VPL];
#pragma unroll
    for (int r = 0; r < kRB; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int i = 0; i < VPL; ++i) o[r][i] = 0.f;
    }
#pragma unroll 1
    for (int t = t0 + w; t < t1; t += kSW) {
        const int g = wb + t;                 // position in the sequence
        int64_t row;
        if (paged) {
            const int32_t pg = p.table[static_cast<int64_t>(b) * p.max_pages + (g >> 4)];
            if (pg < 0 || pg >= p.num_pages) {
                if (lane == 0) raise_flag(p.d_err, KVQ_DEVERR_PAGE);
                continue;                     // the token is skipped
            }
            row = (static_cast<int64_t>(pg) * Hk + hk) * p.page_size + (g & 15);
        } else {
            row = bhk * p.max_seq + g;
        }
        float kx[VPL], vx[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int d = lane + 32 * i;
            kx[i] = vx[i] = 0.f;
            if (t == tok) {              // the new token, quantised above
                kx[i] = kn[i];
                vx[i] = vn[i];
            } else if (d < D) {
                const uint32_t kb = p.k[row * D + d], vb = p.v[row * D + d];
                if (p.fp8) {
                    kx[i] = fp8_val(kb, p.fp8);
                    vx[i] = fp8_val(vb, p.fp8);
                } else {
                    float ks, vs;
                    if (p.static_ns) {
                        const int64_t si = bhk * p.static_ns + (p.static_ns > 1 ? d : 0);
                        ks = p.k_scale[si];
                        vs = p.v_scale[si];
                    } else {
                        const int64_t si = row * NG + (p.group32 ? d >> 5 : 0);
                        ks = p.k_scale[si];
                        vs = p.v_scale[si];
                    }
                    kx[i] = static_cast<float>(static_cast<int>(kb) - 128) * ks;
                    vx[i] = static_cast<float>(static_cast<int>(vb) - 128) * vs;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kRB; ++r) {
            if (r >= nr) break;
            float s = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int d = lane + 32 * i;
                if (d < D) s = fmaf(q_s[r][d], kx[i], s);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (t > lim[r] || t < lo[r]) continue;        // masked for this row
            const float mn = fmaxf(m[r], s);
            const float a = m[r] == -INFINITY ? 0.f : ptx::ex2(m[r] - mn);
            const float pr = ptx::ex2(s - mn);
            l[r] = fmaf(l[r], a, pr);
#pragma unroll
            for (int i = 0; i < VPL; ++i) o[r][i] = fmaf(o[r][i], a, pr * vx[i]);
            m[r] = mn;
        }
    }

    // ---- merge the four warps' states
#pragma unroll
    for (int r = 0; r < kRB; ++r) {
        if (lane == 0) {
            m_s[w][r] = m[r];
            l_s[w][r] = l[r];
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int d = lane + 32 * i;
            if (d < D) o_s[w][r][d] = o[r][i];
        }
    }
    __syncthreads();
    const bool final_rows = p.recent == 0 && ns <= 1;
    for (int x = tid; x < nr * D; x += kST) {
        const int r = x / D, d = x - r * D;
        float M = -INFINITY;
#pragma unroll
        for (int u = 0; u < kSW; ++u) M = fmaxf(M, m_s[u][r]);
        float Ls = 0.f, O = 0.f;
#pragma unroll
        for (int u = 0; u < kSW; ++u) {
            const float f = m_s[u][r] == -INFINITY ? 0.f : ptx::ex2(m_s[u][r] - M);
            Ls = fmaf(l_s[u][r], f, Ls);
            O = fmaf(o_s[u][r][d], f, O);
        }
        const int64_t orow = bh0 + r;
        if (final_rows) {
            p.out[orow * D + d] = Ls > 0.f ? O * __frcp_rn(Ls) : 0.f;
        } else {
            p.ws_o[(orow * splits + j) * D + d] = O;
            if (d == 0) {
                p.ws_m[orow * splits + j] = M;
                p.ws_l[orow * splits + j] = Ls;
            }
        }
    }
}

template <int VPL>
cudaError_t launch_vpl(const DecodeParams& p, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(static_cast<int64_t>(p.B) * p.Hk * p.splits),
                       static_cast<unsigned>((p.G + kRB - 1) / kRB), 1);
    cfg.blockDim = dim3(kST, 1, 1);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_simt<VPL>, p);
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t s) {
    if (p.D < 16 || p.D > kDMax || (p.D % 16) != 0 || p.G < 1 || p.page_size > 16 ||
        (p.page_size != 0 && p.page_size != 16) ||
        static_cast<int64_t>(p.B) * p.Hk * p.splits >= (int64_t{1} << 31) ||
        (p.G + kRB - 1) / kRB > 65535)
        return cudaErrorInvalidValue;
    switch ((p.D + 31) / 32) {
        case 1: return launch_vpl<1>(p, s);
        case 2: return launch_vpl<2>(p, s);
        case 3: return launch_vpl<3>(p, s);
        case 4: return launch_vpl<4>(p, s);
        case 5: return launch_vpl<5>(p, s);
        case 6: return launch_vpl<6>(p, s);
        case 7: return launch_vpl<7>(p, s);
        default: return launch_vpl<8>(p, s);
    }
}

}  // namespace kvq

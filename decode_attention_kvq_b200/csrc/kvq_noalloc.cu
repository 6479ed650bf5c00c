// kvq_noalloc.cu -- kvq_decode_attn_noalloc: decode attention for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run attention: embedded or plugin hosts that hand the library only
// their own input/output buffers, or runtimes whose allocator is not
// reachable from this C interface.  kvq_decode_attn needs a split-K scratch workspace
// from its caller; this entry point instead uses a fixed-size scratch array
// that lives in the library itself (a file-scope __device__ array, present on
// every GPU that loads the library until the process exits).
//
// Host code cannot use the array's name as a device address: the symbol's
// device address is obtained once per device with cudaGetSymbolAddress
// while that device is current, cached, and passed to the kernels.
#include <atomic>

#include "kvq_internal.cuh"

namespace {

constexpr size_t kScratchBytes = 16u << 20;   // 16 MiB of split-K partials

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_decode_scratch on the current device (set up on the
// first call per device).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void* ptr = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!ptr) {
        e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev].store(ptr, std::memory_order_release);
    }
    *out = ptr;
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t kvq_noalloc_scratch_bytes(void) { return kScratchBytes; }

kvq_status kvq_decode_attn_noalloc(const uint16_t* q, int B, int Hq, int Hk, int D,
                                   kvq_scale_mode mode, const kvq_cache_view* kv,
                                   const int32_t* d_seq_lens, int max_seq_len_hint,
                                   float attn_scale, float* out, int num_splits, int32_t* d_err,
                                   kvq_stream_t stream) {
    const size_t need = kvq_decode_workspace_bytes(B, Hq, Hk, D, max_seq_len_hint, num_splits);
    if (need > kScratchBytes) return KVQ_ERR_SCRATCH_TOO_SMALL;
    void* ws = nullptr;
    if (need > 0 && scratch_address(&ws) != cudaSuccess) return KVQ_ERR_CUDA;
    return kvq_decode_attn(q, B, Hq, Hk, D, mode, kv, d_seq_lens, max_seq_len_hint, attn_scale, out,
                           ws, need > 0 ? kScratchBytes : 0, num_splits, d_err, stream);
}

}  // extern "C"

// gdla_decode_noalloc.cu - the decode entry point for callers that cannot
// allocate device memory.
//
// Some callers only ever hold the buffers they are handed: a plugin running
// inside another inference runtime that forbids device allocation on its
// execution path, or a service with a fixed, pre-reserved memory budget where
// a cudaMalloc could fail or synchronise the device mid-request. They cannot
// provide the split-KV workspace gdla_attn_decode asks for. This entry point
// runs the same decode kernels with their scratch in a file-scope device array
// of fixed size (GDLA_DECODE_STATIC_SCRATCH_BYTES), which the CUDA runtime
// places in the module's global memory when the library's module is loaded on
// a device; every device that loads the library keeps that memory until the
// process exits.
//
// In host code `g_decode_scratch` names a host-side stand-in, not a device
// address: passing it to a kernel would fault (or, where the GPU can reach
// host memory, silently use the wrong memory). The device address is looked
// up with cudaGetSymbolAddress once per device and context, with that device
// current.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "gdla.h"
#include "gdla_internal.h"

namespace gdla {

static __device__ __align__(256) float g_decode_scratch[GDLA_DECODE_STATIC_SCRATCH_BYTES / sizeof(float)];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context the cached address belongs to

// Device address of g_decode_scratch on the current device. The first call in
// a context performs the lookup (with that device current) and caches it for
// that context; after a device reset the module is loaded afresh in a new
// context, so the address is looked up again rather than reused.
cudaError_t static_scratch_address(void **addr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    unsigned long long ctx = current_context_id();
    if (ctx == 0 || g_scratch_addr[dev] == nullptr || g_scratch_ctx[dev] != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = current_context_id();  // the lookup made the context current if it was not
    }
    *addr = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace gdla

extern "C" gdla_status_t gdla_attn_decode_noalloc(const void *q_sig, const void *q_noise, const void *k_cache,
                                                  const void *v_cache, const int32_t *cu_seqlens_k,
                                                  int num_cache_rows, int max_seqlen_k, const float *lambda,
                                                  const void *gate_logits, void *out, int batch, int num_kv_heads,
                                                  int window, void *stream) {
    // Same split plan as gdla_attn_decode; sizes whose plan needs more scratch
    // than the fixed array holds are rejected before anything is launched.
    const size_t need = gdla_decode_workspace_bytes(batch, num_kv_heads, max_seqlen_k, window);
    if (need > GDLA_DECODE_STATIC_SCRATCH_BYTES) return GDLA_ERR_WORKSPACE;
    void *ws = nullptr;
    if (need > 0 && gdla::static_scratch_address(&ws) != cudaSuccess) return GDLA_ERR_CUDA;
    // Every scratch slot is written by the split kernel before the combine
    // kernel reads it, so the array's previous contents never matter and
    // nothing has to be cleared between calls.
    return gdla_attn_decode(q_sig, q_noise, k_cache, v_cache, cu_seqlens_k, num_cache_rows, max_seqlen_k, lambda,
                            gate_logits, out, batch, num_kv_heads, window, ws, need > 0 ? GDLA_DECODE_STATIC_SCRATCH_BYTES : 0,
                            stream);
}

// noalloc.cu — lsa_attend_noalloc: sparse attention for callers that cannot
// allocate device memory.
//
// lsa_attend needs a caller-provided workspace for its split partials. Some
// callers cannot call cudaMalloc on this path: an
// engine whose device memory is owned entirely by its own pool allocator
// (a raw cudaMalloc would fail or fragment that pool), or a decode loop that
// must never run an allocation (cudaMalloc/cudaFree may synchronise the
// device). For them this entry point keeps its scratch in a file-scope
// device array of fixed size and forwards to lsa_attend unchanged.
//
// In host code `g_attend_scratch` names a host-side stand-in, not a device
// address: the device address is fetched with cudaGetSymbolAddress, once per
// device, with that device current, on the first call made on it.
#include <cstdint>
#include <mutex>

#include "../../include/lsa.h"
#include "internal.h"

namespace {

static __device__ __align__(256) uint8_t g_attend_scratch[LSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_attend_scratch on the current device (set up on first use).
lsa_status_t scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LSA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return LSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_attend_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return LSA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LSA_OK;
}

}  // namespace

extern "C" lsa_status_t lsa_attend_noalloc(const uint16_t* const* q, const uint16_t* const* k_cache,
                                           const uint16_t* const* v_cache, int32_t H_q, int32_t H_kv, int32_t d,
                                           const int32_t* index_sets, int32_t budget, const lsa_batch_t* batch,
                                           int32_t layers_per_index, float* const* out, int32_t* dev_status,
                                           void* stream) {
    if (batch == nullptr) return LSA_ERR_INVALID_ARG;
    const size_t need = lsa_attend_workspace_size(batch, H_q, H_kv, d, budget, layers_per_index);
    if (need > (size_t)LSA_NOALLOC_SCRATCH_BYTES) return LSA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    const lsa_status_t st = scratch_on_current_device(&scratch);
    if (st != LSA_OK) return st;
    // The array keeps the previous call's contents; lsa_attend writes every
    // partial before reading it, so nothing needs clearing.
    return lsa_attend(q, k_cache, v_cache, H_q, H_kv, d, index_sets, budget, batch, layers_per_index, out, scratch,
                      (size_t)LSA_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}

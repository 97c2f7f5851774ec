// orthrus_attn_static: orthrus_attn for callers that cannot allocate device
// memory.
//
// Some callers have no way to call cudaMalloc at the point where they run
// attention: a host runtime whose allocator is owned by another framework, an
// inference engine that must not allocate after warm-up (every byte is planned
// up front), or a plugin whose interface hands it only input and output
// pointers.  For them this entry point uses a fixed scratch array that lives
// in the library itself, instead of a caller-provided workspace.
//
// The scratch is a file-scope __device__ array of ORTHRUS_STATIC_SCRATCH_BYTES;
// every GPU that loads the library holds it until the process exits.  Its
// device address is looked up once per device, on the first call made while
// that device is current (cudaGetSymbolAddress), so make the first call on each
// device before any stream capture.  All calls share the one array.  Each call
// first clears the array's split-merge counter block on `stream` (an async
// memset of a few hundred bytes, no allocation), so a call that gave up on a
// wait (ORTHRUS_STATUS_TIMEOUT) cannot leave stale counters for the next one;
// the rest of the array is scratch that every call overwrites before reading.
// Calls that overlap on the GPU (other streams, other host threads) race on
// the array.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_scratch[ORTHRUS_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_scratch on the current device (looked up once per device).
void *scratch_address()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int orthrus_attn_static(orthrus_view view, orthrus_dtype dtype, const void *q,
                                   const void *k_cache, const void *v_cache,
                                   const int32_t *ctx_lens, int B, int Hq, int Hkv, int D,
                                   int S_max, int K, float scale, float *out, int32_t *status,
                                   void *stream)
{
    const size_t need = orthrus_attn_workspace_size(B, Hq, Hkv, D, K, dtype);
    if (need == 0)      // invalid sizes or no device: let orthrus_attn name the error
        return orthrus_attn(view, dtype, q, k_cache, v_cache, ctx_lens, B, Hq, Hkv, D, S_max, K,
                            scale, out, nullptr, 0, status, stream);
    if (need > (size_t)ORTHRUS_STATIC_SCRATCH_BYTES) return ORTHRUS_ERR_WORKSPACE;
    void *scratch = scratch_address();
    if (!scratch) return ORTHRUS_ERR_DEVICE;
    if (cudaMemsetAsync(scratch, 0, orthrus::kSyncBytes, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess) {
        cudaGetLastError();
        return ORTHRUS_ERR_LAUNCH;
    }
    return orthrus_attn(view, dtype, q, k_cache, v_cache, ctx_lens, B, Hq, Hkv, D, S_max, K,
                        scale, out, scratch, (size_t)ORTHRUS_STATIC_SCRATCH_BYTES, status, stream);
}

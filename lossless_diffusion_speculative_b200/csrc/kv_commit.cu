// Commit of the accepted prefix (Orthrus technical summary, gist.science,
// section 2.3: commit the synchronised prefix, append the AR correction,
// truncate the cache).  n_b = min(a_b + 1, K) block slots are kept; rollback
// is the length change alone.
//
//   copy kernel    (only with staging buffers): grid (row chunks, B, layers);
//                  16-byte copies of slots 0..n_b-1 from [B, K, Hkv, D]
//                  staging into cache rows [ctx_b, ctx_b + n_b).
//   advance kernel one thread per sequence: ctx_b += n_b, once per step.
// The same copy kernel, with all K slots and no advance, installs a view's
// block K/V rows into the cache tail (orthrus_write_block).
// The advance runs as its own launch after the copies on the same stream, so
// every copy reads the old length.
#include "common.cuh"
#include "kernels.h"

namespace orthrus {

__device__ __forceinline__ bool commit_valid(const CommitArgs &p, int b, int *n_out,
                                             int *ctx_out)
{
    const int c = p.ctx_lens[b];
    if (c < 0 || (int64_t)c + p.K > p.S_max) return false;
    if (p.all_rows) {                    // block install: every slot, no acceptance
        *n_out = p.K;
        *ctx_out = c;
        return true;
    }
    const int a = p.accepted[b];
    if (a < 0 || a > p.K) return false;
    *n_out = a + 1 < p.K ? a + 1 : p.K;
    *ctx_out = c;
    return true;
}

__global__ void __launch_bounds__(256) kv_copy_kernel(CommitArgs p)
{
    const int layer = blockIdx.z;
    const int b = blockIdx.y;
    int n, c;
    if (!commit_valid(p, b, &n, &c)) {              // flagged by the advance kernel
        if (p.all_rows && layer == 0 && blockIdx.x == 0 && threadIdx.x == 0)
            raise_status(p.status, ORTHRUS_STATUS_CAPACITY);
        return;
    }
    // 16-byte units per row and the units this sequence moves per tensor
    const int row_units = p.D * p.elem_bytes / 16;
    const int64_t units = (int64_t)n * p.Hkv * row_units;
    const uint4 *kb = static_cast<const uint4 *>(p.k_blks[layer]);
    const uint4 *vb = static_cast<const uint4 *>(p.v_blks[layer]);
    uint4 *kc = static_cast<uint4 *>(p.k_caches[layer]);
    uint4 *vc = static_cast<uint4 *>(p.v_caches[layer]);
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units;
         u += (int64_t)gridDim.x * blockDim.x) {
        const int x = (int)(u % row_units);
        const int64_t sr = u / row_units;          // (slot, g) with g fastest
        const int g = (int)(sr % p.Hkv);
        const int slot = (int)(sr / p.Hkv);
        const size_t src = (((size_t)b * p.K + slot) * p.Hkv + g) * row_units + x;
        const size_t dst = (((size_t)b * p.Hkv + g) * p.S_max + c + slot) * row_units + x;
        kc[dst] = kb[src];
        vc[dst] = vb[src];
    }
}

__global__ void kv_advance_kernel(CommitArgs p)
{
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= p.B) return;
    int n, c;
    if (!commit_valid(p, b, &n, &c)) {
        const int a = p.accepted[b];
        raise_status(p.status, (a < 0 || a > p.K) ? ORTHRUS_STATUS_ACCEPT
                                                  : ORTHRUS_STATUS_CAPACITY);
        return;
    }
    p.ctx_lens[b] = c + n;
}

cudaError_t launch_kv_commit(const CommitArgs &p, cudaStream_t st)
{
    if (p.copy) {
        const int row_units = p.D * p.elem_bytes / 16;
        const int64_t max_units = (int64_t)p.K * p.Hkv * row_units;
        int gx = (int)((max_units + 255) / 256);
        if (gx > 64) gx = 64;
        dim3 grid(gx, p.B, p.num_layers);
        kv_copy_kernel<<<grid, 256, 0, st>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.all_rows) return cudaSuccess;            // block install never advances
    kv_advance_kernel<<<(p.B + 127) / 128, 128, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace orthrus

// Greedy consensus (Orthrus technical summary, gist.science, section 2.3
// "consensus and commitment"): r_i = argmax of AR logits row i; the accepted
// length a is the number of leading slots whose proposal equals r_i; the next
// anchor is r_min(a, K-1).
//
// Two launches:
//   1. argmax_partial: grid (splits, B*K).  Each CTA streams one vocabulary
//      chunk of one row with 16-byte loads and reduces it to one packed 64-bit
//      key (order-preserving value bits << 32 | ~index), so a plain unsigned
//      max picks the largest value and, among equals, the lowest index.
//   2. prefix_match: one CTA per sequence reduces the chunk keys of its K rows
//      and runs the left-to-right match.
// Ordering reading: NaN ranks above every number (first NaN wins), +0 == -0.
#include "common.cuh"
#include "kernels.h"

namespace orthrus {

__device__ __forceinline__ uint32_t order_bits(float x)
{
    if (x != x) return 0xFFFFFFFFu;               // NaN above everything
    uint32_t u = __float_as_uint(x);
    if (x == 0.f) u = 0u;                          // -0 ties with +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long pack_key(float x, int idx)
{
    return ((unsigned long long)order_bits(x) << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)idx);
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b)
{
    return a > b ? a : b;
}

__device__ __forceinline__ unsigned long long warp_max64(unsigned long long v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = umax64(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

constexpr int kArgmaxThreads = 256;

__global__ void __launch_bounds__(kArgmaxThreads) argmax_partial_kernel(ConsensusArgs p)
{
    const int split = blockIdx.x;
    const int row = blockIdx.y;
    const int lo = split * p.chunk;
    int hi = lo + p.chunk;
    if (hi > p.V) hi = p.V;
    const float *x = p.logits + (size_t)row * p.V;
    unsigned long long best = 0ull;
    if ((p.V & 3) == 0 && (p.chunk & 3) == 0) {
        const float4 *x4 = reinterpret_cast<const float4 *>(x);
        const int lo4 = lo >> 2, hi4 = hi >> 2;
        int j = lo4 + threadIdx.x;
        // two independent loads in flight per thread per iteration
        for (; j + kArgmaxThreads < hi4; j += 2 * kArgmaxThreads) {
            const float4 a = __ldcs(x4 + j);
            const float4 b = __ldcs(x4 + j + kArgmaxThreads);
            const int ia = 4 * j, ib = 4 * (j + kArgmaxThreads);
            best = umax64(best, pack_key(a.x, ia));
            best = umax64(best, pack_key(a.y, ia + 1));
            best = umax64(best, pack_key(a.z, ia + 2));
            best = umax64(best, pack_key(a.w, ia + 3));
            best = umax64(best, pack_key(b.x, ib));
            best = umax64(best, pack_key(b.y, ib + 1));
            best = umax64(best, pack_key(b.z, ib + 2));
            best = umax64(best, pack_key(b.w, ib + 3));
        }
        for (; j < hi4; j += kArgmaxThreads) {
            const float4 a = __ldcs(x4 + j);
            const int ia = 4 * j;
            best = umax64(best, pack_key(a.x, ia));
            best = umax64(best, pack_key(a.y, ia + 1));
            best = umax64(best, pack_key(a.z, ia + 2));
            best = umax64(best, pack_key(a.w, ia + 3));
        }
    } else {
        for (int j = lo + threadIdx.x; j < hi; j += kArgmaxThreads)
            best = umax64(best, pack_key(__ldcs(x + j), j));
    }
    best = warp_max64(best);
    __shared__ unsigned long long red[kArgmaxThreads / 32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = best;
    __syncthreads();
    if (threadIdx.x < 32) {
        unsigned long long v = threadIdx.x < kArgmaxThreads / 32 ? red[threadIdx.x] : 0ull;
        v = warp_max64(v);
        if (threadIdx.x == 0) p.ws[(size_t)row * p.splits + split] = v;
    }
}

__global__ void __launch_bounds__(256) prefix_match_kernel(ConsensusArgs p)
{
    const int b = blockIdx.x;
    __shared__ int32_t r[ORTHRUS_MAX_BLOCK];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    for (int i = warp; i < p.K; i += blockDim.x >> 5) {
        const unsigned long long *w = p.ws + ((size_t)b * p.K + i) * p.splits;
        unsigned long long v = 0ull;
        for (int s = lane; s < p.splits; s += 32) v = umax64(v, w[s]);
        v = warp_max64(v);
        if (lane == 0) r[i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int a = 0;
        while (a < p.K && p.proposed[(size_t)b * p.K + a] == r[a]) ++a;
        p.accepted[b] = a;
        p.next_token[b] = r[a < p.K ? a : p.K - 1];
    }
    if (p.argmax_out)
        for (int i = threadIdx.x; i < p.K; i += blockDim.x) p.argmax_out[(size_t)b * p.K + i] = r[i];
}

cudaError_t launch_consensus(const ConsensusArgs &p, cudaStream_t st)
{
    dim3 g1(p.splits, p.B * p.K);
    argmax_partial_kernel<<<g1, kArgmaxThreads, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prefix_match_kernel<<<p.B, 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace orthrus

// CUDA-core (SIMT) dual-view attention and the split-KV combine.
//
// The SIMT kernel covers what the tensor-core kernel does not: fp32 inputs
// (tf32 tensor cores would miss the accuracy bar) and bf16 shapes other than
// head_dim 128 with G*K <= 128.  One warp owns one query row at a time and
// walks its keys with an online softmax; lanes split the head dimension.
//
// Masks (Orthrus technical summary, gist.science, sections 2.2 and 2.3):
// DIFF (M_diff) row i sees keys [0, C+K); AR row i sees keys [0, C+i].
#include "common.cuh"
#include "kernels.h"

namespace orthrus {

template <typename T, int DPL>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs p)
{
    const Decomp d = make_decomp(p.ctx_lens, p.B, p.Hkv, p.K, p.S_max, gridDim.x,
                                 p.min_keys);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int b = 0; b < p.B; ++b)
            if (seg_len(p.ctx_lens, b, p.K, p.S_max) == 0)
                raise_status(p.status, ORTHRUS_STATUS_CAPACITY);
    }
    if (d.W == 0 || (int)blockIdx.x >= d.P) return;

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int G = p.Hq / p.Hkv;
    const int rows = G * p.K;
    const T *q = static_cast<const T *>(p.q);
    const T *kc = static_cast<const T *>(p.k_cache);
    const T *vc = static_cast<const T *>(p.v_cache);

    PieceIter it(p.ctx_lens, p.B, p.Hkv, p.K, p.S_max, d, blockIdx.x);
    Piece pc;
    while (it.next(pc)) {
        const int C = pc.len - p.K;
        const bool sole = (pc.a == 0 && pc.e == pc.len);
        const int slot = blockIdx.x + pc.s;
        const T *kseg = kc + ((size_t)p.cache_seq(pc.b) * p.Hkv + pc.g) * p.S_max * p.D;
        const T *vseg = vc + ((size_t)p.cache_seq(pc.b) * p.Hkv + pc.g) * p.S_max * p.D;
        for (int r = warp; r < rows; r += nwarps) {
            const int i = r / G;
            const int h = pc.g * G + (r % G);
            const T *qr = q + ((p.q_row0(pc.b) + i) * p.Hq + h) * p.D;
            float qv[DPL], o[DPL];
#pragma unroll
            for (int t = 0; t < DPL; ++t) {
                qv[t] = to_f32(qr[lane + 32 * t]) * p.scale_log2;
                o[t] = 0.f;
            }
            const int lim = p.view == ORTHRUS_DIFF ? pc.len : C + i + 1;
            const int jend = pc.e < lim ? pc.e : lim;
            float m = -INFINITY, l = 0.f;
            for (int j = pc.a; j < jend; ++j) {
                const T *kr = kseg + (size_t)j * p.D;
                float sdot = 0.f;
#pragma unroll
                for (int t = 0; t < DPL; ++t) sdot += qv[t] * to_f32(kr[lane + 32 * t]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    sdot += __shfl_xor_sync(0xffffffffu, sdot, off);
                const float mn = fmaxf(m, sdot);
                const float corr = exp2f(m - mn);
                const float pj = exp2f(sdot - mn);
                l = l * corr + pj;
                const T *vr = vseg + (size_t)j * p.D;
#pragma unroll
                for (int t = 0; t < DPL; ++t) o[t] = o[t] * corr + pj * to_f32(vr[lane + 32 * t]);
                m = mn;
            }
            const float inv = l > 0.f ? 1.f / l : 0.f;
            if (sole) {
                float *orow = p.out + ((p.q_row0(pc.b) + i) * p.Hq + h) * p.D;
#pragma unroll
                for (int t = 0; t < DPL; ++t) orow[lane + 32 * t] = o[t] * inv;
            } else {
                float *orow = p.ws_o + ((size_t)slot * rows + r) * p.D;
#pragma unroll
                for (int t = 0; t < DPL; ++t) orow[lane + 32 * t] = o[t] * inv;
                if (lane == 0)
                    p.ws_lse[(size_t)slot * lse_pitch(rows) + r] = l > 0.f ? m + log2f(l) : -INFINITY;
            }
        }
    }
}

// Combine: for every segment covered by more than one CTA, merge the partials
// with weights 2^(lse_s - max lse) / sum.  One warp per output row; each lane
// owns float4 columns, so every split contributes one coalesced row read per
// warp.  The split weights are computed once per row into shared memory.
constexpr int kCombineWarps = 8;

__global__ void __launch_bounds__(kCombineWarps * 32) attn_combine_kernel(AttnArgs p, int grid_main)
{
    extern __shared__ float wsm[];         // [kCombineWarps][max splits]
    // programmatic dependent launch: start early, read partials only after the
    // attention kernel (and everything before it) has completed
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int s = blockIdx.x;              // segment
    const int b = s / p.Hkv, g = s % p.Hkv;
    const Decomp d = make_decomp(p.ctx_lens, p.B, p.Hkv, p.K, p.S_max, grid_main, p.min_keys);
    if (d.W == 0) return;
    int len;
    const int64_t s0 = seg_start(p.ctx_lens, b, g, p.Hkv, p.K, p.S_max, &len);
    if (len == 0) return;
    const int c_lo = cta_of(d, s0);
    const int c_hi = cta_of(d, s0 + len - 1);
    if (c_lo == c_hi) return;              // written directly by its only CTA
    const int n = c_hi - c_lo + 1;

    const int G = p.Hq / p.Hkv;
    const int rows = G * p.K;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    float *wv = wsm + warp * (grid_main + 1);
    const int r = blockIdx.y * kCombineWarps + warp;
    if (r >= rows) return;
    const int lp = lse_pitch(rows);
    const float *lse = p.ws_lse + (size_t)(c_lo + s) * lp + r;
    float M = -INFINITY;
    for (int c = lane; c < n; c += 32) M = fmaxf(M, lse[(size_t)c * lp]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float wsum = 0.f;
    for (int c = lane; c < n; c += 32) {
        const float l = lse[(size_t)c * lp];
        const float wc = l == -INFINITY ? 0.f : exp2f(l - M);
        wv[c] = wc;
        wsum += wc;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    __syncwarp();
    const float inv = 1.f / wsum;
    const int i = r / G;
    const int h = g * G + (r % G);
    float4 *orow = reinterpret_cast<float4 *>(p.out + ((p.q_row0(b) + i) * p.Hq + h) * p.D);
    const float4 *src = reinterpret_cast<const float4 *>(p.ws_o + ((size_t)(c_lo + s) * rows + r) * p.D);
    const size_t stride4 = (size_t)rows * p.D / 4;          // one split further
    for (int d4 = lane; d4 < p.D / 4; d4 += 32) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        int c = 0;
        for (; c + 4 <= n; c += 4) {
            float4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = __ldcg(src + (size_t)(c + u) * stride4 + d4);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float wc = wv[c + u];
                acc.x += wc * v[u].x;
                acc.y += wc * v[u].y;
                acc.z += wc * v[u].z;
                acc.w += wc * v[u].w;
            }
        }
        for (; c < n; ++c) {
            const float4 v = __ldcg(src + (size_t)c * stride4 + d4);
            const float wc = wv[c];
            acc.x += wc * v.x;
            acc.y += wc * v.y;
            acc.z += wc * v.z;
            acc.w += wc * v.w;
        }
        orow[d4] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
}

template <typename T>
static cudaError_t launch_simt_t(const AttnArgs &p, int grid, cudaStream_t st)
{
    const int dpl = p.D / 32;
    dim3 blk(256);
    switch (dpl) {
#define ORTHRUS_CASE(N) \
    case N: attn_simt_kernel<T, N><<<grid, blk, 0, st>>>(p); break;
        ORTHRUS_CASE(1) ORTHRUS_CASE(2) ORTHRUS_CASE(3) ORTHRUS_CASE(4)
        ORTHRUS_CASE(5) ORTHRUS_CASE(6) ORTHRUS_CASE(7) ORTHRUS_CASE(8)
#undef ORTHRUS_CASE
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_attn_simt(const AttnArgs &p, int grid, cudaStream_t st)
{
    cudaError_t e = p.dtype == ORTHRUS_F32 ? launch_simt_t<float>(p, grid, st)
                                           : launch_simt_t<__nv_bfloat16>(p, grid, st);
    if (e != cudaSuccess) return e;
    return launch_attn_combine(p, grid, st);
}

cudaError_t launch_attn_combine(const AttnArgs &p, int grid_main, cudaStream_t st)
{
    const int rows = (p.Hq / p.Hkv) * p.K;
    dim3 grid(p.B * p.Hkv, (rows + kCombineWarps - 1) / kCombineWarps);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kCombineWarps * 32);
    cfg.dynamicSmemBytes = (size_t)kCombineWarps * (grid_main + 1) * sizeof(float);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_combine_kernel, p, grid_main);
}

}  // namespace orthrus

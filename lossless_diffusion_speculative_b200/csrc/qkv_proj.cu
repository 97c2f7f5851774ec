// The block's QKV projection fused with the cache-tail write, for sm_100a.
//
// What it computes (Orthrus technical summary, gist.science, section 2.3:
// "parallel projection" -- the diffusion head projects the anchor and K-1
// masks in one forward pass -- and "structural verification" -- the filled
// block runs through the frozen AR head; section 2.1: both views attend over
// one shared KV cache): for one layer and one view, with x the block's hidden
// states after the layer's input norm and token row t = b * K + i,
//     q[b, i, h, :]               = W_q[h*D : (h+1)*D, :] x[t]
//     k_cache[b, g, ctx_b + i, :] = W_k[g*D : (g+1)*D, :] x[t]
//     v_cache[b, g, ctx_b + i, :] = W_v[g*D : (g+1)*D, :] x[t]
// each fp32 sum rounded to bf16 (nearest, ties to even).  The view's block
// keys and values land directly in the cache rows its attention reads,
// [ctx_b, ctx_b + K): no staging buffer and no separate install copy.  The
// model-specific elementwise steps between projection and attention (Qwen3's
// per-head RMSNorm of q and k, rotary position embedding) are not on the pages
// and not part of this call.
//
// The projections are the skinny GEMM of skinny_gemm.cuh over the stacked
// weight rows [W_q; W_k; W_v] (three segments); with fewer 128-row tiles than
// half the SMs (Qwen3-8B: 48 tiles) the hidden dimension is split over
// several CTAs per tile and the last split sums the fp32 partials.  Epilogue: a warp's 32 lanes
// hold 32 consecutive output features of one token row, so every bf16 store of
// the warp is 64 contiguous bytes.  A sequence without room for its block
// (ctx_b < 0 or ctx_b + K > S_max) is skipped and raises
// ORTHRUS_STATUS_CAPACITY.
#include <cuda_bf16.h>

#include <mutex>

#include "skinny_gemm.cuh"

namespace orthrus {
namespace qkv {

using namespace sm100;

// Shared-memory table of the epilogue: per token row t = b * K + i, the cache
// row of its key and value in KV head 0, (b * Hkv) * S_max + ctx_b + i, or -1
// when sequence b has no room for its block.
constexpr uint32_t kTokBytes = kMaxLmRows * sizeof(long long);

// The epilogue's store of one 32-token group of one output feature (a warp's
// 32 lanes hold 32 consecutive features: every store of the warp is 64
// contiguous bytes).
struct QkvStore {
    __nv_bfloat16 *q, *kc, *vc;
    const long long *tokrow;
    int qrow, D, S_max, BK;
    __device__ __forceinline__ void operator()(int row, int seg, int seg_lo, bool valid, int c0,
                                               const uint32_t (&x)[32]) const
    {
        if (!valid) return;
        const int f = row - seg_lo;                                   // feature in its segment
        if (seg == 0) {
            __nv_bfloat16 *dst = q + f;
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (c0 + c < BK) dst[(size_t)(c0 + c) * qrow] = __float2bfloat16_rn(__uint_as_float(x[c]));
        } else {
            const int g = f / D, d = f - g * D;                       // KV head, dim
            __nv_bfloat16 *dst = (seg == 1 ? kc : vc) + (size_t)g * S_max * D + d;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                if (c0 + c < BK) {
                    const long long r = tokrow[c0 + c];
                    if (r >= 0) dst[r * D] = __float2bfloat16_rn(__uint_as_float(x[c]));
                }
            }
        }
    }
};

template <int CPS, bool SPLITK>
__global__ void __launch_bounds__(sg::kThreads, 1)
    qkv_proj_kernel(const __grid_constant__ sg::Maps mp, const QkvArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    const sg::Shape &sp = p.shape;
    sg::Smem sm;
    pdl_trigger();
    sg::prologue(sm, smem_raw, sp, CPS, kTokBytes, mp);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sg::tmem_base(sm);

    // ---- everything below may read what earlier kernels wrote
    pdl_wait();
    const int cid = blockIdx.x, grid = gridDim.x;
    if (warp < 4) {
        long long *tokrow = reinterpret_cast<long long *>(sm.extra());
        for (int t = threadIdx.x; t < sp.BK; t += 128) {
            const int b = t / p.K, i = t - b * p.K;
            const int c = p.ctx_lens[b];
            const bool room = c >= 0 && (int64_t)c + p.K <= p.S_max;
            if (!room && i == 0 && cid == 0) raise_status(sp.status, ORTHRUS_STATUS_CAPACITY);
            tokrow[t] = room ? (long long)b * p.Hkv * p.S_max + c + i : -1ll;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        QkvStore st;
        st.q = static_cast<__nv_bfloat16 *>(p.q_out);
        st.kc = static_cast<__nv_bfloat16 *>(p.k_cache);
        st.vc = static_cast<__nv_bfloat16 *>(p.v_cache);
        st.tokrow = tokrow;
        st.qrow = p.Hq * p.D;
        st.D = p.D;
        st.S_max = p.S_max;
        st.BK = sp.BK;
        sg::epilogue_tiles<SPLITK>(sm, sp, cid, grid, tmem, CPS, st);
    } else if (warp == 4) {
        if (lane == 0) sg::producer<CPS>(sm, sp, mp, cid, grid);
        __syncwarp();
    } else {
        if (lane == 0) sg::mma_issuer<CPS>(sm, sp, cid, grid, tmem);
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    sg::tmem_free(tmem);
}

}  // namespace qkv

namespace {

constexpr int kMaxDevices = 64;
std::once_flag g_qkv_once[kMaxDevices];
bool g_qkv_ok[kMaxDevices];

bool qkv_smem_ready(int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::call_once(g_qkv_once[dev], [dev] {
        const int lim = 226 * 1024;            // (room for the kernels' few bytes of static shared memory)
        const cudaFuncAttribute at = cudaFuncAttributeMaxDynamicSharedMemorySize;
        g_qkv_ok[dev] = cudaFuncSetAttribute(qkv::qkv_proj_kernel<1, false>, at, lim) == cudaSuccess &&
                        cudaFuncSetAttribute(qkv::qkv_proj_kernel<2, false>, at, lim) == cudaSuccess &&
                        cudaFuncSetAttribute(qkv::qkv_proj_kernel<4, false>, at, lim) == cudaSuccess &&
                        cudaFuncSetAttribute(qkv::qkv_proj_kernel<1, true>, at, lim) == cudaSuccess &&
                        cudaFuncSetAttribute(qkv::qkv_proj_kernel<2, true>, at, lim) == cudaSuccess &&
                        cudaFuncSetAttribute(qkv::qkv_proj_kernel<4, true>, at, lim) == cudaSuccess;
        if (!g_qkv_ok[dev]) cudaGetLastError();
    });
    return g_qkv_ok[dev];
}

}  // namespace

}  // namespace orthrus

using namespace orthrus;

namespace {

// Split-K plan: with fewer 128-row tiles than half the SMs, every tile's
// hidden dimension is split over ksplit CTAs (one unit each).
struct QkvPlan {
    int Np, cps, nst, ntiles, ksplit, grid;
    size_t part_bytes, total;
};

QkvPlan qkv_plan(int B, int K, int hidden, int Hq, int Hkv, int D, int sms)
{
    QkvPlan q;
    q.Np = sg::padded_n(B * K);
    sg::pipeline_of(q.Np, hidden / 64, &q.cps, &q.nst);
    const int rows[3] = {Hq * D, Hkv * D, Hkv * D};
    q.ntiles = 0;
    for (int r : rows) q.ntiles += (r + sg::kTileRows - 1) / sg::kTileRows;
    const int units = hidden / 64 / q.cps;
    q.ksplit = 1;
    if (2 * q.ntiles <= sms) {
        q.ksplit = sms / q.ntiles;
        if (q.ksplit > units) q.ksplit = units;
    }
    const int g16 = (Hq + 2 * Hkv) * D / 16;
    q.grid = q.ksplit > 1 ? q.ntiles * q.ksplit : (g16 < sms ? g16 : sms);
    const size_t ldp = (size_t)((q.Np + 31) & ~31);         // partial row stride (floats)
    q.part_bytes = q.ksplit > 1 ? (((size_t)q.ksplit * (Hq + 2 * Hkv) * D * ldp * 4 + 255) & ~(size_t)255) : 0;
    q.total = q.part_bytes + (((size_t)q.ntiles * 4 + 255) & ~(size_t)255);
    return q;
}

int qkv_sms()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

extern "C" size_t orthrus_qkv_workspace_size(int B, int K, int hidden, int Hq, int Hkv, int D)
{
    if (B <= 0 || K <= 0 || hidden <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || hidden % 64 != 0) return 0;
    if ((int64_t)B * K > kMaxLmRows) return 0;
    const int sms = qkv_sms();
    if (sms <= 0) return 0;
    return qkv_plan(B, K, hidden, Hq, Hkv, D, sms).total;
}

extern "C" int orthrus_qkv_project(const void *x, const void *w_q, const void *w_k, const void *w_v,
                                   const int32_t *ctx_lens, int B, int K, int hidden, int Hq, int Hkv,
                                   int D, int S_max, void *q_out, void *k_cache, void *v_cache,
                                   void *workspace, size_t workspace_bytes, int32_t *status, void *stream)
{
    if (!x || !w_q || !w_k || !w_v || !ctx_lens || !q_out || !k_cache || !v_cache) return ORTHRUS_ERR_ARG;
    if (B <= 0 || K <= 0 || hidden <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || S_max <= 0 || K > S_max)
        return ORTHRUS_ERR_ARG;
    if ((int64_t)B * K > kMaxLmRows || hidden % 64 != 0 || D % 16 != 0 || Hq % Hkv != 0)
        return ORTHRUS_ERR_UNSUPPORTED;
    if ((int64_t)(Hq + 2 * Hkv) * D >= (1ll << 31) || (int64_t)B * Hkv * S_max * D >= (1ll << 40))
        return ORTHRUS_ERR_UNSUPPORTED;
    const uintptr_t al = (uintptr_t)x | (uintptr_t)w_q | (uintptr_t)w_k | (uintptr_t)w_v | (uintptr_t)workspace;
    if (al & 15u) return ORTHRUS_ERR_ALIGN;
    int dev = 0, sms = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ORTHRUS_ERR_DEVICE;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (sms <= 0 || major != 10) return ORTHRUS_ERR_DEVICE;

    QkvArgs a;
    a.ctx_lens = ctx_lens;
    a.q_out = q_out;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.B = B;
    a.K = K;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = S_max;
    const QkvPlan qp = qkv_plan(B, K, hidden, Hq, Hkv, D, sms);
    if (!workspace || workspace_bytes < qp.total) return ORTHRUS_ERR_WORKSPACE;
    SkinnyShape &sp = a.shape;
    sp.nseg = 3;
    sp.seg_end[0] = Hq * D;
    sp.seg_end[1] = sp.seg_end[0] + Hkv * D;
    sp.seg_end[2] = sp.seg_end[1] + Hkv * D;
    sp.Hd = hidden;
    sp.BK = B * K;
    sp.Np = qp.Np;
    sp.nst = qp.nst;
    sp.halves = 1;
    sp.status = status;
    sp.ksplit = qp.ksplit;
    sp.ws_part = static_cast<float *>(workspace);
    sp.ws_count = reinterpret_cast<unsigned int *>(static_cast<char *>(workspace) + qp.part_bytes);
    const int cps = qp.cps;
    const sg::Layout L = sg::layout_of(sp.Np, sp.nst, cps, qkv::kTokBytes);

    sg::Maps mp;
    if (!sg::encode_w(mp, 0, w_q, Hq * D, hidden) || !sg::encode_w(mp, 1, w_k, Hkv * D, hidden) ||
        !sg::encode_w(mp, 2, w_v, Hkv * D, hidden) || !sg::encode_x(mp, x, B * K, hidden, sp.Np))
        return ORTHRUS_ERR_LAUNCH;
    if (!qkv_smem_ready(dev)) return ORTHRUS_ERR_LAUNCH;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(qp.grid);
    cfg.blockDim = dim3(sg::kThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const bool sk = qp.ksplit > 1;
    cudaError_t e;
    if (cps == 4)
        e = sk ? cudaLaunchKernelEx(&cfg, qkv::qkv_proj_kernel<4, true>, mp, a)
               : cudaLaunchKernelEx(&cfg, qkv::qkv_proj_kernel<4, false>, mp, a);
    else if (cps == 2)
        e = sk ? cudaLaunchKernelEx(&cfg, qkv::qkv_proj_kernel<2, true>, mp, a)
               : cudaLaunchKernelEx(&cfg, qkv::qkv_proj_kernel<2, false>, mp, a);
    else
        e = sk ? cudaLaunchKernelEx(&cfg, qkv::qkv_proj_kernel<1, true>, mp, a)
               : cudaLaunchKernelEx(&cfg, qkv::qkv_proj_kernel<1, false>, mp, a);
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

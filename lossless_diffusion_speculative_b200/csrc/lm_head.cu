// Fused AR LM head + vocabulary argmax + greedy consensus for sm_100a.
//
// What it computes (Orthrus technical summary, gist.science, section 2.3,
// "structural verification" and "consensus and commitment"): the frozen AR
// head scores all K block positions in one pass, logits[t, v] = <h_t, W_v> for
// token row t = b * K + i and vocabulary row v; r_t = argmax_v logits[t, v]
// (lowest index wins ties, NaN ranks above every number); then the greedy
// prefix match of orthrus_consensus: a_b = number of leading i with
// proposed[b, i] == r[b, i], next_b = r[b, min(a_b, K - 1)].
//
// The [B*K, V] logits are never written.  Each CTA owns a contiguous range of
// vocabulary rows (16-row granules split evenly over the grid) and reduces it
// to one packed (value, index) key per token row; keys combine across CTAs
// with a 64-bit atomic max in the workspace, and the last CTA to finish (a
// completion counter) runs the prefix match and clears the workspace.
//
// The logits are the skinny GEMM of skinny_gemm.cuh (the vocabulary rows of
// the weight are the MMA's M, the token rows its N).  Its epilogue: warps 0-3
// read each tile's accumulator from TMEM (thread = vocabulary row), pack each
// (value, row) into an order-preserving 64-bit key and reduce every token
// column over the 32 rows of the warp with a transpose butterfly (31
// exchanges), then over the 4 warps with a shared-memory atomic max.
#include <mutex>

#include "skinny_gemm.cuh"

namespace orthrus {
namespace lmh {

using namespace sm100;

// Order-preserving key of (value, index): a larger key is a larger value, or
// the same value at a lower index; NaN ranks above every number (the first NaN
// wins) and -0 equals +0.  Key 0 is below every real key.
__device__ __forceinline__ uint64_t argmax_key(float x, uint32_t idx)
{
    uint32_t u = __float_as_uint(x);
    if (x != x) {
        u = 0xFFFFFFFFu;
    } else {
        if (u == 0x80000000u) u = 0u;
        u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    return ((uint64_t)u << 32) | (uint32_t)~idx;
}

__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m)
{
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
    return ((uint64_t)hi << 32) | lo;
}

// Column maxima of a warp's 32 x 32 block of keys (k[c] = this lane's row,
// column c): after five exchange rounds lane l holds the maximum of column l.
// Each round splits the live columns in halves; the lane with bit h set keeps
// the upper half and sends the lower one to its partner.
__device__ __forceinline__ uint64_t column_max32(uint64_t (&k)[32], int lane)
{
#pragma unroll
    for (int n = 32; n > 1; n >>= 1) {
        const int h = n >> 1;
        const bool upper = lane & h;
#pragma unroll
        for (int j = 0; j < h; ++j) {
            const uint64_t send = upper ? k[j] : k[j + h];
            const uint64_t mine = upper ? k[j + h] : k[j];
            k[j] = umax64(mine, shfl_xor64(send, h));
        }
    }
    return k[0];
}

// The kernel's own shared memory: CTA keys [kMaxLmRows] u64, argmax rows
// [kMaxLmRows] int32, the last-CTA flag.
constexpr uint32_t kExtraBytes = kMaxLmRows * 8 + kMaxLmRows * 4 + 16;

template <int CPS, bool PAIR>
__global__ void __launch_bounds__(sg::kThreads, 1)
    lm_head_kernel(const __grid_constant__ sg::Maps mp, const LmHeadArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    const sg::Shape &sp = p.shape;
    sg::Smem sm;
    pdl_trigger();
    sg::prologue(sm, smem_raw, sp, CPS, kExtraBytes, mp);
    unsigned long long *ckeys = reinterpret_cast<unsigned long long *>(sm.extra());
    int *rbuf = reinterpret_cast<int *>(sm.extra() + kMaxLmRows * 8);
    volatile int *last_flag = reinterpret_cast<volatile int *>(sm.extra() + kMaxLmRows * 12);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BK = sp.BK;
    for (int t = threadIdx.x; t < BK; t += sg::kThreads) ckeys[t] = 0ull;
    if (threadIdx.x == 0) *last_flag = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sg::tmem_base(sm);

    // ---- everything below may read what earlier kernels wrote
    pdl_wait();
    const int cid = blockIdx.x, grid = gridDim.x;
    if (warp < 4) {
        sg::epilogue_tiles<false, PAIR>(sm, sp, cid, grid, tmem, CPS,
                           [&](int row, int, int, bool valid, int c0, const uint32_t (&x)[32]) {
                               uint64_t k[32];
#pragma unroll
                               for (int c = 0; c < 32; ++c)
                                   k[c] = valid && c0 + c < BK ? argmax_key(__uint_as_float(x[c]), (uint32_t)row)
                                                               : 0ull;
                               const uint64_t m = column_max32(k, lane);
                               if (c0 + lane < BK && m) atomicMax(ckeys + c0 + lane, (unsigned long long)m);
                           });
    } else if (warp == 4) {
        if (lane == 0) sg::producer<CPS, PAIR>(sm, sp, mp, cid, grid);
        __syncwarp();
    } else {
        if (lane == 0) sg::mma_issuer<CPS, PAIR>(sm, sp, cid, grid, tmem);
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    sg::tmem_free(tmem);
    if (*sm.abort_flag) return;

    // ---- combine across CTAs; the last CTA to finish runs the prefix match
    unsigned long long *gkeys = p.ws_keys;
    for (int t = threadIdx.x; t < BK; t += sg::kThreads)
        if (ckeys[t]) atomicMax(gkeys + t, ckeys[t]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *last_flag = atomicAdd(p.ws_done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!*last_flag) return;
    __threadfence();
    for (int t = threadIdx.x; t < BK; t += sg::kThreads) {
        const unsigned long long key = atomicExch(gkeys + t, 0ull);   // read and clear for the next call
        const int r = (int)~(uint32_t)key;
        rbuf[t] = r;
        if (p.argmax_out) p.argmax_out[t] = r;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < p.B; b += sg::kThreads) {
        int a = 0;
        while (a < p.K && p.proposed[b * p.K + a] == rbuf[b * p.K + a]) ++a;
        p.accepted[b] = a;
        p.next_token[b] = rbuf[b * p.K + (a < p.K ? a : p.K - 1)];
    }
    if (threadIdx.x == 0) *p.ws_done = 0u;
}

}  // namespace lmh

namespace {

int lm_sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

// The kernels' shared-memory limit, raised once per device (thread-safe) to
// the largest layout any call uses.
constexpr int kMaxDevices = 64;
std::once_flag g_smem_once[kMaxDevices];
bool g_smem_ok[kMaxDevices];

bool lm_smem_ready(int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::call_once(g_smem_once[dev], [dev] {
        const int lim = 226 * 1024;            // (room for the kernels' few bytes of static shared memory)
        const cudaFuncAttribute at = cudaFuncAttributeMaxDynamicSharedMemorySize;
        g_smem_ok[dev] = cudaFuncSetAttribute(lmh::lm_head_kernel<1, false>, at, lim) == cudaSuccess &&
                         cudaFuncSetAttribute(lmh::lm_head_kernel<2, false>, at, lim) == cudaSuccess &&
                         cudaFuncSetAttribute(lmh::lm_head_kernel<4, false>, at, lim) == cudaSuccess &&
                         cudaFuncSetAttribute(lmh::lm_head_kernel<1, true>, at, lim) == cudaSuccess &&
                         cudaFuncSetAttribute(lmh::lm_head_kernel<2, true>, at, lim) == cudaSuccess &&
                         cudaFuncSetAttribute(lmh::lm_head_kernel<4, true>, at, lim) == cudaSuccess;
        if (!g_smem_ok[dev]) cudaGetLastError();
    });
    return g_smem_ok[dev];
}

}  // namespace

}  // namespace orthrus

using namespace orthrus;

extern "C" {

size_t orthrus_lm_head_workspace_size(int B, int K)
{
    if (B <= 0 || K <= 0 || (int64_t)B * K > kMaxLmRows) return 0;
    return ((size_t)B * K * 8 + 16 + 255) & ~(size_t)255;
}

int orthrus_lm_head_consensus(const void *hidden, const void *lm_head, const int32_t *proposed, int B,
                              int K, int V, int Hd, int32_t *accepted_len, int32_t *next_token,
                              int32_t *argmax_out, void *workspace, size_t workspace_bytes,
                              int32_t *status, void *stream)
{
    if (!hidden || !lm_head || !proposed || !accepted_len || !next_token) return ORTHRUS_ERR_ARG;
    if (B <= 0 || K <= 0 || V <= 0 || Hd <= 0) return ORTHRUS_ERR_ARG;
    if ((int64_t)B * K > kMaxLmRows || Hd % 64 != 0) return ORTHRUS_ERR_UNSUPPORTED;
    const uintptr_t al = (uintptr_t)hidden | (uintptr_t)lm_head | (uintptr_t)workspace;
    if (al & 15u) return ORTHRUS_ERR_ALIGN;
    const size_t need = orthrus_lm_head_workspace_size(B, K);
    if (!workspace || workspace_bytes < need) return ORTHRUS_ERR_WORKSPACE;
    const int sms = lm_sm_count();
    if (sms <= 0) return ORTHRUS_ERR_DEVICE;
    int major = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return ORTHRUS_ERR_DEVICE;

    const int BK = B * K;
    LmHeadArgs a;
    a.proposed = proposed;
    a.accepted = accepted_len;
    a.next_token = next_token;
    a.argmax_out = argmax_out;
    a.ws_keys = static_cast<unsigned long long *>(workspace);
    a.ws_done = reinterpret_cast<unsigned int *>(static_cast<char *>(workspace) + (size_t)BK * 8);
    a.B = B;
    a.K = K;
    a.V = V;
    SkinnyShape &sp = a.shape;
    sp.nseg = 1;
    sp.seg_end[0] = sp.seg_end[1] = sp.seg_end[2] = V;
    sp.Hd = Hd;
    sp.BK = BK;
    sp.Np = sg::padded_n(BK);
    sp.status = status;
    sp.ksplit = 1;
    sp.ws_part = nullptr;
    sp.ws_count = nullptr;
    int cps = 1;
    // with 65-128 token rows every stage serves two 128-row weight tiles
    // (the token rows, as many bytes as a weight tile, are then loaded once per
    // two); fewer token rows keep four chunks per stage, more fill TMEM
    sp.halves = sp.Np > 64 && sp.Np <= 128 ? 2 : 1;
    sg::pipeline_of(sp.Np, Hd / 64, &cps, &sp.nst, sp.halves);
    const sg::Layout L = sg::layout_of(sp.Np, sp.nst, cps, lmh::kExtraBytes, sp.halves);

    sg::Maps mp;
    if (!sg::encode_w(mp, 0, lm_head, V, Hd) || !sg::encode_x(mp, hidden, BK, Hd, sp.Np))
        return ORTHRUS_ERR_LAUNCH;
    mp.w[1] = mp.w[2] = mp.w[0];
    mp.w16[1] = mp.w16[2] = mp.w16[0];
    if (!lm_smem_ready(dev)) return ORTHRUS_ERR_LAUNCH;
    const int V16 = (V + 15) / 16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(V16 < sms ? V16 : sms);
    cfg.blockDim = dim3(sg::kThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (sp.halves == 2)
        e = cps == 4   ? cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<4, true>, mp, a)
            : cps == 2 ? cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<2, true>, mp, a)
                       : cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<1, true>, mp, a);
    else
        e = cps == 4   ? cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<4, false>, mp, a)
            : cps == 2 ? cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<2, false>, mp, a)
                       : cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<1, false>, mp, a);
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

}  // extern "C"

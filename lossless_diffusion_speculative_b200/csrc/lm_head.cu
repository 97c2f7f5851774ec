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
// Per 128-row vocabulary tile (swap-AB: the weight rows are the MMA's M, the
// few token rows its N):
//   D[v, t] = sum_d W[v, d] h[t, d]   tcgen05.mma kind::f16, M = 128, N = Np
//       (token rows padded to 16, two MMAs of Np / 2 when Np > 256), K = 16;
//       A = W chunk [128 x 64] and B = h chunk [Np x 64], both K-major with
//       the 128-byte swizzle, staged by TMA in a ring of stages; a range's
//       last, partial tile is loaded in 16-row boxes
//   epilogue: warps 0-3 read D from TMEM (thread = vocabulary row), pack each
//       (value, row) into an order-preserving 64-bit key and reduce every
//       token column over the 32 rows of the warp with a transpose butterfly
//       (31 exchanges), then over the 4 warps with a shared-memory atomic max
// Roles: warps 0-3 epilogue, warp 4 TMA producer, warp 5 MMA issuer (and TMEM
// allocation).  Two TMEM accumulators (Np <= 256) let the epilogue of a tile
// overlap the MMAs of the next.  Every wait is bounded (ORTHRUS_STATUS_TIMEOUT).
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace orthrus {
namespace lmh {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kTileRows = 128;
constexpr int kChunk = 64;                         // hidden dims per box (128 bytes of bf16)

constexpr uint32_t kABytes = kTileRows * 128;      // 16 KiB
constexpr int kMaxStages = 12;
constexpr uint32_t kRingBudget = 200 * 1024;
constexpr int kTmemCols = 512;

enum : int {
    B_FULL = 0,
    B_EMPTY = B_FULL + kMaxStages,
    B_AFULL = B_EMPTY + kMaxStages,      // accumulator a holds a finished tile
    B_AEMPTY = B_AFULL + 2,              // accumulator a has been read (4 warps)
    B_DRAIN = B_AEMPTY + 2,
    B_COUNT
};

// Dynamic shared memory: [ring: stages x (A | B)] [barriers] [tmem addr, abort,
// last flag] [CTA keys: kMaxLmRows x u64] [argmax rows: kMaxLmRows x int32]
struct Layout {
    uint32_t stage_bytes, ring, bars, misc, keys, rbuf, total;
};

// A pipeline stage holds `cps` adjacent hidden chunks: every weight row then
// gives cps * 128 contiguous bytes per stage, which the memory system serves
// far better than 128-byte pieces 8 KiB apart (weight rows are Hd * 2 bytes).
__host__ __device__ inline Layout layout_of(int Np, int nst, int cps)
{
    Layout l;
    l.stage_bytes = (uint32_t)cps * (kABytes + (uint32_t)Np * 128u);
    l.ring = 0;
    l.bars = (uint32_t)nst * l.stage_bytes;
    l.misc = l.bars + B_COUNT * 8;
    l.keys = (l.misc + 16 + 15) & ~15u;
    l.rbuf = l.keys + kMaxLmRows * 8;
    l.total = l.rbuf + kMaxLmRows * 4 + 1024;      // + room to align the base to 1 KiB
    return l;
}

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
// Round `off` splits the live columns in halves; the lane with bit `off` set
// keeps the upper half and sends the lower one to its partner.
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

struct Smem {
    uint32_t base;
    uint8_t *ptr;
    Layout L;
    volatile int *abort_flag;
    __device__ __forceinline__ uint32_t bar(int i) const { return base + L.bars + 8u * i; }
    __device__ __forceinline__ uint32_t a_of(int st) const { return base + st * L.stage_bytes; }
    int cps;
    __device__ __forceinline__ uint32_t b_of(int st) const { return a_of(st) + cps * kABytes; }
};

// The CTA's vocabulary rows [lo, hi) and tile count.
struct Range {
    int lo, hi, ntile;
};

__device__ __forceinline__ Range range_of(int V, int cid, int grid)
{
    const int V16 = (V + 15) >> 4;
    const int q = V16 / grid, r = V16 - q * grid;
    const int g0 = cid * q + (cid * r) / grid, g1 = (cid + 1) * q + ((cid + 1) * r) / grid;
    Range rg;
    rg.lo = g0 * 16;
    rg.hi = g1 * 16 < V ? g1 * 16 : V;
    rg.ntile = rg.hi > rg.lo ? (rg.hi - rg.lo + kTileRows - 1) / kTileRows : 0;
    return rg;
}

template <int CPS>
__device__ __forceinline__ void producer(const Smem &sh, const LmHeadArgs &p, const Range &rg,
                                         const CUtensorMap *tw, const CUtensorMap *tw16,
                                         const CUtensorMap *th)
{
    const int nk = p.Hd / kChunk;
    const int half = p.Np > 256 ? p.Np / 2 : p.Np;
    // (every CTA sweeps the hidden dimension in the same order, so equal weight
    // rows give bit-equal logits and exact ties resolve to the lower index)
    const uint64_t pol_w = make_policy_evict_first(), pol_h = make_policy_evict_last();
    uint32_t it = 0;
    bool ok = true;
    for (int t = 0; t < rg.ntile && ok; ++t) {
        const int r0 = rg.lo + t * kTileRows;
        const int nrows = rg.hi - r0 < kTileRows ? rg.hi - r0 : kTileRows;
        const int nb16 = (nrows + 15) >> 4;
        const uint32_t a_bytes = nrows == kTileRows ? kABytes : (uint32_t)nb16 * 16u * 128u;
        for (int ks = 0; ks < nk / CPS; ++ks, ++it) {
            const int st = it % p.nst;
            const uint32_t n = it / p.nst;
            if (n > 0 && !wait_bar(sh.bar(B_EMPTY + st), (n - 1) & 1, sh.abort_flag, p.status)) {
                ok = false;
                break;
            }
            const uint32_t full = sh.bar(B_FULL + st);
            mbar_expect_tx(full, CPS * (a_bytes + (uint32_t)p.Np * 128u));
            // (the stage's chunks are adjacent in every weight row: issued back to back)
#pragma unroll
            for (int j = 0; j < CPS; ++j) {
                const int kc = ks * CPS + j;
                const uint32_t a = sh.a_of(st) + j * kABytes;
                if (nrows == kTileRows) {
                    tma_load_2d_hint(a, tw, full, kc * kChunk, r0, pol_w);
                } else {
                    for (int q = 0; q < nb16; ++q)
                        tma_load_2d_hint(a + q * 2048u, tw16, full, kc * kChunk, r0 + 16 * q, pol_w);
                }
                const uint32_t b = sh.b_of(st) + j * (uint32_t)p.Np * 128u;
                tma_load_2d_hint(b, th, full, kc * kChunk, 0, pol_h);
                if (half != p.Np) tma_load_2d_hint(b + (uint32_t)half * 128u, th, full, kc * kChunk, half, pol_h);
            }
        }
    }
    if (!ok) {                       // abort: let every copy already issued land
        for (int st = 0; st < p.nst; ++st) {
            const uint32_t fills = it / p.nst + ((uint32_t)st < it % p.nst ? 1u : 0u);
            if (fills) wait_bar_quiet(sh.bar(B_FULL + st), (fills - 1) & 1);
        }
    }
}

template <int CPS>
__device__ __forceinline__ void mma_issuer(const Smem &sh, const LmHeadArgs &p, const Range &rg, uint32_t tmem)
{
    const int nk = p.Hd / kChunk;
    const int nacc = 2 * p.Np <= kTmemCols ? 2 : 1;
    const bool split = p.Np > 256;
    const int n_mma = split ? p.Np / 2 : p.Np;
    const uint32_t idesc = instr_desc(128, n_mma, false);
    uint32_t it = 0;
    bool ok = true;
    for (int t = 0; t < rg.ntile && ok; ++t) {
        const int acc = t % nacc;
        if (t >= nacc && !wait_bar(sh.bar(B_AEMPTY + acc), (t / nacc - 1) & 1, sh.abort_flag, p.status)) {
            ok = false;
            break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * p.Np);
        for (int ks = 0; ks < nk / CPS; ++ks, ++it) {
            const int st = it % p.nst;
            if (!wait_bar(sh.bar(B_FULL + st), (it / p.nst) & 1, sh.abort_flag, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < CPS; ++j) {
                const uint32_t b = sh.b_of(st) + j * (uint32_t)p.Np * 128u;
                const uint64_t ad = smem_desc(sh.a_of(st) + j * kABytes, 16, 1024);
                const uint64_t bd = smem_desc(b, 16, 1024);
                const uint64_t bd2 = smem_desc(b + (uint32_t)n_mma * 128u, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {        // 16 hidden dims (32 bytes) per MMA
                    const uint32_t on = (ks | j | kk) ? 1u : 0u;
                    tc_mma_ss(d, ad + 2 * kk, bd + 2 * kk, idesc, on);
                    if (split) tc_mma_ss(d + (uint32_t)n_mma, ad + 2 * kk, bd2 + 2 * kk, idesc, on);
                }
            }
            tc_commit(sh.bar(B_EMPTY + st));
        }
        if (ok) tc_commit(sh.bar(B_AFULL + acc));
    }
    if (!ok) {
        tc_commit(sh.bar(B_DRAIN));
        wait_bar_quiet(sh.bar(B_DRAIN), 0);
    }
}

// Warps 0-3.  Returns false after an abort.
__device__ __forceinline__ bool epilogue(const Smem &sh, const LmHeadArgs &p, const Range &rg, uint32_t tmem)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nacc = 2 * p.Np <= kTmemCols ? 2 : 1;
    const int BK = p.B * p.K;
    unsigned long long *ckeys = reinterpret_cast<unsigned long long *>(sh.ptr + sh.L.keys);
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    for (int t = 0; t < rg.ntile; ++t) {
        const int acc = t % nacc;
        if (!wait_bar(sh.bar(B_AFULL + acc), (t / nacc) & 1, sh.abort_flag, p.status)) return false;
        tc_fence_after();
        const int v = rg.lo + t * kTileRows + warp * 32 + lane;
        const bool valid = v < rg.hi;
        for (int c0 = 0; c0 < p.Np; c0 += 32) {
            uint32_t x[32];
            tmem_ld32(lane_base + (uint32_t)(acc * p.Np + c0), x);
            tmem_wait_ld();
            uint64_t k[32];
#pragma unroll
            for (int c = 0; c < 32; ++c)
                k[c] = valid && c0 + c < BK ? argmax_key(__uint_as_float(x[c]), (uint32_t)v) : 0ull;
            const uint64_t m = column_max32(k, lane);
            if (c0 + lane < BK && m) atomicMax(ckeys + c0 + lane, (unsigned long long)m);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sh.bar(B_AEMPTY + acc));
    }
    return true;
}

template <int CPS>
__global__ void __launch_bounds__(kThreads, 1)
    lm_head_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_w16,
                   const __grid_constant__ CUtensorMap tm_h, const LmHeadArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t aligned = (raw + 1023u) & ~1023u;
    Smem sh;
    sh.base = aligned;
    sh.ptr = smem_raw + (aligned - raw);
    sh.L = layout_of(p.Np, p.nst, p.cps);
    sh.cps = p.cps;
    sh.abort_flag = reinterpret_cast<volatile int *>(sh.ptr + sh.L.misc + 4);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(sh.ptr + sh.L.misc);
    volatile int *last_flag = reinterpret_cast<volatile int *>(sh.ptr + sh.L.misc + 8);
    unsigned long long *ckeys = reinterpret_cast<unsigned long long *>(sh.ptr + sh.L.keys);
    int *rbuf = reinterpret_cast<int *>(sh.ptr + sh.L.rbuf);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BK = p.B * p.K;

    // ---- prologue: touches nothing an earlier kernel in the stream may write
    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.nst; ++s) {
            mbar_init(sh.bar(B_FULL + s), 1);
            mbar_init(sh.bar(B_EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(sh.bar(B_AFULL + a), 1);
            mbar_init(sh.bar(B_AEMPTY + a), 4);
        }
        mbar_init(sh.bar(B_DRAIN), 1);
        *sh.abort_flag = 0;
        *last_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int t = threadIdx.x; t < BK; t += kThreads) ckeys[t] = 0ull;
    if (warp == 4 && lane == 0) {
        tma_prefetch(&tm_w);
        tma_prefetch(&tm_w16);
        tma_prefetch(&tm_h);
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         aligned + sh.L.misc),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- everything below may read what earlier kernels wrote
    pdl_wait();
    const Range rg = range_of(p.V, blockIdx.x, gridDim.x);
    if (warp < 4) {
        epilogue(sh, p, rg, tmem);                 // (an abort sets the CTA's abort flag)
    } else if (warp == 4) {
        if (lane == 0) producer<CPS>(sh, p, rg, &tm_w, &tm_w16, &tm_h);
        __syncwarp();
    } else {
        if (lane == 0) mma_issuer<CPS>(sh, p, rg, tmem);
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
    if (*sh.abort_flag) return;

    // ---- combine across CTAs; the last CTA to finish runs the prefix match
    unsigned long long *gkeys = p.ws_keys;
    for (int t = threadIdx.x; t < BK; t += kThreads)
        if (ckeys[t]) atomicMax(gkeys + t, ckeys[t]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *last_flag = atomicAdd(p.ws_done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!*last_flag) return;
    __threadfence();
    for (int t = threadIdx.x; t < BK; t += kThreads) {
        const unsigned long long key = atomicExch(gkeys + t, 0ull);   // read and clear for the next call
        const int r = (int)~(uint32_t)key;
        rbuf[t] = r;
        if (p.argmax_out) p.argmax_out[t] = r;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < p.B; b += kThreads) {
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

// The kernel's shared-memory limit, raised once per device (thread-safe) to
// the largest layout any call uses.
constexpr int kMaxDevices = 64;
std::once_flag g_smem_once[kMaxDevices];
bool g_smem_ok[kMaxDevices];

bool lm_smem_ready(int dev)
{
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::call_once(g_smem_once[dev], [dev] {
        const int lim = 227 * 1024;
        g_smem_ok[dev] =
            cudaFuncSetAttribute(lmh::lm_head_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim) ==
                cudaSuccess &&
            cudaFuncSetAttribute(lmh::lm_head_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim) ==
                cudaSuccess &&
            cudaFuncSetAttribute(lmh::lm_head_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim) ==
                cudaSuccess;
        if (!g_smem_ok[dev]) cudaGetLastError();
    });
    return g_smem_ok[dev];
}

// Chunks per stage: the most (4, 2 or 1) that divide the hidden size and
// still leave two stages in the ring; then as many stages as fit.
void lm_pipeline(int Np, int nk, int *cps, int *nst)
{
    *cps = 1;
    for (int c = 4; c >= 2; c >>= 1) {
        const uint32_t sb = (uint32_t)c * (lmh::kABytes + (uint32_t)Np * 128u);
        if (nk % c == 0 && 2 * sb <= lmh::kRingBudget) {
            *cps = c;
            break;
        }
    }
    const uint32_t sb = (uint32_t)*cps * (lmh::kABytes + (uint32_t)Np * 128u);
    const int n = (int)(lmh::kRingBudget / sb);
    *nst = n > lmh::kMaxStages ? lmh::kMaxStages : n;
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
    int Np = (BK + 15) & ~15;
    if (Np > 256) Np = (BK + 31) & ~31;
    LmHeadArgs a;
    a.proposed = proposed;
    a.accepted = accepted_len;
    a.next_token = next_token;
    a.argmax_out = argmax_out;
    a.ws_keys = static_cast<unsigned long long *>(workspace);
    a.ws_done = reinterpret_cast<unsigned int *>(static_cast<char *>(workspace) + (size_t)BK * 8);
    a.status = status;
    a.B = B;
    a.K = K;
    a.V = V;
    a.Hd = Hd;
    a.Np = Np;
    lm_pipeline(Np, Hd / 64, &a.cps, &a.nst);
    const lmh::Layout L = lmh::layout_of(Np, a.nst, a.cps);

    CUtensorMap tw, tw16, th;
    const uint64_t wdims[2] = {(uint64_t)Hd, (uint64_t)V}, wstr[1] = {(uint64_t)Hd * 2};
    const uint32_t wbox[2] = {64, 128}, wbox16[2] = {64, 16};
    const uint64_t hdims[2] = {(uint64_t)Hd, (uint64_t)BK}, hstr[1] = {(uint64_t)Hd * 2};
    const uint32_t hbox[2] = {64, (uint32_t)(Np > 256 ? Np / 2 : Np)};
    if (!encode_bf16_sw128(&tw, 2, lm_head, wdims, wstr, wbox) ||
        !encode_bf16_sw128(&tw16, 2, lm_head, wdims, wstr, wbox16) ||
        !encode_bf16_sw128(&th, 2, hidden, hdims, hstr, hbox))
        return ORTHRUS_ERR_LAUNCH;
    if (!lm_smem_ready(dev)) return ORTHRUS_ERR_LAUNCH;
    const int V16 = (V + 15) / 16;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(V16 < sms ? V16 : sms);
    cfg.blockDim = dim3(lmh::kThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = a.cps == 4   ? cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<4>, tw, tw16, th, a)
                          : a.cps == 2 ? cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<2>, tw, tw16, th, a)
                                       : cudaLaunchKernelEx(&cfg, lmh::lm_head_kernel<1>, tw, tw16, th, a);
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

}  // extern "C"

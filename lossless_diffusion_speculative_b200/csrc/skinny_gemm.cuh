// Skinny GEMM on the tcgen05 tensor cores, shared by the fused AR LM head
// (lm_head.cu) and the block's QKV projection (qkv_proj.cu):
//
//     D[r, t] = sum_d W[r, d] * X[t, d]
//
// for a handful of token rows t (the decode block: B * K <= 512) against many
// weight rows r streamed once from HBM.  Swap-AB: the weight rows are the
// MMA's M (128 per tile), the token rows its N (padded to 16, two MMAs of N/2
// when N > 256).  The weight rows may come in up to three stacked segments
// (q, k and v projections), each with its own tensor maps.
//
// Work split: the rows are cut into 16-row granules split evenly over the
// grid (one CTA per SM); a CTA walks its range in tiles of up to 128 rows that
// end at the range end or a segment end, loading a partial tile in 16-row
// boxes.  Per tile the hidden dimension is swept in 64-wide chunks (128 bytes
// of bf16, one 128-byte swizzle row), CPS adjacent chunks per pipeline stage:
// every weight row then gives CPS * 128 contiguous bytes per stage, which HBM
// serves far better than 128-byte pieces one weight row (several KiB) apart.
//
// Roles: warp 4 lane 0 TMA producer (weights evict-first, the reused token
// rows evict-last in L2), warp 5 lane 0 MMA issuer (and TMEM allocation),
// warps 0-3 the kernel's epilogue (thread = weight row of the tile, 32 token
// columns per TMEM load).  Two TMEM accumulators (N <= 256) let a tile's
// epilogue overlap the next tile's MMAs.  Every sweep uses the same chunk
// order, so equal weight rows give bit-equal results.  Every wait is bounded
// (ORTHRUS_STATUS_TIMEOUT, then drain and exit).
#pragma once

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace orthrus {
namespace sg {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kTileRows = 128;
constexpr int kChunk = 64;                         // hidden dims per box (128 bytes of bf16)
constexpr uint32_t kABytes = kTileRows * 128;      // 16 KiB: one 128-row chunk of weights
constexpr int kMaxStages = 12;
constexpr uint32_t kRingBudget = 200 * 1024;
constexpr int kTmemCols = 512;
constexpr int kMaxSegs = 3;
constexpr int kSumBatch = 4;                        // split-K partials loaded at once by the last split

enum : int {
    B_FULL = 0,
    B_EMPTY = B_FULL + kMaxStages,
    B_AFULL = B_EMPTY + kMaxStages,      // accumulator a holds a finished tile
    B_AEMPTY = B_AFULL + 2,              // accumulator a has been read (4 warps)
    B_DRAIN = B_AEMPTY + 2,
    B_COUNT
};

using Shape = SkinnyShape;
static_assert(kMaxSkinnySegs == kMaxSegs, "segments");
static_assert(kRingBudget + (B_COUNT * 8 + 32) + 2 * 1024 * 8 + 1024 <= 226 * 1024, "layouts fit the 226 KiB limit");

struct Maps {                            // one launch's tensor maps
    CUtensorMap w[kMaxSegs];             // box (64, 128) per weight segment
    CUtensorMap w16[kMaxSegs];           // box (64, 16): partial tiles
    CUtensorMap x;                       // token rows: box (64, Np) or (64, Np / 2)
};

// Dynamic shared memory: [ring: stages x (halves x CPS x A | CPS x X)]
// [barriers] [tmem address, abort flag, 2 spare words] [the kernel's own
// region].
struct Layout {
    uint32_t stage_bytes, bars, misc, extra, total;
};

__host__ __device__ inline Layout layout_of(int Np, int nst, int cps, uint32_t extra_bytes, int halves = 1)
{
    Layout l;
    l.stage_bytes = (uint32_t)cps * ((uint32_t)halves * kABytes + (uint32_t)Np * 128u);
    l.bars = (uint32_t)nst * l.stage_bytes;
    l.misc = l.bars + B_COUNT * 8;
    l.extra = (l.misc + 16 + 15) & ~15u;
    l.total = l.extra + extra_bytes + 1024;        // + room to align the base to 1 KiB
    return l;
}

struct Smem {
    uint32_t base;
    uint8_t *ptr;
    Layout L;
    int cps, halves;
    volatile int *abort_flag;
    __device__ __forceinline__ uint32_t bar(int i) const { return base + L.bars + 8u * i; }
    // weight chunks of half u of stage st (cps chunks of 16 KiB), then the token rows
    __device__ __forceinline__ uint32_t a_of(int st, int u = 0) const
    {
        return base + st * L.stage_bytes + (uint32_t)(u * cps) * kABytes;
    }
    __device__ __forceinline__ uint32_t b_of(int st) const { return a_of(st) + (uint32_t)(halves * cps) * kABytes; }
    __device__ __forceinline__ uint8_t *extra() const { return ptr + L.extra; }
};

// Hidden-chunk range of split s of ksplit over nk chunks (multiples of cps).
__host__ __device__ __forceinline__ int split_k0(int s, int ksplit, int nk, int cps)
{
    const int units = nk / cps;
    return cps * (s * units / ksplit);
}

// The tiles of CTA `cid`'s range, in order; identical in every role.  Without
// split-K the rows are cut into 16-row granules over the grid and walked in
// tiles of halves x 128 rows (two 128-row halves share each load of the
// token rows when halves = 2); with split-K CTA cid owns 128-row tile
// cid / ksplit (tiles counted per segment) and the hidden chunks [k_lo, k_hi)
// of split cid % ksplit.
struct TileIter {
    int r0, hi, height;
    int e0, e1, e2;                      // segment ends (unused segments end at the last)
    int k_lo, k_hi;                      // hidden chunks of every tile
    __device__ __forceinline__ TileIter(const Shape &sh, int cid, int grid, int cps)
    {
        e0 = sh.seg_end[0];
        e1 = sh.nseg > 1 ? sh.seg_end[1] : e0;
        e2 = sh.nseg > 2 ? sh.seg_end[2] : e1;
        height = kTileRows * sh.halves;
        const int nk = sh.Hd / kChunk;
        if (sh.ksplit > 1) {
            int t = cid / sh.ksplit;
            const int s = cid - (cid / sh.ksplit) * sh.ksplit;
            const int n0 = (e0 + kTileRows - 1) / kTileRows;
            const int n1 = (e1 - e0 + kTileRows - 1) / kTileRows;
            r0 = t < n0 ? t * kTileRows : t < n0 + n1 ? e0 + (t - n0) * kTileRows : e1 + (t - n0 - n1) * kTileRows;
            const int seg_hi = t < n0 ? e0 : t < n0 + n1 ? e1 : e2;
            hi = r0 + kTileRows < seg_hi ? r0 + kTileRows : seg_hi;
            if (r0 >= e2) r0 = hi = e2;
            k_lo = split_k0(s, sh.ksplit, nk, cps);
            k_hi = split_k0(s + 1, sh.ksplit, nk, cps);
            return;
        }
        const int rows = e2;
        const int g16 = (rows + 15) >> 4;
        const int q = g16 / grid, r = g16 - q * grid;
        r0 = 16 * (cid * q + (cid * r) / grid);
        hi = 16 * ((cid + 1) * q + ((cid + 1) * r) / grid);
        if (hi > rows) hi = rows;
        k_lo = 0;
        k_hi = nk;
    }
    // next tile [a, b) of weight segment `seg` (segment-local rows a - seg_lo)
    __device__ __forceinline__ bool next(int &a, int &b, int &seg, int &seg_lo)
    {
        if (r0 >= hi) return false;
        seg = r0 >= e0 ? (r0 >= e1 ? 2 : 1) : 0;
        seg_lo = seg == 0 ? 0 : seg == 1 ? e0 : e1;
        const int seg_hi = seg == 0 ? e0 : seg == 1 ? e1 : e2;
        a = r0;
        b = r0 + height;
        if (b > hi) b = hi;
        if (b > seg_hi) b = seg_hi;
        r0 = b;
        return true;
    }
};

template <int CPS, bool PAIR = false>
__device__ __forceinline__ void producer(const Smem &sm, const Shape &sp, const Maps &mp, int cid, int grid)
{
    const int nk = sp.Hd / kChunk;
    const int half = sp.Np > 256 ? sp.Np / 2 : sp.Np;
    const uint64_t pol_w = make_policy_evict_first(), pol_x = make_policy_evict_last();
    TileIter ti(sp, cid, grid, CPS);
    int a, b, seg, seg_lo;
    uint32_t it = 0;
    bool ok = true;
    (void)nk;
    while (ok && ti.next(a, b, seg, seg_lo)) {
        const int nrows = b - a, y0 = a - seg_lo;
        // rows of each 128-row weight half of the tile (the second may be short or empty)
        const int n0 = nrows < kTileRows ? nrows : kTileRows, n1 = nrows - n0;
        auto half_bytes = [](int n) -> uint32_t {
            return n == kTileRows ? kABytes : (uint32_t)((n + 15) >> 4) * 16u * 128u;
        };
        const uint32_t a_bytes = half_bytes(n0) + (n1 > 0 ? half_bytes(n1) : 0u);
        for (int ks = ti.k_lo / CPS; ks < ti.k_hi / CPS; ++ks, ++it) {
            const int st = it % sp.nst;
            const uint32_t n = it / sp.nst;
            if (n > 0 && !wait_bar(sm.bar(B_EMPTY + st), (n - 1) & 1, sm.abort_flag, sp.status)) {
                ok = false;
                break;
            }
            const uint32_t full = sm.bar(B_FULL + st);
            mbar_expect_tx(full, CPS * (a_bytes + (uint32_t)sp.Np * 128u));
            // (the stage's chunks are adjacent in every weight row: issued back to back)
#pragma unroll
            for (int j = 0; j < CPS; ++j) {
                const int kc = ks * CPS + j;
#pragma unroll
                for (int u = 0; u < (PAIR ? 2 : 1); ++u) {
                    const int nu = u == 0 ? n0 : n1;
                    if (nu <= 0) break;
                    const uint32_t dst = sm.a_of(st, u) + j * kABytes;
                    const int yu = y0 + kTileRows * u;
                    if (nu == kTileRows) {
                        tma_load_2d_hint(dst, &mp.w[seg], full, kc * kChunk, yu, pol_w);
                    } else {
                        for (int q = 0; q < ((nu + 15) >> 4); ++q)
                            tma_load_2d_hint(dst + q * 2048u, &mp.w16[seg], full, kc * kChunk, yu + 16 * q, pol_w);
                    }
                }
                const uint32_t xb = sm.b_of(st) + j * (uint32_t)sp.Np * 128u;
                tma_load_2d_hint(xb, &mp.x, full, kc * kChunk, 0, pol_x);
                if (half != sp.Np) tma_load_2d_hint(xb + (uint32_t)half * 128u, &mp.x, full, kc * kChunk, half, pol_x);
            }
        }
    }
    if (!ok) {                       // abort: let every copy already issued land
        for (int st = 0; st < sp.nst; ++st) {
            const uint32_t fills = it / sp.nst + ((uint32_t)st < it % sp.nst ? 1u : 0u);
            if (fills) wait_bar_quiet(sm.bar(B_FULL + st), (fills - 1) & 1);
        }
    }
}

template <int CPS, bool PAIR = false>
__device__ __forceinline__ void mma_issuer(const Smem &sm, const Shape &sp, int cid, int grid, uint32_t tmem)
{
    const int nk = sp.Hd / kChunk;
    const int acc_cols = sp.halves * sp.Np;              // one accumulator: every half's Np columns
    const int nacc = 2 * acc_cols <= kTmemCols ? 2 : 1;
    const bool split = sp.Np > 256;
    const int n_mma = split ? sp.Np / 2 : sp.Np;
    const uint32_t idesc = instr_desc(128, n_mma, false);
    TileIter ti(sp, cid, grid, CPS);
    int a, b, seg, seg_lo;
    uint32_t it = 0;
    bool ok = true;
    (void)nk;
    for (int t = 0; ok && ti.next(a, b, seg, seg_lo); ++t) {
        const int acc = t % nacc;
        if (t >= nacc && !wait_bar(sm.bar(B_AEMPTY + acc), (t / nacc - 1) & 1, sm.abort_flag, sp.status)) {
            ok = false;
            break;
        }
        tc_fence_after();
        const bool second = PAIR && b - a > kTileRows;      // a second weight half in this tile
        const uint32_t d = tmem + (uint32_t)(acc * acc_cols);
        const int ks0 = ti.k_lo / CPS;
        for (int ks = ks0; ks < ti.k_hi / CPS; ++ks, ++it) {
            const int st = it % sp.nst;
            if (!wait_bar(sm.bar(B_FULL + st), (it / sp.nst) & 1, sm.abort_flag, sp.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < CPS; ++j) {
                const uint32_t xb = sm.b_of(st) + j * (uint32_t)sp.Np * 128u;
                const uint64_t bd = smem_desc(xb, 16, 1024);
                const uint64_t bd2 = smem_desc(xb + (uint32_t)n_mma * 128u, 16, 1024);
#pragma unroll
                for (int u = 0; u < (PAIR ? 2 : 1); ++u) {  // (the token rows are shared by both halves)
                    if (u == 1 && !second) break;
                    const uint64_t ad = smem_desc(sm.a_of(st, u) + j * kABytes, 16, 1024);
                    const uint32_t du = d + (uint32_t)(u * sp.Np);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {    // 16 hidden dims (32 bytes) per MMA
                        const uint32_t on = ((ks - ks0) | j | kk) ? 1u : 0u;
                        tc_mma_ss(du, ad + 2 * kk, bd + 2 * kk, idesc, on);
                        if (split) tc_mma_ss(du + (uint32_t)n_mma, ad + 2 * kk, bd2 + 2 * kk, idesc, on);
                    }
                }
            }
            tc_commit(sm.bar(B_EMPTY + st));
        }
        if (ok) tc_commit(sm.bar(B_AFULL + acc));
    }
    if (!ok) {
        tc_commit(sm.bar(B_DRAIN));
        wait_bar_quiet(sm.bar(B_DRAIN), 0);
    }
}

// Warps 0-3: for every tile, every 32-column group of token rows, calls
// f(row, seg, seg_lo, valid, col0, x) where row is this thread's weight row,
// valid says it lies in the tile, and x[c] holds D[row, col0 + c] (fp32 bits).
// Returns false after an abort.
// With split-K each split writes its fp32 partial; the last split of the
// tile to finish (per-tile counter, acquire/release) sums the partials in
// split order and calls f with the sums.  named barrier 1 joins warps 0-3.
template <bool SPLITK, bool PAIR = false, class F>
__device__ __forceinline__ bool epilogue_tiles(const Smem &sm, const Shape &sp, int cid, int grid, uint32_t tmem,
                                               int cps, F &&f)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int acc_cols = sp.halves * sp.Np;
    const int nacc = 2 * acc_cols <= kTmemCols ? 2 : 1;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const int rows = sp.seg_end[sp.nseg - 1];
    TileIter ti(sp, cid, grid, cps);
    int a, b, seg, seg_lo;
    for (int t = 0; ti.next(a, b, seg, seg_lo); ++t) {
        const int acc = t % nacc;
        if (!wait_bar(sm.bar(B_AFULL + acc), (t / nacc) & 1, sm.abort_flag, sp.status)) return false;
        tc_fence_after();
        const int row = a + warp * 32 + lane;
        const bool valid = row < b;
        if constexpr (!SPLITK) {
            // every weight half of the tile: rows a + 128 u + (warp, lane), its Np columns
#pragma unroll
            for (int u = 0; u < (PAIR ? 2 : 1); ++u) {
                if (u == 1 && b - a <= kTileRows) break;
                const int row_u = row + u * kTileRows;
                for (int c0 = 0; c0 < sp.Np && c0 < sp.BK; c0 += 32) {
                    uint32_t x[32];
                    tmem_ld32(lane_base + (uint32_t)(acc * acc_cols + u * sp.Np + c0), x);
                    tmem_wait_ld();
                    f(row_u, seg, seg_lo, row_u < b, c0, x);
                }
            }
        } else {
            const int split = cid % sp.ksplit, tile = cid / sp.ksplit;
            const int ldp = (sp.Np + 31) & ~31;          // partial row stride: whole 32-column groups
            for (int c0 = 0; c0 < sp.Np && c0 < sp.BK; c0 += 32) {
                uint32_t x[32];
                tmem_ld32(lane_base + (uint32_t)(acc * sp.Np + c0), x);
                tmem_wait_ld();
                if (valid) {
                    float4 *dst = reinterpret_cast<float4 *>(sp.ws_part + ((size_t)split * rows + row) * ldp + c0);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        dst[c] = make_float4(__uint_as_float(x[4 * c]), __uint_as_float(x[4 * c + 1]),
                                             __uint_as_float(x[4 * c + 2]), __uint_as_float(x[4 * c + 3]));
                }
            }
            // The barrier orders the four warps' partial stores before thread
            // 0's release; its acquire, then the barrier, orders every other
            // split's partial before this CTA's loads when it is the last.
            asm volatile("bar.sync 1, 128;" ::: "memory");
            __shared__ int last_split;
            if (threadIdx.x == 0) {
                unsigned int old;
                asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;"
                             : "=r"(old)
                             : "l"(sp.ws_count + tile)
                             : "memory");
                last_split = old == (unsigned)(sp.ksplit - 1);
                if (last_split) sp.ws_count[tile] = 0u;          // every split has arrived
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (last_split) {
                for (int c0 = 0; c0 < sp.Np && c0 < sp.BK; c0 += 32) {
                    // this split's own partial again from TMEM; the others' from
                    // L2, kSumBatch at a time; summed in split order from zero, so the
                    // result does not depend on which split finished last
                    uint32_t own[32];
                    tmem_ld32(lane_base + (uint32_t)(acc * sp.Np + c0), own);
                    tmem_wait_ld();
                    float sum[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) sum[c] = 0.f;
                    for (int s2 = 0; s2 < sp.ksplit; s2 += kSumBatch) {
                        // up to kSumBatch partials' loads in flight at once
                        float4 v[kSumBatch][8];
#pragma unroll
                        for (int u = 0; u < kSumBatch; ++u) {
                            const int su = s2 + u;
                            const float4 *src =
                                reinterpret_cast<const float4 *>(sp.ws_part + ((size_t)su * rows + row) * ldp + c0);
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                v[u][c] = !valid || su >= sp.ksplit ? make_float4(0.f, 0.f, 0.f, 0.f)
                                          : su != split
                                              ? __ldcg(src + c)
                                              : make_float4(__uint_as_float(own[4 * c]), __uint_as_float(own[4 * c + 1]),
                                                            __uint_as_float(own[4 * c + 2]), __uint_as_float(own[4 * c + 3]));
                        }
#pragma unroll
                        for (int u = 0; u < kSumBatch; ++u) {
                            if (s2 + u < sp.ksplit) {
#pragma unroll
                                for (int c = 0; c < 8; ++c) {
                                    sum[4 * c] += v[u][c].x;
                                    sum[4 * c + 1] += v[u][c].y;
                                    sum[4 * c + 2] += v[u][c].z;
                                    sum[4 * c + 3] += v[u][c].w;
                                }
                            }
                        }
                    }
                    uint32_t x[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) x[c] = __float_as_uint(sum[c]);
                    f(row, seg, seg_lo, valid, c0, x);
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sm.bar(B_AEMPTY + acc));
    }
    return true;
}

// Block prologue of every skinny GEMM kernel (all threads): shared-memory
// carve-up, barrier init, TMEM allocation.  Returns the TMEM base address.
__device__ __forceinline__ uint32_t prologue(Smem &sm, uint8_t *smem_raw, const Shape &sp, int cps,
                                             uint32_t extra_bytes, const Maps &mp)
{
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t aligned = (raw + 1023u) & ~1023u;
    sm.base = aligned;
    sm.ptr = smem_raw + (aligned - raw);
    sm.L = layout_of(sp.Np, sp.nst, cps, extra_bytes, sp.halves);
    sm.cps = cps;
    sm.halves = sp.halves;
    sm.abort_flag = reinterpret_cast<volatile int *>(sm.ptr + sm.L.misc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < sp.nst; ++s) {
            mbar_init(sm.bar(B_FULL + s), 1);
            mbar_init(sm.bar(B_EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(sm.bar(B_AFULL + a), 1);
            mbar_init(sm.bar(B_AEMPTY + a), 4);
        }
        mbar_init(sm.bar(B_DRAIN), 1);
        *sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 4 && lane == 0) {
        for (int s = 0; s < sp.nseg; ++s) {
            tma_prefetch(&mp.w[s]);
            tma_prefetch(&mp.w16[s]);
        }
        tma_prefetch(&mp.x);
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         aligned + sm.L.misc),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    return 0;
}

__device__ __forceinline__ uint32_t tmem_base(const Smem &sm)
{
    return *reinterpret_cast<volatile uint32_t *>(sm.ptr + sm.L.misc);
}

__device__ __forceinline__ void tmem_free(uint32_t tmem)
{
    if ((threadIdx.x >> 5) == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

// Host: chunks per stage (the most of 4, 2, 1 that divide the hidden chunks
// and leave two stages in the ring) and the stage count.
inline void pipeline_of(int Np, int nk, int *cps, int *nst, int halves = 1)
{
    *cps = 1;
    for (int c = 4; c >= 2; c >>= 1) {
        const uint32_t sb = (uint32_t)c * ((uint32_t)halves * kABytes + (uint32_t)Np * 128u);
        if (nk % c == 0 && 2 * sb <= kRingBudget) {
            *cps = c;
            break;
        }
    }
    const uint32_t sb = (uint32_t)*cps * ((uint32_t)halves * kABytes + (uint32_t)Np * 128u);
    const int n = (int)(kRingBudget / sb);
    *nst = n > kMaxStages ? kMaxStages : n;
}

inline int padded_n(int BK)
{
    return BK <= 256 ? (BK + 15) & ~15 : (BK + 31) & ~31;
}

// Host: encode the token-row map and one weight segment's two maps.
inline bool encode_x(Maps &m, const void *x, int BK, int Hd, int Np)
{
    const uint64_t dims[2] = {(uint64_t)Hd, (uint64_t)BK}, str[1] = {(uint64_t)Hd * 2};
    const uint32_t box[2] = {64, (uint32_t)(Np > 256 ? Np / 2 : Np)};
    return encode_bf16_sw128(&m.x, 2, x, dims, str, box);
}

inline bool encode_w(Maps &m, int s, const void *w, int rows, int Hd)
{
    const uint64_t dims[2] = {(uint64_t)Hd, (uint64_t)rows}, str[1] = {(uint64_t)Hd * 2};
    const uint32_t box[2] = {64, 128}, box16[2] = {64, 16};
    return encode_bf16_sw128(&m.w[s], 2, w, dims, str, box) && encode_bf16_sw128(&m.w16[s], 2, w, dims, str, box16);
}

}  // namespace sg
}  // namespace orthrus

// Rejection-sampling verification at temperature T > 0.  The pages evaluate
// greedy and rejection-sampling decoding (Orthrus-Qwen3, agentlenshq.com blog,
// "limitations"; results "depending on task and temperature", gist.science
// technical summary, section 4) without a formula; this is the standard
// lossless speculative-sampling rule, which keeps the AR head's distribution.
//
// For sequence b, left to right over block slots i, with p = softmax(AR logits
// / T) and q = softmax(draft logits / T) of row t = b * K + i and x =
// proposed[b, i]: x is kept iff u_accept[t] * q(x) < p(x) (probability
// min(1, p(x) / q(x))).  At the first rejection a the next token is drawn from
// the residual r = max(0, p - q) by inverse CDF with u_resample[b] (from p
// itself when r is empty); with every slot kept it is the last proposal.
//
// Two launches:
//   1. rs_stats: grid (splits, B*K).  Each CTA streams one vocabulary chunk of
//      one row of both logit arrays (16-byte streaming loads) and reduces it to
//      (max, sum of 2^(c x - max)) per array, c = log2(e) / T.
//   2. rs_resid: grid (rsplit, B).  Every CTA of sequence b merges the chunk
//      statistics into each row's normalisers and takes the K accept decisions
//      (the same in every CTA), keeping the first rejection a.  When a < K,
//      each CTA sums the residual of row a over its share of 128-element tiles
//      (one warp per tile) into the workspace; the last CTA of the sequence to
//      finish (a counter in the workspace) scans the tile sums to the tile
//      holding u_resample * (total) and one warp scans that tile to the drawn
//      token.  The tile sums and the scan are the same arithmetic in the same
//      order whatever the number of CTAs, so the draw does not depend on it.
#include "common.cuh"
#include "kernels.h"

namespace orthrus {

namespace {

constexpr int kStatsThreads = 256;
constexpr int kVerifyThreads = 256;
constexpr int kTileElems = 128;                       // residual tile: 32 lanes x 4

struct Stat {
    float m, l;                                       // max and sum of 2^(y - m), log2 units
};

__device__ __forceinline__ void stat_add(Stat &s, float y)
{
    if (y > s.m) {
        s.l = s.l * fast_exp2(s.m - y);               // (m = -inf: 0)
        s.m = y;
    }
    s.l += fast_exp2(y - s.m);
}

__device__ __forceinline__ Stat stat_merge(Stat a, Stat b)
{
    const float m = fmaxf(a.m, b.m);
    if (m == -INFINITY) return a;
    Stat r;
    r.m = m;
    r.l = a.l * fast_exp2(a.m - m) + b.l * fast_exp2(b.m - m);
    return r;
}

__device__ __forceinline__ Stat warp_stat(Stat s)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        Stat t;
        t.m = __shfl_xor_sync(0xffffffffu, s.m, o);
        t.l = __shfl_xor_sync(0xffffffffu, s.l, o);
        s = stat_merge(s, t);
    }
    return s;
}

__global__ void __launch_bounds__(kStatsThreads) rs_stats_kernel(RejectArgs p)
{
    const int split = blockIdx.x, row = blockIdx.y;
    const int lo = split * p.chunk;
    const int hi = lo + p.chunk < p.V ? lo + p.chunk : p.V;
    const float *a = p.ar + (size_t)row * p.V;
    const float *d = p.dr + (size_t)row * p.V;
    const float c = p.c;
    Stat sp = {-INFINITY, 0.f}, sq = {-INFINITY, 0.f};
    if ((p.V & 3) == 0 && (p.chunk & 3) == 0) {
        const float4 *a4 = reinterpret_cast<const float4 *>(a), *d4 = reinterpret_cast<const float4 *>(d);
        for (int j = (lo >> 2) + threadIdx.x; j < (hi >> 2); j += kStatsThreads) {
            const float4 x = __ldcs(a4 + j), y = __ldcs(d4 + j);
            stat_add(sp, x.x * c);
            stat_add(sp, x.y * c);
            stat_add(sp, x.z * c);
            stat_add(sp, x.w * c);
            stat_add(sq, y.x * c);
            stat_add(sq, y.y * c);
            stat_add(sq, y.z * c);
            stat_add(sq, y.w * c);
        }
    } else {
        for (int j = lo + threadIdx.x; j < hi; j += kStatsThreads) {
            stat_add(sp, __ldcs(a + j) * c);
            stat_add(sq, __ldcs(d + j) * c);
        }
    }
    sp = warp_stat(sp);
    sq = warp_stat(sq);
    __shared__ Stat red[2][kStatsThreads / 32];
    if ((threadIdx.x & 31) == 0) {
        red[0][threadIdx.x >> 5] = sp;
        red[1][threadIdx.x >> 5] = sq;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        Stat u = {-INFINITY, 0.f}, v = {-INFINITY, 0.f};
        if (threadIdx.x < kStatsThreads / 32) {
            u = red[0][threadIdx.x];
            v = red[1][threadIdx.x];
        }
        u = warp_stat(u);
        v = warp_stat(v);
        if (threadIdx.x == 0) p.ws[(size_t)row * p.splits + split] = make_float4(u.m, u.l, v.m, v.l);
    }
}

__device__ __forceinline__ float block_excl_scan(float v, float *tmp, float *total)
{
    // exclusive prefix over the block's threads in thread order (fixed order)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        float run = 0.f;
        for (int w = 0; w < kVerifyThreads / 32; ++w) {
            const float s = tmp[w];
            tmp[w] = run;
            run += s;
        }
        *total = run;
    }
    __syncthreads();
    return tmp[warp] + incl - v;
}

struct ResidShared {
    Stat rp[ORTHRUS_MAX_BLOCK], rq[ORTHRUS_MAX_BLOCK];
    float tile_sum[kMaxRejectTiles];
    float scan_tmp[kVerifyThreads / 32];
    float total;
    int first_rej, tile_found, last;
};

// Residual mass of element v of one row (0 past the end).  The products are
// explicitly rounded: the residual is the difference of two rounded
// probabilities, exactly zero where the views agree, never an FMA-contracted
// rounding error.
struct RowMass {
    const float *ar, *dr;
    float c, mp, mq, ip, iq;
    int V;
    bool from_p;
    __device__ __forceinline__ float operator()(int v) const
    {
        if (v >= V) return 0.f;
        const float pv = __fmul_rn(fast_exp2(ar[v] * c - mp), ip);
        if (from_p) return pv;
        const float r = pv - __fmul_rn(fast_exp2(dr[v] * c - mq), iq);
        return r > 0.f ? r : 0.f;
    }
};

// Sum of tile k (128 elements: lane l holds elements 4l..4l+3, added in order,
// then a butterfly over the lanes); every lane returns the sum.
__device__ __forceinline__ float tile_mass(const RowMass &mass, int k, int lane)
{
    const int v0 = k * kTileElems + lane * 4;
    float s = mass(v0) + mass(v0 + 1) + mass(v0 + 2) + mass(v0 + 3);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Inverse-CDF search over the row's tile sums (in shared memory): the token
// whose cumulative mass first exceeds u * total.  Returns false (nothing
// written) when the total is not positive.  Called by the whole block.
__device__ bool draw_from_tiles(const RejectArgs &p, const RowMass &mass, ResidShared &sh, int ntile, int b,
                                int a)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // tiles in contiguous runs per thread, then a block scan of the runs
    const int per = (ntile + kVerifyThreads - 1) / kVerifyThreads;
    const int t0 = threadIdx.x * per, t1 = t0 + per < ntile ? t0 + per : ntile;
    float run = 0.f;
    for (int k = t0; k < t1; ++k) run += sh.tile_sum[k];
    const float pre = block_excl_scan(run, sh.scan_tmp, &sh.total);
    const float R = sh.total;
    if (!(R > 0.f)) return false;
    const float target = p.u_resample[b] * R;
    if (threadIdx.x == 0) sh.tile_found = -1;
    __syncthreads();
    // the run holding the target (the last nonempty one if rounding put it past the end)
    float acc = pre;
    int kt = -1;
    for (int k = t0; k < t1; ++k) {
        if (sh.tile_sum[k] > 0.f) kt = k;
        if (sh.tile_sum[k] > 0.f && target < acc + sh.tile_sum[k]) break;
        acc += sh.tile_sum[k];
    }
    const bool holds = t0 < t1 && pre <= target && (target < pre + run || threadIdx.x == kVerifyThreads - 1 ||
                                                    t1 == ntile);
    if (holds && kt >= 0) atomicMax(&sh.tile_found, kt);
    __syncthreads();
    int k = sh.tile_found;
    if (k < 0) {                                      // (rounding: fall back to the last nonempty tile)
        if (threadIdx.x == 0)
            for (int j = ntile - 1; j >= 0; --j)
                if (sh.tile_sum[j] > 0.f) {
                    sh.tile_found = j;
                    break;
                }
        __syncthreads();
        k = sh.tile_found;
    }
    // prefix of the tiles before k (same order as the runs), then one warp scans tile k
    if (warp == 0 && k >= 0) {
        float before = 0.f;
        for (int j = lane; j < k; j += 32) before += sh.tile_sum[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
        const int v0 = k * kTileElems + lane * 4;
        const float m0 = mass(v0), m1 = mass(v0 + 1), m2 = mass(v0 + 2), m3 = mass(v0 + 3);
        const float own = m0 + m1 + m2 + m3;
        float incl = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        const float t = target - before;              // position inside tile k
        const float ex = incl - own;
        const unsigned in = __ballot_sync(0xffffffffu, own > 0.f && t < incl);
        int pick = -1;
        if (in) {
            const int l = __ffs(in) - 1;
            if (lane == l) {
                float c = ex;
                pick = v0 + 3;
                const float ms[4] = {m0, m1, m2, m3};
                int last_nz = -1;
                for (int e = 0; e < 4; ++e) {
                    if (ms[e] > 0.f) last_nz = v0 + e;
                    if (ms[e] > 0.f && t < c + ms[e]) {
                        pick = v0 + e;
                        last_nz = -2;
                        break;
                    }
                    c += ms[e];
                }
                if (last_nz >= 0) pick = last_nz;
            }
            pick = __shfl_sync(0xffffffffu, pick, l);
        } else {
            // the target lies at or past the tile's end: the tile's last nonzero element
            const unsigned nz = __ballot_sync(0xffffffffu, own > 0.f);
            const int l = 31 - __clz(nz);
            if (lane == l) pick = m3 > 0.f ? v0 + 3 : m2 > 0.f ? v0 + 2 : m1 > 0.f ? v0 + 1 : v0;
            pick = __shfl_sync(0xffffffffu, pick, l);
        }
        if (lane == 0) {
            p.accepted[b] = a;
            p.next_token[b] = pick;
        }
    }
    return true;
}

__global__ void __launch_bounds__(kVerifyThreads) rs_resid_kernel(RejectArgs p)
{
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __shared__ ResidShared sh;
    static_assert(ORTHRUS_MAX_BLOCK <= kVerifyThreads, "one block slot per thread");
    // ---- thread i < K: slot i's proposal and its logits in both views, loaded
    // before (and overlapping) the statistics merge
    int x = -1;
    float ar_x = 0.f, dr_x = 0.f, ua = 0.f;
    if (threadIdx.x < p.K) {
        const size_t row = (size_t)b * p.K + threadIdx.x;
        x = p.proposed[row];
        ua = p.u_accept[row];
        if (x >= 0 && x < p.V) {
            ar_x = p.ar[row * p.V + x];
            dr_x = p.dr[row * p.V + x];
        }
    }
    // ---- each row's normalisers from its chunk statistics
    for (int i = warp; i < p.K; i += kVerifyThreads / 32) {
        const float4 *w = p.ws + ((size_t)b * p.K + i) * p.splits;
        Stat u = {-INFINITY, 0.f}, v = {-INFINITY, 0.f};
        for (int s = lane; s < p.splits; s += 32) {
            const float4 x = w[s];
            u = stat_merge(u, Stat{x.x, x.y});
            v = stat_merge(v, Stat{x.z, x.w});
        }
        u = warp_stat(u);
        v = warp_stat(v);
        if (lane == 0) {
            sh.rp[i] = u;
            sh.rq[i] = v;
        }
    }
    if (threadIdx.x == 0) sh.first_rej = p.K;
    __syncthreads();
    // ---- every slot's accept decision; the first rejection wins
    if (threadIdx.x < p.K) {
        const int i = threadIdx.x;
        bool keep = false;
        if (x >= 0 && x < p.V) {
            const float px = fast_exp2(ar_x * p.c - sh.rp[i].m) / sh.rp[i].l;
            const float qx = fast_exp2(dr_x * p.c - sh.rq[i].m) / sh.rq[i].l;
            keep = ua * qx < px;
        }
        if (!keep) atomicMin(&sh.first_rej, i);
    }
    __syncthreads();
    const int a = sh.first_rej;
    if (a == p.K) {
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            p.accepted[b] = p.K;
            p.next_token[b] = p.proposed[(size_t)b * p.K + p.K - 1];
        }
        return;
    }
    // ---- this CTA's share of the residual tile sums of row a
    const size_t row = (size_t)b * p.K + a;
    RowMass mass;
    mass.ar = p.ar + row * p.V;
    mass.dr = p.dr + row * p.V;
    mass.c = p.c;
    mass.mp = sh.rp[a].m;
    mass.mq = sh.rq[a].m;
    mass.ip = 1.f / sh.rp[a].l;
    mass.iq = 1.f / sh.rq[a].l;
    mass.V = p.V;
    mass.from_p = false;
    const int ntile = (p.V + kTileElems - 1) / kTileElems;
    float *tiles = p.ws_tiles + (size_t)b * ntile;
    const int k0 = blockIdx.x * p.rtiles;
    const int k1 = k0 + p.rtiles < ntile ? k0 + p.rtiles : ntile;
    for (int k = k0 + warp; k < k1; k += kVerifyThreads / 32) {
        const float s = tile_mass(mass, k, lane);
        if (lane == 0) tiles[k] = s;
    }
    // ---- the last CTA of the sequence draws
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int done = atomicAdd(p.ws_count + b, 1);
        sh.last = done == (int)gridDim.x - 1;
        if (sh.last) {
            __threadfence();
            p.ws_count[b] = 0;                        // left zero for the next call
        }
    }
    __syncthreads();
    if (!sh.last) return;
    for (int k = threadIdx.x; k < ntile; k += kVerifyThreads) sh.tile_sum[k] = __ldcg(tiles + k);
    __syncthreads();
    if (draw_from_tiles(p, mass, sh, ntile, b, a)) return;
    // the residual is empty (p and q agree on row a): draw from p, in this CTA alone
    mass.from_p = true;
    for (int k = warp; k < ntile; k += kVerifyThreads / 32) {
        const float s = tile_mass(mass, k, lane);
        if (lane == 0) sh.tile_sum[k] = s;
    }
    __syncthreads();
    draw_from_tiles(p, mass, sh, ntile, b, a);
}

}  // namespace

cudaError_t launch_rejection(const RejectArgs &p, cudaStream_t st)
{
    dim3 g1(p.splits, p.B * p.K);
    rs_stats_kernel<<<g1, kStatsThreads, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    rs_resid_kernel<<<dim3(p.rsplit, p.B), kVerifyThreads, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace orthrus

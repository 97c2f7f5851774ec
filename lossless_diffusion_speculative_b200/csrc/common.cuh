// Shared device helpers of liborthrus: the split-KV work decomposition, the
// status word, and small numeric helpers.  Used by every kernel file.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/orthrus.h"

namespace orthrus {

// ----------------------------------------------------------------------------
// Status word: device-detected errors are OR-ed in, the work is skipped.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void raise_status(int32_t *status, int32_t bit)
{
    if (status) atomicOr(status, bit);
}

// ----------------------------------------------------------------------------
// Split-KV decomposition ("stream-K" over keys).
//
// Sequence b contributes Hkv segments (one per KV head g) of len_b = ctx_b + K
// keys each (0 when ctx_b is out of range).  All segments are laid end to end
// in the order s = b*Hkv + g; the flat key space [0, W) is cut into P_eff
// contiguous, equal ranges, one per CTA.  A CTA's range can touch several
// segments, and a segment can be covered by several CTAs.  Every (CTA c,
// segment s) piece writes either the final output (when c alone covers s) or
// a partial (O normalised, log2-sum-exp) into workspace slot c + s; slots are
// unique because consecutive CTAs share at most one segment.
// ----------------------------------------------------------------------------
struct Decomp {
    int64_t W;      // total keys over all segments
    int P;          // CTAs that carry work
};

__device__ __forceinline__ int seg_len(const int32_t *ctx_lens, int b, int K,
                                       int S_max)
{
    const int c = __ldg(ctx_lens + b);
    return (c < 0 || (int64_t)c + K > S_max) ? 0 : c + K;
}

// Total work and active CTA count; identical in every kernel that uses it.
__device__ __forceinline__ Decomp make_decomp(const int32_t *ctx_lens, int B,
                                              int Hkv, int K, int S_max,
                                              int grid, int min_keys)
{
    int64_t W = 0;
    for (int b = 0; b < B; ++b) W += (int64_t)Hkv * seg_len(ctx_lens, b, K, S_max);
    Decomp d;
    d.W = W;
    int64_t want = (W + min_keys - 1) / min_keys;
    if (want < 1) want = 1;
    d.P = (int)(want < grid ? want : grid);
    return d;
}

__device__ __forceinline__ int64_t range_start(const Decomp &d, int c)
{
    return (int64_t)c * d.W / d.P;
}

// The CTA whose range holds flat key x: max{c : range_start(c) <= x}.
__device__ __forceinline__ int cta_of(const Decomp &d, int64_t x)
{
    return (int)(((x + 1) * d.P - 1) / d.W);
}

// Flat start of segment (b, g); also returns len_b.  O(B).
__device__ __forceinline__ int64_t seg_start(const int32_t *ctx_lens, int b,
                                             int g, int Hkv, int K, int S_max,
                                             int *len_out)
{
    int64_t off = 0;
    for (int bb = 0; bb < b; ++bb) off += (int64_t)Hkv * seg_len(ctx_lens, bb, K, S_max);
    const int len = seg_len(ctx_lens, b, K, S_max);
    *len_out = len;
    return off + (int64_t)g * len;
}

// A piece = the part of one segment inside one CTA's range.
struct Piece {
    int b, g;       // sequence, KV head
    int s;          // segment index b*Hkv + g
    int len;        // segment length (ctx_b + K)
    int a, e;       // key range [a, e) within the segment, 0 <= a < e <= len
    int64_t s0;     // flat start of the segment
};

// Iterates the pieces of CTA c in flat order.  Usage:
//   PieceIter it(...); Piece p; while (it.next(p)) {...}
struct PieceIter {
    const int32_t *ctx;
    int B, Hkv, K, S_max;
    int64_t lo, hi;      // CTA range
    int b, g;            // current segment
    int64_t off_b;       // flat start of sequence b
    int len_b;

    __device__ __forceinline__ PieceIter(const int32_t *ctx_lens, int B_, int Hkv_,
                                         int K_, int S_max_, const Decomp &d, int c)
        : ctx(ctx_lens), B(B_), Hkv(Hkv_), K(K_), S_max(S_max_)
    {
        lo = range_start(d, c);
        hi = range_start(d, c + 1);
        off_b = 0;
        b = 0;
        g = 0;
        len_b = B > 0 ? seg_len(ctx, 0, K, S_max) : 0;
        // skip whole sequences that end at or before lo
        while (b < B && off_b + (int64_t)Hkv * len_b <= lo) {
            off_b += (int64_t)Hkv * len_b;
            ++b;
            len_b = b < B ? seg_len(ctx, b, K, S_max) : 0;
        }
        if (b < B && len_b > 0) g = (int)((lo - off_b) / len_b);
    }

    __device__ __forceinline__ bool next(Piece &p)
    {
        while (b < B) {
            if (len_b == 0 || g >= Hkv) {
                off_b += (int64_t)Hkv * len_b;
                ++b;
                g = 0;
                len_b = b < B ? seg_len(ctx, b, K, S_max) : 0;
                continue;
            }
            const int64_t s0 = off_b + (int64_t)g * len_b;
            if (s0 >= hi) return false;
            const int64_t a = lo > s0 ? lo - s0 : 0;
            const int64_t e = hi < s0 + len_b ? hi - s0 : len_b;
            p.b = b;
            p.g = g;
            p.s = b * Hkv + g;
            p.len = len_b;
            p.a = (int)a;
            p.e = (int)e;
            p.s0 = s0;
            ++g;
            if (e > a) return true;
        }
        return false;
    }
};

// ----------------------------------------------------------------------------
// Numeric helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x)
{
    return __bfloat162float(x);
}

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace orthrus

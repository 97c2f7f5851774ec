// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/orthrus.h"

namespace orthrus {

// Everything one attention launch needs, passed by value to the kernels.
struct AttnArgs {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *ctx_lens;
    float *out;
    int32_t *ws_sync;    // [3, kMaxSyncUnits] split-merge flags and counters (zero between calls)
    int32_t *ws_plan;    // [kMaxSyncUnits, kPlanEntryInts] per-CTA cached work plans
    float *ws_o;         // [slots, rows, D] split partials (O normalised)
    float *ws_lse;       // [slots, lse_pitch(rows)] log2-sum-exp of each partial
    int32_t *status;
    int B, Hq, Hkv, D, S_max, K;
    int view;            // orthrus_view
    int dtype;           // orthrus_dtype
    float scale_log2;    // softmax scale * log2(e)
    int min_keys;        // smallest key range worth a CTA
    // Sequence b of the call reads the cache of sequence b / cache_div and the
    // query / output rows from q_row0(b); a decode call has cache_div = 1 and
    // q_seq_rows = K (rows b * K).  Chunked prefill runs prompt chunk
    // prefill_chunk_of(j, cache_div) of sequence s as call sequence
    // s * cache_div + j.
    int cache_div;
    int q_seq_rows;
    __host__ __device__ __forceinline__ int cache_seq(int b) const { return cache_div == 1 ? b : b / cache_div; }
    __host__ __device__ __forceinline__ size_t q_row0(int b) const;
};

// Order of a prompt's chunks in a chunked-prefill call: shortest and longest
// alternate (0, n-1, 1, n-2, ...), so that the equal key ranges of the work
// split each hold a few short segments instead of one range holding all of
// them (every segment costs a fixed query load and epilogue on top of its
// keys).
__host__ __device__ __forceinline__ int prefill_chunk_of(int j, int n)
{
    return (j & 1) ? n - 1 - (j >> 1) : (j >> 1);
}

__host__ __device__ __forceinline__ size_t AttnArgs::q_row0(int b) const
{
    return cache_div == 1 ? (size_t)b * q_seq_rows
                          : (size_t)(b / cache_div) * q_seq_rows +
                                (size_t)prefill_chunk_of(b % cache_div, cache_div) * K;
}

// Workspace layout shared by the attention paths: a fixed block of flags and
// counters used by the tensor-core path's in-kernel split merge (zero before
// and after every call):
//   first[u]  unit u has published the partial of the first piece of its range
//             (set only when that piece is shared and is not also its last)
//   last[u]   unit u has published the partial of the last piece of its range
//   depart[u] units done reading the flags of the segment that unit u opens
// then `slots` fp32 partial tiles [rows, D], then their log2-sum-exp values.
constexpr int kMaxSyncUnits = 160;     // >= the tensor-core path's CTA count (148 on B200)
constexpr int kSyncFirst = 0, kSyncLast = 1, kSyncDepart = 2;
constexpr size_t kSyncBytes = 3 * kMaxSyncUnits * sizeof(int32_t);
// After it, one cached work plan per CTA of the tensor-core path: the split
// of the key space that CTA computed, keyed by the shape and the context
// lengths it was computed for (batches of up to kPlanMaxB sequences), so that
// a later call with the same lengths loads it instead of recomputing it.
constexpr int kPlanMaxB = 32;
constexpr int kPlanEntryInts = 64;     // key (8) + lengths (32) + plan (10), padded
constexpr size_t kPlanBytes = (size_t)kMaxSyncUnits * kPlanEntryInts * sizeof(int32_t);
inline size_t attn_ws_o_bytes(int slots, int rows, int D)
{
    return ((size_t)slots * rows * D * sizeof(float) + 255) & ~(size_t)255;
}
// log2-sum-exp rows are padded to whole 16-byte groups (bulk-copyable)
__host__ __device__ inline int lse_pitch(int rows) { return (rows + 3) & ~3; }
inline size_t attn_ws_lse_bytes(int slots, int rows)
{
    return ((size_t)slots * lse_pitch(rows) * sizeof(float) + 255) & ~(size_t)255;
}
inline size_t attn_ws_bytes(int slots, int rows, int D)
{
    return kSyncBytes + kPlanBytes + attn_ws_o_bytes(slots, rows, D) + attn_ws_lse_bytes(slots, rows);
}

// TMA tensor map of a bf16 tensor with 128-byte swizzle: dims[0] innermost
// (elements), strides[i] = bytes between consecutive indices of dimension i+1.
bool encode_bf16_sw128(CUtensorMap *m, int rank, const void *base, const uint64_t *dims,
                       const uint64_t *strides, const uint32_t *box);

cudaError_t launch_attn_simt(const AttnArgs &p, int grid, cudaStream_t st);
cudaError_t launch_attn_combine(const AttnArgs &p, int grid_main, cudaStream_t st);

// Tensor-core path (bf16, D == 128, G*K <= 128, sm_100).  attn_tc_plan gives
// the split units (clusters) and the smallest key range worth one unit.
bool attn_tc_supported(int dtype, int D, int rows);
bool attn_tc_plan(int *units, int *min_keys);
cudaError_t launch_attn_tc(const AttnArgs &p, int units, cudaStream_t st);

struct ConsensusArgs {
    const float *logits;
    const int32_t *proposed;
    int32_t *accepted;
    int32_t *next_token;
    int32_t *argmax_out;
    unsigned long long *ws;   // [B*K, splits] packed (value, index) keys
    int32_t *status;
    int B, K, V, splits, chunk;
};
cudaError_t launch_consensus(const ConsensusArgs &p, cudaStream_t st);

// Shape of one skinny-GEMM launch (skinny_gemm.cuh): weight rows in up to
// three stacked segments against a few token rows.
constexpr int kMaxSkinnySegs = 3;
struct SkinnyShape {
    int nseg;                            // weight segments (1..3)
    int seg_end[kMaxSkinnySegs];         // segment s = rows [seg_end[s-1], seg_end[s])
    int Hd;                              // hidden size (multiple of 64)
    int BK;                              // token rows
    int Np;                              // token rows padded for the MMA's N
    int nst;                             // pipeline stages
    int halves;                          // 128-row weight tiles per pass (1, or 2 without split-K)
    int32_t *status;
    // split-K (ksplit > 1): CTA u computes tile u / ksplit over hidden chunks
    // [k0(u % ksplit), k0(u % ksplit + 1)) into an fp32 partial; the last
    // split of a tile (per-tile counter) sums the partials in split order
    int ksplit;
    float *ws_part;                      // [ksplit, rows, Np rounded up to 32] fp32 partials
    unsigned int *ws_count;              // [tiles] splits done, zero between calls
};

// Fused AR LM head + argmax + consensus (lm_head.cu).
constexpr int kMaxLmRows = ORTHRUS_MAX_LM_ROWS;   // B * K token rows per call
struct LmHeadArgs {
    const int32_t *proposed;
    int32_t *accepted;
    int32_t *next_token;
    int32_t *argmax_out;
    unsigned long long *ws_keys;         // [B*K] packed (value, index) maxima, zero between calls
    unsigned int *ws_done;               // CTAs finished, zero between calls
    int B, K, V;
    SkinnyShape shape;
};

// The block's QKV projection written into the query buffer and the cache tail
// (qkv_proj.cu).
struct QkvArgs {
    const int32_t *ctx_lens;
    void *q_out;                         // [B, K, Hq, D] bf16
    void *k_cache, *v_cache;             // [B, Hkv, S_max, D] bf16
    int B, K, Hq, Hkv, D, S_max;
    SkinnyShape shape;
};

// Rejection-sampling verification (rejection.cu).
constexpr int kMaxRejectTiles = 2048;    // vocabulary <= 2048 * 128 = 262144
struct RejectArgs {
    const float *ar, *dr;                // [B*K, V] AR-view and draft-view logits
    const int32_t *proposed;             // [B*K]
    const float *u_accept;               // [B*K] uniform draws in [0, 1)
    const float *u_resample;             // [B]
    int32_t *accepted;
    int32_t *next_token;
    float4 *ws;                          // [B*K, splits] (max, sum) of both views, log2 units
    float *ws_tiles;                     // [B, ceil(V / 128)] residual tile sums of the rejected row
    int32_t *ws_count;                   // [B] CTAs done with the residual (zero between calls)
    int32_t *status;
    int B, K, V, splits, chunk;
    int rsplit, rtiles;                  // residual pass: CTAs per sequence, tiles per CTA
    float c;                             // log2(e) / temperature
};
cudaError_t launch_rejection(const RejectArgs &p, cudaStream_t st);

struct CommitArgs {
    void *k_caches[ORTHRUS_MAX_LAYERS];
    void *v_caches[ORTHRUS_MAX_LAYERS];
    const void *k_blks[ORTHRUS_MAX_LAYERS];
    const void *v_blks[ORTHRUS_MAX_LAYERS];
    int32_t *ctx_lens;
    const int32_t *accepted;
    int32_t *status;
    int num_layers, B, Hkv, D, S_max, K, elem_bytes;
    int copy;
    int all_rows;        // 1: install all K block slots, no acceptance, no advance
};
cudaError_t launch_kv_commit(const CommitArgs &p, cudaStream_t st);

}  // namespace orthrus

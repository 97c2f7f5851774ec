// liborthrus C ABI: host-side argument checks, launch configuration and the
// choice between the tensor-core and CUDA-core attention paths.  Declarations
// and the contract of every entry point are in include/orthrus.h.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace orthrus;

namespace {

constexpr int kVersion = (1 << 16) | 0;

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// SM count of the current device (queried per call: cheap, and correct when
// the caller switches devices).
int current_sm_count()
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return sms;
}

// CTAs per attention launch and key granularity, per path.
struct AttnPlan {
    bool tc;
    int grid;
    int min_keys;
    int slots;
};

bool attn_shape_ok(int B, int Hq, int Hkv, int D, int S_max, int K, orthrus_dtype dt)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || S_max <= 0 || K <= 0) return false;
    if (Hq % Hkv) return false;
    if (dt != ORTHRUS_BF16 && dt != ORTHRUS_F32) return false;
    return true;
}

bool attn_shape_supported(int Hq, int Hkv, int D, int K)
{
    return D % 32 == 0 && D <= ORTHRUS_MAX_HEAD_DIM && K <= ORTHRUS_MAX_BLOCK &&
           (int64_t)(Hq / Hkv) * K <= 4096;
}

// `grid` is the number of split units (CTAs).
AttnPlan plan_attn(int B, int Hq, int Hkv, int D, int K, orthrus_dtype dt, int sms)
{
    AttnPlan pl;
    const int rows = (Hq / Hkv) * K;
    pl.tc = attn_tc_supported(dt, D, rows) && attn_tc_plan(&pl.grid, &pl.min_keys);
    if (!pl.tc) {
        pl.grid = 2 * sms;
        pl.min_keys = 64;
    }
    pl.slots = pl.grid + B * Hkv;
    // equal-length segments split evenly when the unit count is a multiple of
    // the segment count (no unit straddles a segment boundary): rounded down
    // to one when that idles at most 1/16 of the units; otherwise every unit
    // works and some straddle two segments (ragged lengths gain nothing from
    // the rounding either)
    const int segs = B * Hkv;
    if (pl.grid >= segs && pl.grid % segs <= pl.grid / 16) pl.grid -= pl.grid % segs;
    return pl;
}

}  // namespace

extern "C" {

int orthrus_version(void) { return kVersion; }

const char *orthrus_error_string(int code)
{
    switch (code) {
    case ORTHRUS_OK: return "ok";
    case ORTHRUS_ERR_ARG: return "invalid argument";
    case ORTHRUS_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ORTHRUS_ERR_ALIGN: return "pointer not 16-byte aligned";
    case ORTHRUS_ERR_WORKSPACE: return "workspace missing or too small";
    case ORTHRUS_ERR_LAUNCH: return "CUDA launch failed";
    case ORTHRUS_ERR_DEVICE: return "no usable CUDA device";
    default: return "unknown error";
    }
}

size_t orthrus_attn_workspace_size(int B, int Hq, int Hkv, int D, int K, orthrus_dtype dtype)
{
    if (!attn_shape_ok(B, Hq, Hkv, D, 1, K, dtype) || !attn_shape_supported(Hq, Hkv, D, K))
        return 0;
    const int sms = current_sm_count();
    if (sms <= 0) return 0;
    const AttnPlan pl = plan_attn(B, Hq, Hkv, D, K, dtype, sms);
    return attn_ws_bytes(pl.slots, (Hq / Hkv) * K, D);
}

}  // extern "C"

namespace {

// One attention launch (both paths).  cache_div / q_seq_rows: see AttnArgs.
int attn_call(orthrus_view view, orthrus_dtype dtype, const void *q, const void *k_cache,
              const void *v_cache, const int32_t *ctx_lens, int B, int Hq, int Hkv, int D, int S_max,
              int K, float scale, float *out, void *workspace, size_t workspace_bytes, int32_t *status,
              void *stream, int cache_div, int q_seq_rows)
{
    if (view != ORTHRUS_DIFF && view != ORTHRUS_AR) return ORTHRUS_ERR_ARG;
    if (!q || !k_cache || !v_cache || !ctx_lens || !out) return ORTHRUS_ERR_ARG;
    if (!attn_shape_ok(B, Hq, Hkv, D, S_max, K, dtype)) return ORTHRUS_ERR_ARG;
    if (K > S_max) return ORTHRUS_ERR_ARG;
    if (!(scale == scale) || isinf(scale)) return ORTHRUS_ERR_ARG;
    // the on-device work split counts 64-key boxes over all segments in 32 bits
    if ((int64_t)B * Hkv * ((S_max + 63) / 64) >= (int64_t)1 << 31) return ORTHRUS_ERR_UNSUPPORTED;
    if (!attn_shape_supported(Hq, Hkv, D, K)) return ORTHRUS_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (workspace && !aligned16(workspace)))
        return ORTHRUS_ERR_ALIGN;
    const int sms = current_sm_count();
    if (sms <= 0) return ORTHRUS_ERR_DEVICE;
    const AttnPlan pl = plan_attn(B, Hq, Hkv, D, K, dtype, sms);
    const int rows = (Hq / Hkv) * K;
    const size_t need = attn_ws_bytes(pl.slots, rows, D);
    if (!workspace || workspace_bytes < need) return ORTHRUS_ERR_WORKSPACE;

    AttnArgs a;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.ctx_lens = ctx_lens;
    a.out = out;
    char *ws = static_cast<char *>(workspace);
    a.ws_sync = reinterpret_cast<int32_t *>(ws);
    a.ws_plan = reinterpret_cast<int32_t *>(ws + kSyncBytes);
    a.ws_o = reinterpret_cast<float *>(ws + kSyncBytes + kPlanBytes);
    a.ws_lse = reinterpret_cast<float *>(ws + kSyncBytes + kPlanBytes + attn_ws_o_bytes(pl.slots, rows, D));
    a.status = status;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = S_max;
    a.K = K;
    a.view = view;
    a.dtype = dtype;
    const float sc = scale > 0.f ? scale : 1.0f / sqrtf((float)D);
    a.scale_log2 = sc * kLog2e;
    a.min_keys = pl.min_keys;
    a.cache_div = cache_div;
    a.q_seq_rows = q_seq_rows;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = pl.tc ? launch_attn_tc(a, pl.grid, st) : launch_attn_simt(a, pl.grid, st);
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

// Chunked prefill: call sequence s * nch + j is prompt chunk
// c = prefill_chunk_of(j, nch) of sequence s, an AR-view block of kc tokens
// after c * kc context tokens.
__global__ void prefill_ctx_kernel(int32_t *ctx, int n, int nch, int kc, int offset)
{
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < n) ctx[b] = prefill_chunk_of(b % nch, nch) * kc + offset;
}

int prefill_chunk(int G)
{
    int kc = 128;
    while (kc > 1 && G * kc > 128) kc >>= 1;
    return kc;
}

struct PrefillPlan {
    int kc, nch, r;
    size_t ws_attn, ctx_off, total;
};

PrefillPlan prefill_plan(int B, int S, int Hq, int Hkv, int D, orthrus_dtype dtype)
{
    PrefillPlan pp;
    pp.kc = prefill_chunk(Hq / Hkv);
    if (pp.kc > S) pp.kc = S;
    pp.nch = S / pp.kc;
    pp.r = S - pp.nch * pp.kc;
    const size_t w1 = pp.nch ? orthrus_attn_workspace_size(B * pp.nch, Hq, Hkv, D, pp.kc, dtype) : 0;
    const size_t w2 = pp.r ? orthrus_attn_workspace_size(B, Hq, Hkv, D, pp.r, dtype) : 0;
    pp.ws_attn = ((w1 > w2 ? w1 : w2) + 255) & ~(size_t)255;
    pp.ctx_off = pp.ws_attn;
    pp.total = pp.ctx_off + (((size_t)B * (pp.nch + 1) * sizeof(int32_t) + 255) & ~(size_t)255);
    if ((pp.nch && !w1) || (pp.r && !w2)) pp.total = 0;
    return pp;
}

}  // namespace

extern "C" {

int orthrus_attn(orthrus_view view, orthrus_dtype dtype, const void *q, const void *k_cache,
                 const void *v_cache, const int32_t *ctx_lens, int B, int Hq, int Hkv, int D,
                 int S_max, int K, float scale, float *out, void *workspace,
                 size_t workspace_bytes, int32_t *status, void *stream)
{
    return attn_call(view, dtype, q, k_cache, v_cache, ctx_lens, B, Hq, Hkv, D, S_max, K, scale, out,
                     workspace, workspace_bytes, status, stream, 1, K);
}

size_t orthrus_prefill_workspace_size(int B, int S, int Hq, int Hkv, int D, orthrus_dtype dtype)
{
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv) return 0;
    return prefill_plan(B, S, Hq, Hkv, D, dtype).total;
}

int orthrus_prefill_attn(orthrus_dtype dtype, const void *q, const void *k_cache, const void *v_cache,
                         int B, int S, int Hq, int Hkv, int D, int S_max, float scale, float *out,
                         void *workspace, size_t workspace_bytes, int32_t *status, void *stream)
{
    if (!q || !k_cache || !v_cache || !out) return ORTHRUS_ERR_ARG;
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || S_max <= 0 || Hq % Hkv) return ORTHRUS_ERR_ARG;
    if (S > S_max) return ORTHRUS_ERR_ARG;
    if (dtype != ORTHRUS_BF16 && dtype != ORTHRUS_F32) return ORTHRUS_ERR_ARG;
    const PrefillPlan pp = prefill_plan(B, S, Hq, Hkv, D, dtype);
    if (!pp.total) return ORTHRUS_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < pp.total) return ORTHRUS_ERR_WORKSPACE;
    if (!aligned16(workspace)) return ORTHRUS_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char *ws = static_cast<char *>(workspace);
    int32_t *ctx1 = reinterpret_cast<int32_t *>(ws + pp.ctx_off);
    int32_t *ctx2 = ctx1 + (size_t)B * pp.nch;
    const size_t esz = dtype == ORTHRUS_BF16 ? 2 : 4;
    if (pp.nch) {
        const int n = B * pp.nch;
        prefill_ctx_kernel<<<(n + 255) / 256, 256, 0, st>>>(ctx1, n, pp.nch, pp.kc, 0);
        if (cudaGetLastError() != cudaSuccess) return ORTHRUS_ERR_LAUNCH;
        const int rc = attn_call(ORTHRUS_AR, dtype, q, k_cache, v_cache, ctx1, n, Hq, Hkv, D, S_max, pp.kc,
                                 scale, out, ws, pp.ws_attn, status, stream, pp.nch, S);
        if (rc != ORTHRUS_OK) return rc;
    }
    if (pp.r) {
        prefill_ctx_kernel<<<(B + 255) / 256, 256, 0, st>>>(ctx2, B, 1, 0, pp.nch * pp.kc);
        if (cudaGetLastError() != cudaSuccess) return ORTHRUS_ERR_LAUNCH;
        const size_t off = (size_t)pp.nch * pp.kc * Hq * D;
        const int rc = attn_call(ORTHRUS_AR, dtype, static_cast<const char *>(q) + off * esz, k_cache, v_cache,
                                 ctx2, B, Hq, Hkv, D, S_max, pp.r, scale, out + off, ws, pp.ws_attn, status,
                                 stream, 1, S);
        if (rc != ORTHRUS_OK) return rc;
    }
    return ORTHRUS_OK;
}

static void consensus_split(int B, int K, int V, int sms, int *splits, int *chunk)
{
    const int rows = B * K;
    int s = (4 * sms + rows - 1) / rows;         // about four CTAs per SM in total
    const int max_s = (V + 2047) / 2048;         // at least 2048 logits per CTA
    if (s > max_s) s = max_s;
    if (s < 1) s = 1;
    int c = (V + s - 1) / s;
    c = (c + 3) & ~3;                            // whole float4 groups
    s = (V + c - 1) / c;
    *splits = s;
    *chunk = c;
}

size_t orthrus_consensus_workspace_size(int B, int K, int V)
{
    if (B <= 0 || K <= 0 || V <= 0 || K > ORTHRUS_MAX_BLOCK) return 0;
    const int sms = current_sm_count();
    if (sms <= 0) return 0;
    int s, c;
    consensus_split(B, K, V, sms, &s, &c);
    return (size_t)B * K * s * sizeof(unsigned long long);
}

int orthrus_consensus(const float *logits, const int32_t *proposed, int B, int K, int V,
                      int32_t *accepted_len, int32_t *next_token, int32_t *argmax_out,
                      void *workspace, size_t workspace_bytes, int32_t *status, void *stream)
{
    if (!logits || !proposed || !accepted_len || !next_token) return ORTHRUS_ERR_ARG;
    if (B <= 0 || K <= 0 || V <= 0) return ORTHRUS_ERR_ARG;
    if (K > ORTHRUS_MAX_BLOCK || (int64_t)B * K > 65535) return ORTHRUS_ERR_UNSUPPORTED;
    if (!aligned16(logits) || (workspace && !aligned16(workspace))) return ORTHRUS_ERR_ALIGN;
    const int sms = current_sm_count();
    if (sms <= 0) return ORTHRUS_ERR_DEVICE;
    ConsensusArgs a;
    consensus_split(B, K, V, sms, &a.splits, &a.chunk);
    const size_t need = (size_t)B * K * a.splits * sizeof(unsigned long long);
    if (!workspace || workspace_bytes < need) return ORTHRUS_ERR_WORKSPACE;
    a.logits = logits;
    a.proposed = proposed;
    a.accepted = accepted_len;
    a.next_token = next_token;
    a.argmax_out = argmax_out;
    a.ws = static_cast<unsigned long long *>(workspace);
    a.status = status;
    a.B = B;
    a.K = K;
    a.V = V;
    const cudaError_t e = launch_consensus(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

// Rejection workspace: [B] int32 counters (padded to 16 bytes), the chunk
// statistics [B*K, splits] float4, then the residual tile sums [B, ntile].
struct RejectLayout {
    size_t count, stats, tiles, total;
};

static RejectLayout rejection_layout(int B, int K, int V, int splits)
{
    RejectLayout l;
    const size_t ntile = ((size_t)V + 127) / 128;
    l.count = 0;
    l.stats = ((size_t)B * sizeof(int32_t) + 15) & ~(size_t)15;
    l.tiles = l.stats + (size_t)B * K * splits * sizeof(float4);
    l.total = l.tiles + (((size_t)B * ntile * sizeof(float) + 15) & ~(size_t)15);
    return l;
}

size_t orthrus_rejection_workspace_size(int B, int K, int V)
{
    if (B <= 0 || K <= 0 || V <= 0 || K > ORTHRUS_MAX_BLOCK) return 0;
    const int sms = current_sm_count();
    if (sms <= 0) return 0;
    int s, c;
    consensus_split(B, K, V, sms, &s, &c);
    return rejection_layout(B, K, V, s).total;
}

int orthrus_rejection_verify(const float *ar_logits, const float *draft_logits, const int32_t *proposed,
                             const float *u_accept, const float *u_resample, float temperature, int B,
                             int K, int V, int32_t *accepted_len, int32_t *next_token, void *workspace,
                             size_t workspace_bytes, int32_t *status, void *stream)
{
    if (!ar_logits || !draft_logits || !proposed || !u_accept || !u_resample || !accepted_len ||
        !next_token)
        return ORTHRUS_ERR_ARG;
    if (B <= 0 || K <= 0 || V <= 0 || !(temperature > 0.f) || isinf(temperature)) return ORTHRUS_ERR_ARG;
    if (K > ORTHRUS_MAX_BLOCK || V > kMaxRejectTiles * 128 || (int64_t)B * K > 65535)
        return ORTHRUS_ERR_UNSUPPORTED;
    if (!aligned16(ar_logits) || !aligned16(draft_logits) || (workspace && !aligned16(workspace)))
        return ORTHRUS_ERR_ALIGN;
    const int sms = current_sm_count();
    if (sms <= 0) return ORTHRUS_ERR_DEVICE;
    RejectArgs a;
    consensus_split(B, K, V, sms, &a.splits, &a.chunk);
    const RejectLayout lay = rejection_layout(B, K, V, a.splits);
    if (!workspace || workspace_bytes < lay.total) return ORTHRUS_ERR_WORKSPACE;
    // residual pass: about one CTA per SM in total, at least one tile per warp
    const int ntile = (V + 127) / 128;
    int rs = (sms + B - 1) / B;
    const int max_rs = (ntile + 7) / 8;
    if (rs > max_rs) rs = max_rs;
    if (rs < 1) rs = 1;
    a.rtiles = (ntile + rs - 1) / rs;
    a.rsplit = (ntile + a.rtiles - 1) / a.rtiles;
    a.ar = ar_logits;
    a.dr = draft_logits;
    a.proposed = proposed;
    a.u_accept = u_accept;
    a.u_resample = u_resample;
    a.accepted = accepted_len;
    a.next_token = next_token;
    char *w = static_cast<char *>(workspace);
    a.ws_count = reinterpret_cast<int32_t *>(w + lay.count);
    a.ws = reinterpret_cast<float4 *>(w + lay.stats);
    a.ws_tiles = reinterpret_cast<float *>(w + lay.tiles);
    a.status = status;
    a.B = B;
    a.K = K;
    a.V = V;
    a.c = kLog2e / temperature;
    const cudaError_t e = launch_rejection(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

static int fill_layer_ptrs(CommitArgs &a, int num_layers, void *const *k_caches,
                           void *const *v_caches, const void *const *k_blks,
                           const void *const *v_blks, int D)
{
    if (!k_blks || !v_blks || !k_caches || !v_caches) return ORTHRUS_ERR_ARG;
    if ((D * a.elem_bytes) % 16) return ORTHRUS_ERR_UNSUPPORTED;
    for (int l = 0; l < num_layers; ++l) {
        if (!k_caches[l] || !v_caches[l] || !k_blks[l] || !v_blks[l]) return ORTHRUS_ERR_ARG;
        if (!aligned16(k_caches[l]) || !aligned16(v_caches[l]) || !aligned16(k_blks[l]) ||
            !aligned16(v_blks[l]))
            return ORTHRUS_ERR_ALIGN;
        a.k_caches[l] = k_caches[l];
        a.v_caches[l] = v_caches[l];
        a.k_blks[l] = k_blks[l];
        a.v_blks[l] = v_blks[l];
    }
    a.copy = 1;
    return ORTHRUS_OK;
}

static int commit_common(int num_layers, int B, int Hkv, int D, int S_max, int K,
                         orthrus_dtype dtype, CommitArgs &a)
{
    if (num_layers <= 0 || B <= 0 || Hkv <= 0 || D <= 0 || S_max <= 0 || K <= 0 || K > S_max)
        return ORTHRUS_ERR_ARG;
    if (dtype != ORTHRUS_BF16 && dtype != ORTHRUS_F32) return ORTHRUS_ERR_ARG;
    if (num_layers > ORTHRUS_MAX_LAYERS || B > 65535) return ORTHRUS_ERR_UNSUPPORTED;
    memset(&a, 0, sizeof(a));
    a.elem_bytes = dtype == ORTHRUS_BF16 ? 2 : 4;
    a.num_layers = num_layers;
    a.B = B;
    a.Hkv = Hkv;
    a.D = D;
    a.S_max = S_max;
    a.K = K;
    return ORTHRUS_OK;
}

int orthrus_kv_commit(int num_layers, void *const *k_caches, void *const *v_caches,
                      const void *const *k_blks, const void *const *v_blks, int32_t *ctx_lens,
                      const int32_t *accepted_len, int B, int Hkv, int D, int S_max, int K,
                      orthrus_dtype dtype, int32_t *status, void *stream)
{
    if (!ctx_lens || !accepted_len) return ORTHRUS_ERR_ARG;
    CommitArgs a;
    int rc = commit_common(num_layers, B, Hkv, D, S_max, K, dtype, a);
    if (rc != ORTHRUS_OK) return rc;
    if (k_blks) {
        rc = fill_layer_ptrs(a, num_layers, k_caches, v_caches, k_blks, v_blks, D);
        if (rc != ORTHRUS_OK) return rc;
    }
    a.ctx_lens = ctx_lens;
    a.accepted = accepted_len;
    a.status = status;
    const cudaError_t e = launch_kv_commit(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

int orthrus_write_block(int num_layers, void *const *k_caches, void *const *v_caches,
                        const void *const *k_blks, const void *const *v_blks,
                        const int32_t *ctx_lens, int B, int Hkv, int D, int S_max, int K,
                        orthrus_dtype dtype, int32_t *status, void *stream)
{
    if (!ctx_lens) return ORTHRUS_ERR_ARG;
    CommitArgs a;
    int rc = commit_common(num_layers, B, Hkv, D, S_max, K, dtype, a);
    if (rc != ORTHRUS_OK) return rc;
    rc = fill_layer_ptrs(a, num_layers, k_caches, v_caches, k_blks, v_blks, D);
    if (rc != ORTHRUS_OK) return rc;
    a.all_rows = 1;
    a.ctx_lens = const_cast<int32_t *>(ctx_lens);      // read only in this mode
    a.status = status;
    const cudaError_t e = launch_kv_commit(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ERR_LAUNCH;
}

int orthrus_attn_path(int B, int Hq, int Hkv, int D, int K, orthrus_dtype dtype)
{
    if (!attn_shape_ok(B, Hq, Hkv, D, 1, K, dtype)) return ORTHRUS_ERR_ARG;
    if (!attn_shape_supported(Hq, Hkv, D, K)) return ORTHRUS_ERR_UNSUPPORTED;
    const int sms = current_sm_count();
    if (sms <= 0) return ORTHRUS_ERR_DEVICE;
    return plan_attn(B, Hq, Hkv, D, K, dtype, sms).tc ? 1 : 0;
}

}  // extern "C"

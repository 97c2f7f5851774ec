/*
 * orthrus.h — C ABI of liborthrus.so, the B200 (sm_100a) hot path of one Orthrus
 * dual-view diffusion decoding step:
 *
 *   1. orthrus_attn(DIFF)   the diffusion view's attention over the shared KV cache
 *   2. orthrus_attn(AR)     the frozen AR view's verification attention, same cache
 *   3. orthrus_consensus    greedy left-to-right consensus on the AR logits
 *   4. orthrus_kv_commit    keep the accepted prefix; rollback = length truncation
 *
 * Source of the method: "Orthrus: Memory-Efficient Parallel Token Generation via
 * Dual-View Diffusion" (gist.science technical summary), section 2.1 (two
 * attention paths over one shared KV cache), section 2.2 (block mask M_diff),
 * section 2.3 (parallel projection, structural verification, consensus and
 * commitment); Orthrus-Qwen3 (agentlenshq.com blog), "how Orthrus works"
 * (K = 32 tokens per block, single-step denoising, verification pass).
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no memory, keeps no state between calls and never synchronises
 *     the device; work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and the call returns at once.
 *   - Return value: ORTHRUS_OK (0) or a negative ORTHRUS_ERR_* code for errors
 *     found on the host (bad argument, unsupported shape, misalignment, too
 *     small a workspace, launch failure).  Nothing is enqueued on error.
 *   - Errors only the device can see (a ctx_lens value over capacity, an
 *     accepted length out of range, a bounded wait that gave up) are OR-ed into
 *     the caller's int32 `status` word (device pointer, may be NULL) as
 *     ORTHRUS_STATUS_* bits; the affected work is skipped, never trapped.  Read
 *     the word after synchronising the stream.  The word is passed per call
 *     rather than kept inside the library (there is no global
 *     "get status" call): a library-owned word would be shared by every
 *     stream, thread and CUDA graph of the process, while a caller-owned one
 *     can be per stream or per step, is captured in graphs like any other
 *     argument and is cleared by the caller when it chooses.
 *   - No call takes a host-side context-length hint.  The attention work split
 *     is computed on the device from ctx_lens, so ctx_lens never has to be
 *     copied to the host, a whole decode step (attention, consensus, commit)
 *     runs without a host synchronisation, and a captured graph stays valid as
 *     the lengths grow.
 *   - Tensors are dense, row-major, with the layouts stated per argument.
 *   - Block slot i of sequence b sits at absolute position ctx_lens[b] + i;
 *     slot 0 is the anchor.
 *
 * Numerics: bf16 (or fp32) inputs, fp32 accumulation, fp32 attention output.
 */
#ifndef ORTHRUS_H
#define ORTHRUS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols; everything else in the library is hidden. */
#if defined(__GNUC__)
#define ORTHRUS_API __attribute__((visibility("default")))
#else
#define ORTHRUS_API
#endif

typedef enum {
    ORTHRUS_DIFF = 0, /* diffusion view: mask M_diff (context + whole block)  */
    ORTHRUS_AR = 1    /* AR verification view: causal within the block        */
} orthrus_view;

typedef enum {
    ORTHRUS_BF16 = 0,
    ORTHRUS_F32 = 1
} orthrus_dtype;

#define ORTHRUS_OK 0
#define ORTHRUS_ERR_ARG (-1)          /* NULL pointer, non-positive size, bad enum */
#define ORTHRUS_ERR_UNSUPPORTED (-2)  /* shape the kernels do not cover           */
#define ORTHRUS_ERR_ALIGN (-3)        /* pointer not 16-byte aligned              */
#define ORTHRUS_ERR_WORKSPACE (-4)    /* workspace missing or too small           */
#define ORTHRUS_ERR_LAUNCH (-5)       /* CUDA launch / attribute call failed      */
#define ORTHRUS_ERR_DEVICE (-6)       /* no usable sm_100 device / driver entry   */

#define ORTHRUS_STATUS_CAPACITY 0x1   /* ctx_lens[b] < 0 or ctx_lens[b] + K > S_max */
#define ORTHRUS_STATUS_ACCEPT 0x2     /* accepted_len[b] outside [0, K]             */
#define ORTHRUS_STATUS_TIMEOUT 0x4    /* an on-chip pipeline wait gave up          */

/* Largest supported sizes (checked on the host). */
#define ORTHRUS_MAX_HEAD_DIM 256
#define ORTHRUS_MAX_BLOCK 128          /* K */
#define ORTHRUS_MAX_LAYERS 64          /* per orthrus_kv_commit call */

/*
 * orthrus_attn_workspace_size — bytes of scratch orthrus_attn needs for these
 * sizes on the CURRENT device: a 1920-byte block of split-merge flags and
 * counters, then a 40960-byte cache of the per-CTA work split (each CTA's key
 * range, stored with the shape and context lengths it was computed for, so a
 * later call with the same lengths reads it back instead of recomputing it),
 * then the split-KV partials: one fp32 [G*K, D] tile plus G*K log-sum-exp
 * values per (split unit, KV segment) boundary.  Independent of the context
 * lengths.  Returns 0 for invalid sizes.
 */
ORTHRUS_API size_t orthrus_attn_workspace_size(int B, int Hq, int Hkv, int D, int K,
                                   orthrus_dtype dtype);

/*
 * orthrus_attn — one view's attention for one layer.
 *
 * For every sequence b, query head h (KV head g = h / (Hq/Hkv)) and block slot
 * i in [0, K):
 *     out[b,i,h,:] = sum_j softmax_j(scale * <q[b,i,h,:], k_cache[b,g,j,:]>) v_cache[b,g,j,:]
 * over the visible keys j:
 *     DIFF (mask M_diff; section 2.2 rules 1-2): j in [0, ctx_lens[b] + K)
 *          — the clean context before the anchor plus the whole block,
 *          bidirectionally;
 *     AR   (structural verification; section 2.3): j in [0, ctx_lens[b] + i]
 *          — causal within the block.
 *
 *   view      ORTHRUS_DIFF or ORTHRUS_AR.
 *   dtype     element type of q, k_cache, v_cache (bf16 or fp32).
 *   q         [B, K, Hq, D]      this view's block queries.
 *   k_cache   [B, Hkv, S_max, D] shared cache; rows [0, ctx_lens[b]) hold the
 *             committed context, rows [ctx_lens[b], ctx_lens[b]+K) hold THIS
 *             view's block keys (written by the caller before the call).
 *             Rows at and beyond ctx_lens[b]+K are never read.
 *   v_cache   [B, Hkv, S_max, D] same for values.
 *   ctx_lens  [B] int32 committed lengths (device memory, read on the device).
 *   scale     softmax scale; <= 0 selects 1/sqrt(D).
 *   out       [B, K, Hq, D] fp32.
 *   workspace device scratch of at least orthrus_attn_workspace_size() bytes,
 *             16-byte aligned.  Zero-fill it once before its first use
 *             (cudaMemset): its leading counter block must be zero when a call
 *             starts, and every call that completes leaves it zero again; the
 *             work-split cache after it must hold zeros or what earlier calls
 *             of this library wrote there (the rest is scratch, clobbered).  A
 *             call that ended with ORTHRUS_STATUS_TIMEOUT may leave counters
 *             set: zero it again.  Calls that overlap on the device must not
 *             share it.
 *   status    optional device int32 (see ORTHRUS_STATUS_*).  A sequence whose
 *             ctx_lens[b] is negative or leaves no room for the block
 *             (ctx_lens[b] + K > S_max) sets ORTHRUS_STATUS_CAPACITY and its
 *             outputs are left unspecified.
 *
 * Supported: Hq % Hkv == 0; D % 32 == 0, D <= 256; K <= 128; G*K <= 128 for
 * bf16 with D == 128 (tensor-core path); any other accepted shape runs the
 * CUDA-core path.  All pointers 16-byte aligned.
 *
 * Residency: the tensor-core path launches one cooperative grid of at most one
 * CTA per SM whose CTAs merge split partials with each other, so all of them
 * must run at the same time.  The cooperative launch guarantees that: while
 * kernels on other streams hold SMs the grid is scheduled only once it fits,
 * and a device that can never hold it (for example an MPS or green-context
 * partition with fewer SMs than this device reports) fails the launch with
 * ORTHRUS_ERR_LAUNCH instead of stalling.
 */
ORTHRUS_API int orthrus_attn(orthrus_view view, orthrus_dtype dtype, const void *q,
                 const void *k_cache, const void *v_cache,
                 const int32_t *ctx_lens, int B, int Hq, int Hkv, int D,
                 int S_max, int K, float scale, float *out, void *workspace,
                 size_t workspace_bytes, int32_t *status, void *stream);

/*
 * orthrus_prefill_workspace_size — scratch bytes for orthrus_prefill_attn
 * (zero-fill once before first use, as for orthrus_attn).  0 for invalid sizes.
 */
ORTHRUS_API size_t orthrus_prefill_workspace_size(int B, int S, int Hq, int Hkv, int D,
                                                  orthrus_dtype dtype);

/*
 * orthrus_prefill_attn — causal attention over a prompt whose keys and values
 * already sit in the cache: the frozen AR head builds the shared cache's causal
 * representation of the prompt (section 2.1), before any block is decoded.
 *
 *     out[b, s, h, :] = sum_{j <= s} softmax_j(scale * <q[b,s,h,:], k_cache[b,g,j,:]>) v_cache[b,g,j,:]
 *
 * for every sequence b, prompt position s < S and query head h (KV head
 * g = h / (Hq/Hkv)).  It runs as chunked AR-view attention: prompt chunk c of
 * Kc tokens is exactly an AR-view block after c * Kc context tokens, so the
 * chunks of every sequence go to the tensor-core attention kernel as one
 * batch reading their sequence's cache (Kc = the largest power of two with
 * (Hq/Hkv) * Kc <= 128; a ragged tail of S mod Kc tokens is a second launch).
 *
 *   q        [B, S, Hq, D] (bf16 or fp32, as dtype).
 *   k_cache, v_cache  [B, Hkv, S_max, D]; rows [0, S) hold the prompt's keys
 *            and values.  S <= S_max.
 *   out      [B, S, Hq, D] fp32.
 *   workspace >= orthrus_prefill_workspace_size(B, S, Hq, Hkv, D, dtype)
 *            bytes, 16-byte aligned, zero-filled once before first use.
 * Supported shapes and alignment as orthrus_attn.
 */
ORTHRUS_API int orthrus_prefill_attn(orthrus_dtype dtype, const void *q, const void *k_cache,
                                     const void *v_cache, int B, int S, int Hq, int Hkv, int D,
                                     int S_max, float scale, float *out, void *workspace,
                                     size_t workspace_bytes, int32_t *status, void *stream);

/*
 * orthrus_consensus_workspace_size — scratch bytes for orthrus_consensus
 * (one packed (value, index) candidate per vocabulary chunk per row).
 */
ORTHRUS_API size_t orthrus_consensus_workspace_size(int B, int K, int V);

/*
 * orthrus_consensus — greedy consensus (section 2.3 "consensus and
 * commitment": strict left-to-right, a proposal is accepted only while it equals
 * the AR greedy token; at the first mismatch the AR token takes its place).
 *
 *   logits       [B, K, V] fp32 AR-view logits; row i scores the token after
 *                block slot i, i.e. the candidate proposed[b, i].
 *   proposed     [B, K] int32 diffusion-view proposals p_1..p_K.
 *   accepted_len [B] int32 out: a_b = number of leading i with
 *                proposed[b,i] == r[b,i], in [0, K], where
 *                r[b,i] = argmax_v logits[b,i,v] (lowest index wins ties; NaN
 *                ranks above every number, the first NaN wins; +0 == -0).
 *   next_token   [B] int32 out: r[b, min(a_b, K-1)] — the AR correction token
 *                (or, when all K proposals match, the last one), which becomes
 *                the next block's anchor.
 *   argmax_out   optional [B, K] int32 out: r itself (may be NULL).
 *   workspace    >= orthrus_consensus_workspace_size(B, K, V) bytes, 16-byte
 *                aligned, clobbered.
 */
ORTHRUS_API int orthrus_consensus(const float *logits, const int32_t *proposed, int B,
                      int K, int V, int32_t *accepted_len, int32_t *next_token,
                      int32_t *argmax_out, void *workspace,
                      size_t workspace_bytes, int32_t *status, void *stream);

/*
 * orthrus_rejection_workspace_size — scratch bytes for orthrus_rejection_verify
 * (one int32 counter per sequence, one 16-byte (max, sum) pair of both views per
 * vocabulary chunk per row, and one float per 128-token tile of the vocabulary
 * per sequence).
 */
ORTHRUS_API size_t orthrus_rejection_workspace_size(int B, int K, int V);

/*
 * orthrus_rejection_verify — lossless verification at temperature T > 0, the
 * sampling counterpart of orthrus_consensus (the pages evaluate greedy and
 * rejection-sampling decoding -- Orthrus-Qwen3, agentlenshq.com blog,
 * "limitations"; gist.science technical summary, section 4 -- without giving
 * the rule; this is the standard speculative-sampling rule, which leaves the
 * AR head's distribution unchanged).
 *
 * For sequence b, left to right over block slots i, with p = softmax(
 * ar_logits[b, i, :] / T), q = softmax(draft_logits[b, i, :] / T) and x =
 * proposed[b, i]:
 *     x is kept  iff  u_accept[b, i] * q(x) < p(x)   (probability min(1, p/q));
 * a proposal outside [0, V) is never kept.  accepted_len[b] = number of leading
 * slots kept, in [0, K].  At the first rejection a, next_token[b] is drawn from
 * the residual r(v) = max(0, p(v) - q(v)) by inverse CDF: the smallest v whose
 * cumulative residual exceeds u_resample[b] * sum_v r(v) (from p itself when the
 * residual is empty).  With all K kept, next_token[b] = proposed[b, K - 1]
 * (the AR view has not scored a token after the block).
 *
 *   ar_logits, draft_logits  [B, K, V] fp32, finite; 16-byte aligned.
 *   proposed     [B, K] int32 (drawn by the caller from q).
 *   u_accept     [B, K] fp32 uniform draws in [0, 1) (the caller's generator).
 *   u_resample   [B] fp32 uniform draws in [0, 1).
 *   temperature  > 0.
 *   workspace    >= orthrus_rejection_workspace_size(B, K, V) bytes, 16-byte
 *                aligned.  Zero-fill it once before its first use: its leading
 *                per-sequence counters must be zero when a call starts, and
 *                every call leaves them zero again (the rest is clobbered).
 *                Calls that overlap on the device must not share it.
 * Supported: K <= ORTHRUS_MAX_BLOCK, V <= 262144, B * K <= 65535.
 * Numerics: fp32 with exp2 on the special-function unit; a decision whose
 * margin is within ~1e-6 relative of its threshold can differ from an exact
 * evaluation.
 */
ORTHRUS_API int orthrus_rejection_verify(const float *ar_logits, const float *draft_logits,
                                         const int32_t *proposed, const float *u_accept,
                                         const float *u_resample, float temperature, int B,
                                         int K, int V, int32_t *accepted_len, int32_t *next_token,
                                         void *workspace, size_t workspace_bytes, int32_t *status,
                                         void *stream);

/*
 * orthrus_kv_commit — commit the accepted prefix of the block for every layer
 * and advance the committed length once (section 2.3: commit the synchronised
 * prefix and truncate the cache; rollback is a length change, no data moves).
 *
 * For each sequence b: n_b = min(accepted_len[b] + 1, K) block slots are kept
 * (the anchor plus the accepted proposals, whose AR-view K/V are exact).
 *   - If k_blks is NULL the block already sits in cache rows
 *     [ctx_lens[b], ctx_lens[b]+K) (the AR view wrote it there) and nothing
 *     is copied.
 *   - Otherwise, for each layer l, block slots 0..n_b-1 of
 *     k_blks[l] / v_blks[l] ([B, K, Hkv, D], the caller's AR staging buffers)
 *     are copied into cache rows [ctx_lens[b], ctx_lens[b]+n_b) of
 *     k_caches[l] / v_caches[l] ([B, Hkv, S_max, D]).
 * Then ctx_lens[b] += n_b (once, not per layer).  Rows past the new length
 * are garbage that the next block overwrites.
 *
 *   num_layers   1..ORTHRUS_MAX_LAYERS; the four pointer arrays are HOST
 *                arrays of num_layers device pointers (ignored when k_blks is
 *                NULL; then k_caches/v_caches may be NULL too).
 *   accepted_len [B] int32 from orthrus_consensus.  A value outside [0, K], or
 *                a ctx_lens[b] that would leave no room (ctx + K > S_max), sets
 *                the matching status bit and sequence b is left untouched.
 */
ORTHRUS_API int orthrus_kv_commit(int num_layers, void *const *k_caches,
                      void *const *v_caches, const void *const *k_blks,
                      const void *const *v_blks, int32_t *ctx_lens,
                      const int32_t *accepted_len, int B, int Hkv, int D,
                      int S_max, int K, orthrus_dtype dtype, int32_t *status,
                      void *stream);

/*
 * orthrus_write_block — install a view's block K/V into the cache tail.
 *
 * The DIFF view's block (anchor + K-1 mask positions) and the AR view's block
 * (anchor + the proposals) each occupy cache rows [ctx_lens[b], ctx_lens[b]+K)
 * while that view's attention runs (section 2.1: both views work on one shared
 * cache; section 2.3: the projected block is routed to the AR head).  For each
 * layer l, all K slots of k_blks[l] / v_blks[l] ([B, K, Hkv, D]) are copied
 * into rows [ctx_lens[b], ctx_lens[b]+K) of k_caches[l] / v_caches[l]
 * ([B, Hkv, S_max, D]).  ctx_lens is only read.  A sequence with no room
 * (ctx_lens[b] < 0 or ctx_lens[b] + K > S_max) sets ORTHRUS_STATUS_CAPACITY
 * and is skipped.  The four pointer arrays are HOST arrays of num_layers
 * device pointers (1..ORTHRUS_MAX_LAYERS); D * element size must be a
 * multiple of 16 bytes.
 */
ORTHRUS_API int orthrus_write_block(int num_layers, void *const *k_caches,
                                    void *const *v_caches, const void *const *k_blks,
                                    const void *const *v_blks, const int32_t *ctx_lens,
                                    int B, int Hkv, int D, int S_max, int K,
                                    orthrus_dtype dtype, int32_t *status, void *stream);

/*
 * orthrus_attn_path — which attention kernel orthrus_attn runs for these sizes
 * on the current device: 1 = tensor-core (tcgen05) path, 0 = CUDA-core path,
 * or a negative ORTHRUS_ERR_* code.
 */
ORTHRUS_API int orthrus_attn_path(int B, int Hq, int Hkv, int D, int K, orthrus_dtype dtype);

/*
 * orthrus_attn_static — orthrus_attn without a caller workspace, for callers
 * that cannot allocate device memory: runtimes whose allocator belongs to
 * another framework, engines that forbid allocation after their memory plan is
 * fixed, or plugins that receive only input and output pointers.  (This entry
 * point is a property of this library; the paper has no counterpart.)
 *
 * Same arguments and results as orthrus_attn, minus workspace and
 * workspace_bytes.  The split-KV scratch is a fixed array inside the library
 * of ORTHRUS_STATIC_SCRATCH_BYTES, held on every GPU that loads the library
 * until the process exits; the call allocates and frees nothing.  Sizes whose
 * orthrus_attn_workspace_size() exceeds that limit are rejected with
 * ORTHRUS_ERR_WORKSPACE (bf16 attention with G*K = 128 and D = 128 fits up to
 * about 100 (sequence, KV head) pairs on a 148-SM B200).  The first call on a
 * device looks up the
 * array's device address while that device is current: make it before any
 * stream capture.  All calls share the array.  Every call first clears the
 * array's split-merge counter block on `stream` (an asynchronous memset, no
 * allocation), so each call starts from the state orthrus_attn requires of a
 * workspace, even after an earlier call ended with ORTHRUS_STATUS_TIMEOUT.
 * Calls that overlap on the GPU (other streams, other host threads) race on
 * the array and must be serialised by the caller.
 */
#define ORTHRUS_STATIC_SCRATCH_BYTES (16u << 20)
ORTHRUS_API int orthrus_attn_static(orthrus_view view, orthrus_dtype dtype, const void *q,
                                    const void *k_cache, const void *v_cache,
                                    const int32_t *ctx_lens, int B, int Hq, int Hkv, int D,
                                    int S_max, int K, float scale, float *out, int32_t *status,
                                    void *stream);

/*
 * orthrus_lm_head_workspace_size — bytes of scratch orthrus_lm_head_consensus
 * needs: one 8-byte running maximum per token row plus a completion counter.
 * Returns 0 for invalid sizes (B * K above ORTHRUS_MAX_LM_ROWS).
 */
#define ORTHRUS_MAX_LM_ROWS 512
ORTHRUS_API size_t orthrus_lm_head_workspace_size(int B, int K);

/*
 * orthrus_lm_head_consensus — the AR view's LM head fused with the greedy
 * consensus (section 2.3 "structural verification": the frozen AR head scores
 * all K block positions in one pass; "consensus and commitment": strict
 * left-to-right acceptance, the AR token replaces the first mismatch).  The
 * [B, K, V] logits are never written to memory.
 *
 * For token row t = b * K + i:
 *     logits[t, v] = sum_d hidden[b, i, d] * lm_head[v, d]   (fp32 accumulation)
 *     r[b, i]      = argmax_v logits[t, v]   (lowest index wins ties; NaN ranks
 *                    above every number, the first NaN wins; +0 == -0)
 * then, exactly as orthrus_consensus: accepted_len[b] = number of leading i
 * with proposed[b, i] == r[b, i], in [0, K]; next_token[b] = r[b, min(a, K-1)].
 *
 *   hidden       [B, K, Hd] bf16: the AR view's final hidden states (after the
 *                model's final norm); row i scores the token after block slot i.
 *   lm_head      [V, Hd] bf16: the output projection, one row per vocabulary
 *                entry (Hd contiguous).
 *   proposed     [B, K] int32 diffusion-view proposals.
 *   accepted_len [B] int32 out; next_token [B] int32 out; argmax_out optional
 *                [B, K] int32 out (r itself, may be NULL).
 *   workspace    >= orthrus_lm_head_workspace_size(B, K) bytes, 16-byte
 *                aligned.  Zero-fill it once before its first use: the call
 *                needs it zero when it starts and leaves it zero when it
 *                completes.  A call that ended with ORTHRUS_STATUS_TIMEOUT may
 *                leave it set: zero it again.  Calls that overlap on the device
 *                must not share it.
 *   status       optional device int32 (ORTHRUS_STATUS_TIMEOUT only).
 *
 * Supported: B * K <= ORTHRUS_MAX_LM_ROWS, Hd a multiple of 64, V < 2^31;
 * hidden, lm_head and workspace 16-byte aligned; sm_100 devices only.
 * Numerics: logits are fp32 sums of exact bf16 products; an argmax whose top
 * two logits differ by less than the fp32 rounding of the row can differ from
 * an exact (fp64) evaluation.
 */
ORTHRUS_API int orthrus_lm_head_consensus(const void *hidden, const void *lm_head,
                                          const int32_t *proposed, int B, int K, int V, int Hd,
                                          int32_t *accepted_len, int32_t *next_token,
                                          int32_t *argmax_out, void *workspace,
                                          size_t workspace_bytes, int32_t *status, void *stream);

/*
 * orthrus_qkv_project — one layer's QKV projection of a view's block, with the
 * block's keys and values written straight into the cache rows that view's
 * attention reads (section 2.3 "parallel projection": the diffusion head
 * projects the anchor and K-1 masks in one forward pass; "structural
 * verification": the filled block runs through the frozen AR head; section
 * 2.1: both views attend over one shared KV cache).  It replaces the
 * projection -> staging buffer -> orthrus_write_block round trip.
 *
 * For token row t = b * K + i (each fp32 sum rounded to bf16, nearest-even):
 *     q_out[b, i, h, :]             = w_q[h*D : (h+1)*D, :] . x[b, i, :]
 *     k_cache[b, g, ctx_b + i, :]   = w_k[g*D : (g+1)*D, :] . x[b, i, :]
 *     v_cache[b, g, ctx_b + i, :]   = w_v[g*D : (g+1)*D, :] . x[b, i, :]
 * with ctx_b = ctx_lens[b]; no other cache row is touched.
 *
 *   x            [B, K, hidden] bf16: the block's hidden states after the
 *                layer's input norm.
 *   w_q          [Hq * D, hidden] bf16; w_k, w_v [Hkv * D, hidden] bf16 (the
 *                layer's projection weights, one row per output feature).
 *   ctx_lens     [B] int32 (device).  A sequence with ctx_lens[b] < 0 or
 *                ctx_lens[b] + K > S_max sets ORTHRUS_STATUS_CAPACITY and its
 *                cache rows are not written.
 *   q_out        [B, K, Hq, D] bf16 out.
 *   k_cache, v_cache  [B, Hkv, S_max, D] bf16, rows [ctx_b, ctx_b + K) written.
 * Model-specific steps between projection and attention that the pages do
 * not describe (per-head RMSNorm of q and k, rotary embedding) are not applied.
 *   workspace    >= orthrus_qkv_workspace_size() bytes, 16-byte aligned,
 *                zero-filled once before first use (its per-tile counters must
 *                be zero when a call starts; every completed call leaves them
 *                zero).  Calls that overlap on the device must not share it.
 * Supported: B * K <= ORTHRUS_MAX_LM_ROWS, hidden a multiple of 64, D a
 * multiple of 16, Hq % Hkv == 0; x, the weights and the workspace 16-byte
 * aligned; sm_100 devices only.
 */
ORTHRUS_API size_t orthrus_qkv_workspace_size(int B, int K, int hidden, int Hq, int Hkv, int D);
ORTHRUS_API int orthrus_qkv_project(const void *x, const void *w_q, const void *w_k,
                                    const void *w_v, const int32_t *ctx_lens, int B, int K,
                                    int hidden, int Hq, int Hkv, int D, int S_max, void *q_out,
                                    void *k_cache, void *v_cache, void *workspace,
                                    size_t workspace_bytes, int32_t *status, void *stream);

/* Human-readable text for an ORTHRUS_* return code (static storage). */
ORTHRUS_API const char *orthrus_error_string(int code);

/* Library ABI version: (major << 16) | minor. */
ORTHRUS_API int orthrus_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ORTHRUS_H */

// Tensor-core dual-view attention for sm_100a: TMA-staged bf16 K/V tiles,
// tcgen05.mma with TMEM accumulators, one query row per softmax thread, and
// split-KV partials merged inside the kernel (one launch per call).
//
// What it computes (Orthrus technical summary, gist.science, sections 2.2 and
// 2.3): for one KV head g of sequence b, the G*K block queries (G query heads
// per KV head, K block slots; row m = i*G + hl) attend over keys [0, C+K) of
// the shared cache (DIFF, mask M_diff) or keys [0, C+i] (AR, causal within the
// block).
//
// Work split: the flattened key space of all (sequence, KV head) segments is
// cut into equal ranges, one per CTA (one CTA per SM, see common.cuh); a CTA's
// range holds one or more pieces (segment intersections).  After a piece the
// softmax warps write its rows, normalised by the row sum: the final output
// when the CTA covers the whole segment, else one split partial (with its
// log2-sum-exp).  After its last piece a CTA that shares a segment waits for
// the segment's other CTAs (a counter in the workspace; all CTAs are resident,
// one per SM) and merges its share of the segment's rows.
//
// Per 128-key tile (two 64-row TMA boxes per tensor):
//   S  = Q K^T      tcgen05.mma kind::f16, M=128, N=64|128, K=128 (8 steps),
//                   A = Q (smem, K-major, 128B swizzle), B = K tile (smem, K-major)
//   softmax         4 warps, thread m owns TMEM lane m: mask, running max with
//                   lazy rescaling (threshold 2^8), exp2, row sum
//   P = P_hi + P_lo two bf16 terms (hi = p truncated to bf16, lo = p - hi
//                   truncated) written to TMEM over the consumed S columns; the
//                   two-term split keeps each weight within 2^-14 relative, where
//                   a single bf16 P (2^-9) would break the 2e-3 * RMS tolerance
//   O += P V        tcgen05.mma kind::f16 with A from TMEM, B = V tile (smem,
//                   MN-major), N = 128 = head_dim, twice (hi, lo)
// Roles: warps 0-3 softmax + output rows, warp 4 TMA producer, warp 5 S MMAs
// (+ TMEM allocation), warp 6 PV MMAs (an MMA issue blocks its thread while
// the tensor pipe is busy, so S and PV each get a thread of their own).
// S is triple-buffered in TMEM (3 x 128 columns) next to the O accumulator
// (128 columns); the query tile, three K stages and three V stages sit in
// shared memory (under a full HBM stream a K tile lands ~2 us after its
// request, longer than two tile periods); after a piece the rings stage the
// output rows for their bulk copies.
// Launched with programmatic dependent launch: barrier setup, TMEM allocation
// and descriptor prefetch overlap the previous kernel; nothing an earlier
// kernel may write (ctx_lens, queries, cache, workspace) is read before
// griddepcontrol.wait.
// Every mbarrier wait is bounded (ORTHRUS_STATUS_TIMEOUT, then drain and exit).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdlib.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace orthrus {
namespace tc {

using namespace sm100;

constexpr int kD = 128;
constexpr int kRows = 128;                  // M of every MMA (G*K <= 128 used)
constexpr int kKStages = 3;
constexpr int kVStages = 3;
constexpr int kSBuf = 3;                    // S can run two tiles ahead of PV
constexpr int kThreads = 224;
constexpr int kBoxKeys = 64;
constexpr uint32_t kHalfBytes = kRows * 128;            // 128 rows x 128 B = 16 KiB
constexpr uint32_t kQBytes = 2 * kHalfBytes;            // 128 query rows x 256 B
constexpr uint32_t kStageBytes = 2 * kHalfBytes;        // 128 keys x 256 B
constexpr uint32_t kBoxBytes = kBoxKeys * 128;          // 8 KiB (64 keys x 64 dims)
constexpr uint32_t kStagePitch = 132;                  // floats per staged O row (conflict-free)
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + kQBytes;
constexpr uint32_t kSmemV = kSmemK + kKStages * kStageBytes;
constexpr uint32_t kSmemBar = kSmemV + kVStages * kStageBytes;
// staging rows for the output bulk copies after a piece, over the rings (idle
// once the piece's last PV has finished; the producer starts the next piece
// only after B_MERGED); the padded pitch keeps the row-per-thread writes free
// of bank conflicts
constexpr uint32_t kSmemStage = kSmemK;
static_assert(kSmemStage + kRows * kStagePitch * 4 <= kSmemBar, "staging rows fit in the rings");
// split merge, after the last piece, over the idle query tile and rings: the
// gathered partial rows (n x nr rows of D floats, n * nr < rows + n <= 128 +
// kMaxSyncUnits), their log2-sum-exp runs (n x nl floats, nl <= nr + 6) and
// two weight rows per warp (8 x n floats)
constexpr uint32_t kSmemGather = kSmemQ;
static_assert(kSmemGather + (kRows + kMaxSyncUnits) * kD * 4 + (kRows + 7 * kMaxSyncUnits) * 4 + 16 +
                      8 * kMaxSyncUnits * 4 <= kSmemBar,
              "split merge fits in the rings");

enum : int {
    B_QFULL = 0,    // tx: the piece's query tile has landed
    B_QEMPTY,       // the piece's S MMAs are done with it
    B_KFULL,
    B_KEMPTY = B_KFULL + kKStages,
    B_VFULL = B_KEMPTY + kKStages,
    B_VEMPTY = B_VFULL + kVStages,
    B_SFULL = B_VEMPTY + kVStages,
    B_PFULL = B_SFULL + kSBuf,
    B_PVDONE = B_PFULL + kSBuf,
    B_OFREE = B_PVDONE + kSBuf,
    B_EPI,          // the 128 softmax threads (local, bounded)
    B_MERGED,       // the piece's rows are out: the rings may be refilled
    B_GATHER,       // tx: the split partials of a segment have landed in smem
    B_DRAIN,
    B_DRAIN2,
    B_COUNT
};

constexpr uint32_t kSmemMisc = kSmemBar + B_COUNT * 8;
// (after tmem address and abort flag) the CTA's work plan, then the (at most
// two) pieces of its range whose segments other CTAs share
constexpr uint32_t kSmemPlan = kSmemMisc + 16;
constexpr uint32_t kSmemPend = kSmemPlan + 48;
constexpr uint32_t kSmemUsed = kSmemPend + 2 * 32;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;       // room to align the base to 1 KiB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = kSBuf * 128;                 // 384: O accumulator

static_assert(kSmemAlloc <= 232448, "shared memory budget");

// ---------------------------------------------------------------- work split
// The key space of every (sequence b, KV head g) segment, len_b = ctx_b + K
// keys (0 when ctx_b is out of range), is counted in 64-key boxes, nbx_b =
// ceil(len_b / 64) per segment; all segments are laid end to end in the order
// s = b * Hkv + g and the flat box space [0, NB) is cut into P equal ranges
// (to a box), one per CTA.  A range meets one or more segments; each meeting
// is a piece.  Pieces start on a box boundary of their segment and end on one
// or at the segment's end, so only a segment's last box is ever partial.  In
// every (CTA c, segment s) piece the CTA writes the final rows when it covers
// s alone, else a partial in workspace slot c + s (unique: consecutive CTAs
// share at most one segment).  All of it is 32-bit arithmetic (the host keeps
// B * Hkv * ceil(S_max / 64) below 2^31).
struct Plan {
    int NB;          // boxes over all segments
    int P;           // CTAs with work (P <= grid)
    int q, r;        // NB = q * P + r (range starts: c * q + c * r / P)
    int lo, hi;      // this CTA's box range [lo, hi)
    int b0;          // first sequence whose segments meet the range (B: none)
    int off0;        // flat box offset of sequence b0
    int g0;          // KV head of the range's first piece
    int len0;        // length of sequence b0's segments
};
static_assert(sizeof(Plan) == 40, "plan slot");

__device__ __forceinline__ int nbox_of(int len) { return (len + kBoxKeys - 1) / kBoxKeys; }

__device__ __forceinline__ int plan_start(const Plan &pl, int c) { return c * pl.q + (c * pl.r) / pl.P; }

// The CTA whose range holds flat box x: max{c : plan_start(c) <= x}.
__device__ __forceinline__ int plan_cta_of(const Plan &pl, int x)
{
    return (int)(((int64_t)(x + 1) * pl.P - 1) / pl.NB);
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

struct PlanArgs {
    const int32_t *ctx_lens;
    int32_t *status;
    int B, Hkv, K, S_max;
};

// Computed by all 32 lanes of one warp (lane l reads ctx_lens[l], [l + 32],
// ...); every lane returns the same plan.  CTA 0 also raises
// ORTHRUS_STATUS_CAPACITY for every sequence without room for its block.
__device__ __noinline__ Plan make_plan(const PlanArgs p, int grid, int cid, int min_boxes)
{
    const int lane = threadIdx.x & 31;
    Plan pl;
    int NB = 0, len_first = 0;
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        int len = 0;
        if (b < p.B) {
            len = seg_len(p.ctx_lens, b, p.K, p.S_max);
            if (len == 0 && cid == 0) raise_status(p.status, ORTHRUS_STATUS_CAPACITY);
        }
        if (base == 0) len_first = len;
        NB += __shfl_sync(0xffffffffu, warp_incl_scan(p.Hkv * nbox_of(len), lane), 31);
    }
    pl.NB = NB;
    int P = NB > 0 ? (NB + min_boxes - 1) / min_boxes : 1;
    if (P > grid) P = grid;
    pl.P = P;
    pl.q = NB / P;
    pl.r = NB - pl.q * P;
    pl.lo = plan_start(pl, cid);
    pl.hi = plan_start(pl, cid + 1);
    pl.b0 = p.B;
    pl.off0 = 0;
    pl.g0 = 0;
    pl.len0 = 0;
    if (cid < P && pl.hi > pl.lo) {
        int carry = 0;
        for (int base = 0; base < p.B; base += 32) {
            const int b = base + lane;
            int len = len_first;
            if (base > 0) len = b < p.B ? seg_len(p.ctx_lens, b, p.K, p.S_max) : 0;
            const int nb = p.Hkv * nbox_of(len);
            const int incl = warp_incl_scan(nb, lane);
            const int start = carry + incl - nb;
            const unsigned hit = __ballot_sync(0xffffffffu, nb > 0 && start <= pl.lo && pl.lo < start + nb);
            if (hit) {
                const int l = __ffs(hit) - 1;
                pl.b0 = base + l;
                pl.off0 = __shfl_sync(0xffffffffu, start, l);
                pl.len0 = __shfl_sync(0xffffffffu, len, l);
                pl.g0 = (pl.lo - pl.off0) / nbox_of(pl.len0);
                break;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    return pl;
}

// Cached plans (in the workspace): entry c, for CTA c, holds
//   [0] tag, [1] B, [2] Hkv, [3] K, [4] S_max, [5] grid, [6] min_boxes, [7] 0,
//   [8, 8 + B) the ctx_lens values the plan was computed for, [40, 50) the plan.
// Each CTA reads and writes only its own entry; a later call sees what an
// earlier one wrote (griddepcontrol.wait / stream order).
constexpr int kPlanTag = 0x4F525448;
constexpr int kPlanAt = 40;
static_assert(kPlanAt + 10 <= kPlanEntryInts && 8 + kPlanMaxB <= kPlanAt, "plan entry layout");

// The CTA's plan, by all 32 lanes of one warp: the cached entry when its key
// and lengths match the live ones (one round of loads), else computed and
// cached.  Lane 0 stores it to *out.
__device__ __noinline__ void plan_prologue(const PlanArgs p, int32_t *cache, int grid, int cid,
                                           int min_boxes, Plan *out)
{
    const int lane = threadIdx.x & 31;
    int32_t *e = cache + (size_t)cid * kPlanEntryInts;
    if (p.B <= kPlanMaxB) {
        // ints [0, 52) of the entry, 16 bytes per lane, and the live lengths
        int4 w = make_int4(0, 0, 0, 0);
        if (lane < 13) w = *reinterpret_cast<const int4 *>(e + 4 * lane);
        const int live = lane < p.B ? __ldg(p.ctx_lens + lane) : 0;
        const int src = 2 + (lane >> 2), comp = lane & 3;      // cached length of sequence `lane`
        const int cx = __shfl_sync(0xffffffffu, w.x, src), cy = __shfl_sync(0xffffffffu, w.y, src);
        const int cz = __shfl_sync(0xffffffffu, w.z, src), cw = __shfl_sync(0xffffffffu, w.w, src);
        const int cached = comp == 0 ? cx : comp == 1 ? cy : comp == 2 ? cz : cw;
        bool bad = lane < p.B && cached != live;
        if (lane == 0) bad |= w.x != kPlanTag || w.y != p.B || w.z != p.Hkv || w.w != p.K;
        if (lane == 1) bad |= w.x != p.S_max || w.y != grid || w.z != min_boxes;
        if (!__any_sync(0xffffffffu, bad)) {
            // hit: the plan is ints [40, 50): lanes 10, 11 and 12
            int v[12];
            const int4 a = make_int4(__shfl_sync(0xffffffffu, w.x, 10), __shfl_sync(0xffffffffu, w.y, 10),
                                     __shfl_sync(0xffffffffu, w.z, 10), __shfl_sync(0xffffffffu, w.w, 10));
            const int4 b = make_int4(__shfl_sync(0xffffffffu, w.x, 11), __shfl_sync(0xffffffffu, w.y, 11),
                                     __shfl_sync(0xffffffffu, w.z, 11), __shfl_sync(0xffffffffu, w.w, 11));
            const int c0 = __shfl_sync(0xffffffffu, w.x, 12), c1 = __shfl_sync(0xffffffffu, w.y, 12);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
            v[8] = c0; v[9] = c1;
            if (lane == 0) {
                Plan pl;
                pl.NB = v[0]; pl.P = v[1]; pl.q = v[2]; pl.r = v[3]; pl.lo = v[4]; pl.hi = v[5];
                pl.b0 = v[6]; pl.off0 = v[7]; pl.g0 = v[8]; pl.len0 = v[9];
                *out = pl;
            }
            // (capacity errors are raised again on every call, not cached)
            if (cid == 0 && lane < p.B && seg_len(p.ctx_lens, lane, p.K, p.S_max) == 0)
                raise_status(p.status, ORTHRUS_STATUS_CAPACITY);
            return;
        }
    }
    const Plan pl = make_plan(p, grid, cid, min_boxes);
    if (lane == 0) *out = pl;
    if (p.B <= kPlanMaxB) {
        if (lane < p.B) e[8 + lane] = __ldg(p.ctx_lens + lane);
        if (lane == 0) {
            *reinterpret_cast<int4 *>(e) = make_int4(kPlanTag, p.B, p.Hkv, p.K);
            *reinterpret_cast<int4 *>(e + 4) = make_int4(p.S_max, grid, min_boxes, 0);
            *reinterpret_cast<int4 *>(e + kPlanAt) = make_int4(pl.NB, pl.P, pl.q, pl.r);
            *reinterpret_cast<int4 *>(e + kPlanAt + 4) = make_int4(pl.lo, pl.hi, pl.b0, pl.off0);
            *reinterpret_cast<int2 *>(e + kPlanAt + 8) = make_int2(pl.g0, pl.len0);
        }
    }
}

// One piece: segment (b, g) meets the CTA's range in keys [a, e).
struct TPiece {
    int b, g, s;     // sequence, KV head, segment index b * Hkv + g
    int len;         // segment length in keys
    int a, e;        // keys [a, e) of the segment, 0 <= a < e <= len, a a multiple of 64
    int s0, nbx;     // flat box start of the segment, its box count
};

// Iterates the pieces of the CTA's range in flat order (from the plan).
struct BoxIter {
    const int32_t *ctx;
    int B, Hkv, K, S_max;
    int lo, hi, b, g, off, nbx, len;

    __device__ __forceinline__ BoxIter(const Plan &pl, const AttnArgs &p)
        : ctx(p.ctx_lens), B(p.B), Hkv(p.Hkv), K(p.K), S_max(p.S_max), lo(pl.lo), hi(pl.hi), b(pl.b0),
          g(pl.g0), off(pl.off0), nbx(nbox_of(pl.len0)), len(pl.len0)
    {
    }

    __device__ __forceinline__ bool next(TPiece &pc)
    {
        while (b < B) {
            if (nbx == 0 || g >= Hkv) {
                off += Hkv * nbx;
                ++b;
                g = 0;
                len = b < B ? seg_len(ctx, b, K, S_max) : 0;
                nbx = nbox_of(len);
                continue;
            }
            const int s0 = off + g * nbx;
            if (s0 >= hi) return false;
            const int A = lo > s0 ? lo : s0, E = hi < s0 + nbx ? hi : s0 + nbx;
            pc.b = b;
            pc.g = g;
            pc.s = b * Hkv + g;
            pc.len = len;
            pc.s0 = s0;
            pc.nbx = nbx;
            pc.a = (A - s0) * kBoxKeys;
            pc.e = (E - s0) * kBoxKeys < len ? (E - s0) * kBoxKeys : len;
            ++g;
            if (E > A) return true;
        }
        return false;
    }
};

// The same, not inlined: the softmax warps' iterator then lives in local
// memory (touched once per piece) instead of holding registers through the
// tile loop, where the softmax needs every register it can get.
__device__ __noinline__ bool next_piece(BoxIter &it, TPiece &pc) { return it.next(pc); }

// ---------------------------------------------------------------- tiling
// A piece [a, e) is read in 64-key boxes; box k starts at a + 64k except the
// last, which is right-aligned to end at e (it may overlap the previous box or
// start below 0, where TMA fills zeros), so no key at or past e is ever read.
// Tiles take the boxes two at a time (the last tile may hold one).
struct Tiling {
    int a, e, nbox, skip;     // skip: leading rows of the last box to mask
    int ntile;
    __device__ __forceinline__ Tiling(int a_, int e_) : a(a_), e(e_)
    {
        nbox = (e - a + kBoxKeys - 1) / kBoxKeys;
        skip = a + kBoxKeys * nbox - e;
        ntile = (nbox + 1) / 2;
    }
    __device__ __forceinline__ int box_start(int k) const
    {
        return k < nbox - 1 ? a + kBoxKeys * k : e - kBoxKeys;
    }
    __device__ __forceinline__ int boxes_in_tile(int t) const { return nbox - 2 * t >= 2 ? 2 : 1; }
    __device__ __forceinline__ int box_of(int t, int kb) const { return 2 * t + kb; }
};

// A segment shared with other CTAs: the n CTAs [c_lo, c_lo + n) hold its
// partials in workspace slots c_lo + s, ..., c_lo + n - 1 + s.  The segment
// is the last piece of every one of them except the last CTA, c_lo + n - 1,
// for which it is the first piece; it is also that CTA's last piece when
// hi_last (its range ends within the segment).
struct SplitInfo {
    int b, g, s, c_lo, n;
    bool hi_last;
    size_t row0;     // the sequence's first query / output row
};
// What the epilogue records of a shared piece (in shared memory, so that
// nothing stays live in registers across the tile loop).
struct SharedPiece {
    int s0, nbx;     // flat box start and box count of the segment
    int b, g, s;
    int idx;         // position of the piece in the CTA's range
};

struct Shared {
    uint32_t base;                 // shared address of the 1 KiB-aligned window
    volatile int *abort_flag;
    __device__ __forceinline__ uint32_t bar(int i) const { return base + kSmemBar + 8u * i; }
};

// ---------------------------------------------------------------- roles
// Counters shared by the roles: `piece`/`qp` count the pieces of the CTA's
// range (Q loads, MMAs, O use), `kv`/`gt` count tiles.  Every barrier phase
// is awaited in order.

// Per piece: the query tile (2 halves x 128 rows x 128 B, once the previous
// piece's S MMAs are done with it), then the K tiles into the K ring and the V
// tiles into the V ring.  Each ring is filled as soon as it has a free slot (K
// before V when both have), so a V tile never waits for a K slot or the other
// way round.
__device__ __forceinline__ void producer(const Shared &sh, const AttnArgs &p, const Plan &pl,
                                         const CUtensorMap *tq, const CUtensorMap *tk,
                                         const CUtensorMap *tv)
{
    const int G = p.Hq / p.Hkv;
    const uint32_t q_bytes = 2u * 128u * G * p.K;
    BoxIter it(pl, p);
    TPiece pc;
    uint32_t piece = 0, qloads = 0, kq = 0, kv = 0;   // pieces, Q tiles, K tiles, V tiles
    bool ok = true;
    auto slot_free = [&](uint32_t item, int nst, int bempty) {
        const uint32_t n = item / nst;
        return n == 0 || mbar_test(sh.bar(bempty + item % nst), (n - 1) & 1);
    };
    while (ok && it.next(pc)) {
        const Tiling tl(pc.a, pc.e);
        if (piece > 0 && !wait_bar(sh.bar(B_QEMPTY), (piece - 1) & 1, sh.abort_flag, p.status)) {
            ok = false;
            break;
        }
        mbar_expect_tx(sh.bar(B_QFULL), q_bytes);
        const int qy = (int)p.q_row0(pc.b);
        tma_load_3d(sh.base + kSmemQ, tq, sh.bar(B_QFULL), 0, pc.g * G, qy);
        tma_load_3d(sh.base + kSmemQ + kHalfBytes, tq, sh.bar(B_QFULL), 64, pc.g * G, qy);
        ++qloads;
        // the K and V rings held the previous piece's output rows
        if (piece > 0 && !wait_bar(sh.bar(B_MERGED), (piece - 1) & 1, sh.abort_flag, p.status)) {
            ok = false;
            break;
        }
        const int z = p.cache_seq(pc.b) * p.Hkv + pc.g;
        int nk = 0, nv = 0;                      // this piece's K and V tiles issued
        unsigned long long t0 = 0;
        uint32_t idle = 0;
        while (nk < tl.ntile || nv < tl.ntile) {
            bool issued = false;
            for (int pass = 0; pass < 2 && !issued; ++pass) {
                // K first unless the K stream is ahead of the V stream
                const bool use_k = (pass == 0) == (nk <= nv);
                if (use_k && nk < tl.ntile && slot_free(kq, kKStages, B_KEMPTY)) {
                    const uint32_t full = sh.bar(B_KFULL + kq % kKStages);
                    const uint32_t dst = sh.base + kSmemK + (kq % kKStages) * kStageBytes;
                    const int t = nk, nb = tl.boxes_in_tile(t);
                    mbar_expect_tx(full, nb * 2u * kBoxBytes);
                    for (int kb = 0; kb < nb; ++kb) {
                        const int y = tl.box_start(tl.box_of(t, kb));
                        tma_load_3d(dst + kb * kBoxBytes, tk, full, 0, y, z);
                        tma_load_3d(dst + kHalfBytes + kb * kBoxBytes, tk, full, 64, y, z);
                    }
                    ++nk;
                    ++kq;
                    issued = true;
                } else if (!use_k && nv < tl.ntile && slot_free(kv, kVStages, B_VEMPTY)) {
                    const uint32_t full = sh.bar(B_VFULL + kv % kVStages);
                    const uint32_t dst = sh.base + kSmemV + (kv % kVStages) * kStageBytes;
                    const int t = nv, nb = tl.boxes_in_tile(t);
                    mbar_expect_tx(full, nb * 2u * kBoxBytes);
                    for (int kb = 0; kb < nb; ++kb) {
                        const int y = tl.box_start(tl.box_of(t, kb));
                        tma_load_3d(dst + kb * kBoxBytes, tv, full, 0, y, z);
                        tma_load_3d(dst + kHalfBytes + kb * kBoxBytes, tv, full, 64, y, z);
                    }
                    ++nv;
                    ++kv;
                    issued = true;
                }
            }
            if (issued) {
                idle = 0;
            } else {                    // bounded: the same limit as wait_bar
                if (idle == 0) t0 = global_ns();
                if ((++idle & 63u) == 0) {
                    if (*sh.abort_flag) { ok = false; break; }
                    if (global_ns() - t0 > kTimeoutNs) {
                        *sh.abort_flag = 1;
                        raise_status(p.status, ORTHRUS_STATUS_TIMEOUT);
                        ok = false;
                        break;
                    }
                }
                __nanosleep(20);
            }
        }
        ++piece;
    }
    if (!ok) {
        // abort: let every copy already issued land before the CTA exits
        if (qloads) wait_bar_quiet(sh.bar(B_QFULL), (qloads - 1) & 1);
        for (uint32_t s = 0; s < kKStages; ++s) {
            const uint32_t fills = kq / kKStages + (s < kq % kKStages ? 1u : 0u);
            if (fills) wait_bar_quiet(sh.bar(B_KFULL + s), (fills - 1) & 1);
        }
        for (uint32_t s = 0; s < kVStages; ++s) {
            const uint32_t fills = kv / kVStages + (s < kv % kVStages ? 1u : 0u);
            if (fills) wait_bar_quiet(sh.bar(B_VFULL + s), (fills - 1) & 1);
        }
    }
}

// Two MMA threads, each in its own warp, so that a batch of S MMAs and a
// batch of PV MMAs are fed to the tensor pipe independently (an MMA issue
// blocks its thread while the pipe is busy).
//   S thread:  S(t) = Q K(t)^T once K(t) has landed and S buffer t % kSBuf is
//              free again (PV(t - kSBuf) done)
//   PV thread: O += P(t) V(t) once P(t) is written and V(t) has landed (the
//              first PV of a piece also waits until the previous piece's O
//              has been read out)
__device__ __forceinline__ void s_issuer(const Shared &sh, const AttnArgs &p, const Plan &pl,
                                         uint32_t tmem)
{
    BoxIter it(pl, p);
    TPiece pc;
    uint32_t qp = 0, kq = 0, gt = 0;
    bool ok = true;
    while (ok && it.next(pc)) {
        const Tiling tl(pc.a, pc.e);
        if (!wait_bar(sh.bar(B_QFULL), qp & 1, sh.abort_flag, p.status)) { ok = false; break; }
        for (int t = 0; t < tl.ntile; ++t, ++kq, ++gt) {
            const uint32_t st = kq % kKStages, n = kq / kKStages, buf = gt % kSBuf;
            if (!wait_bar(sh.bar(B_KFULL + st), n & 1, sh.abort_flag, p.status) ||
                (gt >= kSBuf && !wait_bar(sh.bar(B_PVDONE + buf), (gt / kSBuf - 1) & 1, sh.abort_flag, p.status))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t idesc_s = instr_desc(128, 64 * tl.boxes_in_tile(t), false);
            const uint64_t kd = smem_desc(sh.base + kSmemK + st * kStageBytes, 16, 1024);
            const uint64_t qd = smem_desc(sh.base + kSmemQ, 16, 1024);
            const uint32_t dcol = tmem + buf * 128;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {   // 16 head dims per step
                const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
                tc_mma_ss(dcol, qd + off, kd + off, idesc_s, kk > 0);
            }
            tc_commit(sh.bar(B_SFULL + buf));
            tc_commit(sh.bar(B_KEMPTY + st));
            if (t == tl.ntile - 1) tc_commit(sh.bar(B_QEMPTY));
        }
        ++qp;
    }
    if (!ok) {                          // abort: wait for every MMA issued so far
        tc_commit(sh.bar(B_DRAIN));
        wait_bar_quiet(sh.bar(B_DRAIN), 0);
    }
}

__device__ __forceinline__ void pv_issuer(const Shared &sh, const AttnArgs &p, const Plan &pl,
                                          uint32_t tmem)
{
    const uint32_t idesc_pv = instr_desc(128, 128, true);
    BoxIter it(pl, p);
    TPiece pc;
    uint32_t qp = 0, kv = 0, gt = 0;
    bool ok = true;
    while (ok && it.next(pc)) {
        const Tiling tl(pc.a, pc.e);
        for (int t = 0; t < tl.ntile; ++t, ++kv, ++gt) {
            const uint32_t st = kv % kVStages, n = kv / kVStages, buf = gt % kSBuf;
            if (!wait_bar(sh.bar(B_PFULL + buf), (gt / kSBuf) & 1, sh.abort_flag, p.status) ||
                !wait_bar(sh.bar(B_VFULL + st), n & 1, sh.abort_flag, p.status) ||
                (t == 0 && qp > 0 && !wait_bar(sh.bar(B_OFREE), (qp - 1) & 1, sh.abort_flag, p.status))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // 16 keys per step (+2048 B of V, +8 columns of P)
            const uint64_t vd = smem_desc(sh.base + kSmemV + st * kStageBytes, kHalfBytes, 1024);
            const uint32_t pcol = tmem + buf * 128, ocol = tmem + kColO;
            const uint32_t acc0 = t == 0 ? 0u : 1u;
            if (tl.boxes_in_tile(t) == 2) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc_mma_ts(ocol, pcol + 8 * kk, vd + kk * 128, idesc_pv, kk == 0 ? acc0 : 1u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    tc_mma_ts(ocol, pcol + 64 + 8 * kk, vd + kk * 128, idesc_pv, 1u);
            } else {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_ts(ocol, pcol + 8 * kk, vd + kk * 128, idesc_pv, kk == 0 ? acc0 : 1u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_ts(ocol, pcol + 64 + 8 * kk, vd + kk * 128, idesc_pv, 1u);
            }
            tc_commit(sh.bar(B_VEMPTY + st));
            tc_commit(sh.bar(B_PVDONE + buf));
        }
        ++qp;
    }
    if (!ok) {
        tc_commit(sh.bar(B_DRAIN2));
        wait_bar_quiet(sh.bar(B_DRAIN2), 0);
    }
}

// Softmax of one S tile row (this thread's row), written back as P_hi / P_lo.
// P_hi = p with the low 16 mantissa bits dropped (exactly a bf16 value),
// P_lo = (p - P_hi) likewise; p - (P_hi + P_lo) < 2^-14 p.  Both halves are
// packed two keys per 32-bit TMEM column (even key in the low half) with a
// byte permute, so no conversion instruction is needed.
__device__ __forceinline__ float softmax_tile(uint32_t (&s)[128], int nb, float sl2, float mb,
                                              uint32_t p_addr)
{
    float2 lsum = make_float2(0.f, 0.f);
    const float2 sc = make_float2(sl2, sl2), nm = make_float2(-mb, -mb);
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
        if (ch < 2 * nb) {
            uint32_t hi[16], lo[16];
            float2 pe[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                pe[j] = ffma2(make_float2(__uint_as_float(s[32 * ch + 2 * j]),
                                          __uint_as_float(s[32 * ch + 2 * j + 1])),
                              sc, nm);
#pragma unroll
            for (int j = 0; j < 16; ++j) pe[j] = make_float2(fast_exp2(pe[j].x), fast_exp2(pe[j].y));
            float2 l2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                lsum = fadd2(lsum, pe[j]);
                l2 = fadd2(l2, pe[j + 1]);
            }
            lsum = fadd2(lsum, l2);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint32_t u0 = __float_as_uint(pe[j].x), u1 = __float_as_uint(pe[j].y);
                hi[j] = __byte_perm(u0, u1, 0x7632);
                const float2 r = fsub2(pe[j], make_float2(__uint_as_float(u0 & 0xFFFF0000u),
                                                          __uint_as_float(u1 & 0xFFFF0000u)));
                lo[j] = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
            }
            tmem_st16(p_addr + 16 * ch, hi);
            tmem_st16(p_addr + 64 + 16 * ch, lo);
        }
    }
    return lsum.x + lsum.y;
}

// Merge of one shared segment, by CTA cid (see softmax_epilogue).  Every
// partial is published by its row-warps (flag += 1 each, release).  Lane q of
// warp 0 watches the flag of the segment's CTA c_lo + q and, once it is
// complete, gathers that partial's share of rows for this CTA (nr rows from
// r_lo, stored with the 16-byte-chunk swizzle of the epilogue) and their
// log2-sum-exp values into shared memory with bulk copies, so the gather
// overlaps the wait for the segment's slowest CTA.  Once every flag has been
// seen the CTA departs (depart[c_lo] += 1; the last to depart clears the
// segment's flags and the counter for the next call).  Each warp then merges
// whole rows, two at a time: lanes compute the weights 2^(lse_q - max) / sum
// of the rows' partials (the log-sum-exp merge of flash-decoding), then lane
// c4 accumulates 16-byte column c4 over the partials and stores it.
// Returns the B_GATHER phases used (0 or 1), or -1 after an abort.
__device__ __noinline__ int split_merge(uint32_t base, volatile int *abort_flag, uint8_t *smem,
                                        int32_t *ws_sync, const float *ws_o, const float *ws_lse,
                                        float *out, int32_t *status, SplitInfo sp, int cid, int rows,
                                        int G, int K, int Hq, uint32_t gph)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar = base + kSmemBar + 8u * B_GATHER;
    const int lp = lse_pitch(rows);
    const int j = cid - sp.c_lo;
    const int r_lo = j * rows / sp.n, nr = (j + 1) * rows / sp.n - r_lo;
    // each partial's log2-sum-exp run covering this CTA's rows, 16-byte aligned
    const int l_lo = r_lo & ~3;
    const int nl = ((r_lo + nr + 3) & ~3) - l_lo;                       // lse floats per partial
    const uint32_t o_bytes = (uint32_t)nr * kD * 4, l_bytes = (uint32_t)nl * 4;
    const uint32_t s_lse = kSmemGather + (uint32_t)sp.n * o_bytes;     // after the O rows
    const uint32_t s_w = s_lse + (((uint32_t)sp.n * l_bytes + 15u) & ~15u);   // [4 warps][2][n] weights
    const int c_hi = sp.c_lo + sp.n - 1;
    const int nw = (rows + 31) >> 5;                                    // row-warps per partial
    // the flag CTA c of the segment sets: its last piece's, except for c_hi
    // when the segment is its first piece but not its last
    auto flag_of = [&](int c) {
        return ws_sync + ((c == c_hi && !sp.hi_last) ? kSyncFirst : kSyncLast) * kMaxSyncUnits + c;
    };
    bool ok = true;
    if (warp == 0) {
        if (nr > 0) {
            if (lane == 0) mbar_expect_tx(bar, (uint32_t)sp.n * (o_bytes + l_bytes));
            __syncwarp();
            for (int q = lane; q < sp.n; q += 32) {
                const int32_t *flag = flag_of(sp.c_lo + q);
                if (counter_load_relaxed(flag) < nw) {
                    const unsigned long long t0 = global_ns();
                    while (counter_load_relaxed(flag) < nw) {
                        if (*abort_flag || global_ns() - t0 > kTimeoutNs) {
                            *abort_flag = 1;
                            raise_status(status, ORTHRUS_STATUS_TIMEOUT);
                            ok = false;
                            break;
                        }
                    }
                }
                if (!ok) break;
                // (the fence after the relaxed read that saw the releases orders
                // the partial's writes before this lane's later reads; the
                // proxy fence extends that to its bulk reads)
                fence_acquire_gpu();
                fence_proxy_async_global();
                const size_t slot = (size_t)sp.c_lo + q + sp.s;
                bulk_load(base + kSmemGather + q * o_bytes, ws_o + (slot * rows + r_lo) * kD, o_bytes, bar);
                bulk_load(base + s_lse + q * l_bytes, ws_lse + slot * lp + l_lo, l_bytes, bar);
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        // every lane has seen its flags: depart; the last CTA to leave clears them
        int last = 0;
        if (ok && lane == 0)
            last = counter_fetch_add_acq_rel(ws_sync + kSyncDepart * kMaxSyncUnits + sp.c_lo, 1) == sp.n - 1;
        if (__shfl_sync(0xffffffffu, last, 0)) {
            for (int q = lane; q < sp.n; q += 32) *flag_of(sp.c_lo + q) = 0;
            if (lane == 0) ws_sync[kSyncDepart * kMaxSyncUnits + sp.c_lo] = 0;
        }
    }
    if (nr == 0) return ok ? 0 : -1;
    if (!ok || !wait_bar(bar, gph & 1, abort_flag, status)) {
        if (warp == 0) wait_bar_quiet(bar, gph & 1);          // let the copies issued land
        return -1;
    }
    const float4 *gbuf = reinterpret_cast<const float4 *>(smem + kSmemGather);
    const float *glse = reinterpret_cast<const float *>(smem + s_lse) + (r_lo - l_lo);
    float *wsm = reinterpret_cast<float *>(smem + s_w) + warp * 2 * sp.n;
    // each warp merges rows r and r + 4 together (two independent chains)
    for (int r = warp; r < nr; r += 8) {
        const int r1 = r + 4 < nr ? r + 4 : r;              // (a repeat is not stored)
        float M0 = -INFINITY, M1 = -INFINITY;
        for (int q = lane; q < sp.n; q += 32) {
            M0 = fmaxf(M0, glse[q * nl + r]);
            M1 = fmaxf(M1, glse[q * nl + r1]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            M0 = fmaxf(M0, __shfl_xor_sync(0xffffffffu, M0, o));
            M1 = fmaxf(M1, __shfl_xor_sync(0xffffffffu, M1, o));
        }
        float L0 = 0.f, L1 = 0.f;
        for (int q = lane; q < sp.n; q += 32) {
            const float l0 = glse[q * nl + r], l1 = glse[q * nl + r1];
            const float w0 = l0 == -INFINITY ? 0.f : fast_exp2(l0 - M0);   // a partial that
            const float w1 = l1 == -INFINITY ? 0.f : fast_exp2(l1 - M1);   // saw no key
            wsm[q] = w0;
            wsm[sp.n + q] = w1;
            L0 += w0;
            L1 += w1;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            L0 += __shfl_xor_sync(0xffffffffu, L0, o);
            L1 += __shfl_xor_sync(0xffffffffu, L1, o);
        }
        __syncwarp();
        const float inv0 = L0 > 0.f ? 1.f / L0 : 0.f, inv1 = L1 > 0.f ? 1.f / L1 : 0.f;
        float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
        float2 b0 = make_float2(0.f, 0.f), b1 = make_float2(0.f, 0.f);
        // partial rows are stored with chunk c of row m at position c ^ (m & 7)
        const float4 *v = gbuf + r * 32 + (lane ^ ((r_lo + r) & 7));
        const float4 *u = gbuf + r1 * 32 + (lane ^ ((r_lo + r1) & 7));
#pragma unroll 4
        for (int q = 0; q < sp.n; ++q, v += nr * 32, u += nr * 32) {
            const float2 w = make_float2(wsm[q], wsm[q]), z = make_float2(wsm[sp.n + q], wsm[sp.n + q]);
            const float4 x = *v, y = *u;
            a0 = ffma2(make_float2(x.x, x.y), w, a0);
            a1 = ffma2(make_float2(x.z, x.w), w, a1);
            b0 = ffma2(make_float2(y.x, y.y), z, b0);
            b1 = ffma2(make_float2(y.z, y.w), z, b1);
        }
        __syncwarp();                                         // wsm is rewritten next
        int row = r_lo + r;
        float *dst = out + ((sp.row0 + row / G) * Hq + sp.g * G + row % G) * kD;
        reinterpret_cast<float4 *>(dst)[lane] = make_float4(a0.x * inv0, a0.y * inv0, a1.x * inv0, a1.y * inv0);
        if (r1 != r) {
            row = r_lo + r1;
            dst = out + ((sp.row0 + row / G) * Hq + sp.g * G + row % G) * kD;
            reinterpret_cast<float4 *>(dst)[lane] = make_float4(b0.x * inv1, b0.y * inv1, b1.x * inv1, b1.y * inv1);
        }
    }
    return 1;
}

__device__ __forceinline__ bool softmax_epilogue(const Shared &sh, uint8_t *smem, const AttnArgs &p,
                                                 const Plan &pl, int cid, uint32_t tmem)
{
    const int warp = threadIdx.x >> 5;          // 0..3 = TMEM lane quarter
    const int lane = threadIdx.x & 31;
    const int m = warp * 32 + lane;             // query row of this thread
    const int G = p.Hq / p.Hkv;
    const int rows = G * p.K;
    const bool row_ok = m < rows;
    const bool warp_ok = warp * 32 < rows;
    const int i = m / G;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = p.scale_log2;

    BoxIter it(pl, p);
    TPiece pc;
    uint32_t gt = 0, qp = 0, piece = 0, epi = 0;
    int npend = 0;                               // shared segments awaiting the merge
    uint32_t gph = 0;                            // B_GATHER phases used
    // all 128 softmax threads meet here; bounded, unlike a named barrier
    auto epi_sync = [&]() -> bool {
        mbar_arrive(sh.bar(B_EPI));
        const bool ok = wait_bar(sh.bar(B_EPI), epi & 1, sh.abort_flag, p.status);
        ++epi;
        return ok;
    };
    while (next_piece(it, pc)) {
        const int C = pc.len - p.K;
        const int lim = p.view == ORTHRUS_AR ? C + i : 0x7FFFFFFF;   // last visible key
        const Tiling tl(pc.a, pc.e);
        float m_run = -INFINITY, l_run = 0.f;
        for (int t = 0; t < tl.ntile; ++t, ++gt) {
            const uint32_t buf = gt % kSBuf;
            if (!wait_bar(sh.bar(B_SFULL + buf), (gt / kSBuf) & 1, sh.abort_flag, p.status)) return false;
            tc_fence_after();
            const int nb = tl.boxes_in_tile(t);
            if (warp_ok) {
                uint32_t s[128];
                tmem_ld32(lane_base + buf * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(s));
                tmem_ld32(lane_base + buf * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
                if (nb == 2) {
                    tmem_ld32(lane_base + buf * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(s + 64));
                    tmem_ld32(lane_base + buf * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(s + 96));
                }
                tmem_wait_ld();
                // valid key rows of each box: r in [r_lo, r_hi]
                int r_lo[2], r_hi[2];
#pragma unroll
                for (int kb = 0; kb < 2; ++kb) {
                    const int k = tl.box_of(t, kb);
                    const int ks = tl.box_start(k);
                    r_lo[kb] = (k == tl.nbox - 1) ? tl.skip : 0;
                    const long long hi = (long long)lim - ks;
                    r_hi[kb] = hi > 63 ? 63 : (int)hi;
                    if (!row_ok || kb >= nb) { r_lo[kb] = 64; r_hi[kb] = -1; }
                }
                const bool full = r_lo[0] == 0 && r_hi[0] == 63 &&
                                  (nb == 1 || (r_lo[1] == 0 && r_hi[1] == 63));
                if (!full) {
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const int kb = c >> 6, r = c & 63;
                        if (r < r_lo[kb] || r > r_hi[kb]) s[c] = __float_as_uint(-INFINITY);
                    }
                }
                float mx[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
#pragma unroll
                for (int c = 0; c < 64; c += 16) {
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        mx[u] = fmax3(mx[u], __uint_as_float(s[c + 2 * u]), __uint_as_float(s[c + 2 * u + 1]));
                }
                if (nb == 2) {
#pragma unroll
                    for (int c = 64; c < 128; c += 16) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            mx[u] = fmax3(mx[u], __uint_as_float(s[c + 2 * u]), __uint_as_float(s[c + 2 * u + 1]));
                    }
                }
                const float m_tile =
                    fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sl2;
                float factor = 1.f;
                if (m_run == -INFINITY) {
                    m_run = m_tile;                       // first visible keys: O is still zero
                } else if (m_tile > m_run + 8.f) {
                    factor = fast_exp2(m_run - m_tile);   // lazy rescale, rare
                    l_run *= factor;
                    m_run = m_tile;
                }
                if (__any_sync(0xffffffffu, factor != 1.f)) {
                    // O must hold PV(t-1) before it is rescaled (t >= 1 here)
                    const uint32_t pg = gt - 1, pb = pg % kSBuf;
                    if (!wait_bar(sh.bar(B_PVDONE + pb), (pg / kSBuf) & 1, sh.abort_flag, p.status))
                        return false;
                    tc_fence_after();
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t o[32];
                        tmem_ld32(lane_base + kColO + 32 * ch, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
                        tmem_st32(lane_base + kColO + 32 * ch, o);
                    }
                }
                const float mb = m_run == -INFINITY ? 0.f : m_run;
                l_run += softmax_tile(s, nb, sl2, mb, lane_base + buf * 128);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sh.bar(B_PFULL + buf));
        }

        // ---- write the piece's rows: O normalised by the row sum, staged one
        // row per thread in the idle K ring (the piece's MMAs are done) and
        // sent with one bulk copy per row; plus the row's log2-sum-exp when
        // other CTAs hold the rest of the segment (merged after the last piece)
        {
            const uint32_t pg = gt - 1, pb = pg % kSBuf;
            if (!wait_bar(sh.bar(B_PVDONE + pb), (pg / kSBuf) & 1, sh.abort_flag, p.status)) return false;
            tc_fence_after();
        }
        const bool sole = pc.a == 0 && pc.e == pc.len;
        const bool last = pc.s0 + nbox_of(pc.e) == pl.hi;     // the range's last piece
        const size_t slot = (size_t)cid + pc.s;
        if (!sole && npend < 2) {
            // (only the first and the last piece of a range can be shared;
            // kept in shared memory, read back after the last piece)
            if (threadIdx.x == 0) {
                SharedPiece sp;
                sp.s0 = pc.s0;
                sp.nbx = pc.nbx;
                sp.b = pc.b;
                sp.g = pc.g;
                sp.s = pc.s;
                sp.idx = (int)piece;
                reinterpret_cast<SharedPiece *>(smem + kSmemPend)[npend] = sp;
            }
            ++npend;
        }
        if (warp_ok) {
            // a row can see no key of this piece (AR view, piece past C + i):
            // zero output, zero weight in the merge
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            const float2 inv2 = make_float2(inv, inv);
            // the O row in four chunks of 32 columns (TMEM load, wait, scale, stage)
            auto stage_row = [&](float4 *srow, int swz) {
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + kColO + 32 * ch, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const float2 x = fmul2(make_float2(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1])), inv2);
                        const float2 y = fmul2(make_float2(__uint_as_float(o[4 * c + 2]), __uint_as_float(o[4 * c + 3])), inv2);
                        srow[(8 * ch + c) ^ swz] = make_float4(x.x, x.y, y.x, y.y);
                    }
                }
            };
            if (sole) {
                // final rows: padded staging (conflict-free), one bulk copy per row
                stage_row(reinterpret_cast<float4 *>(smem + kSmemStage) + m * (kStagePitch / 4), 0);
                fence_proxy_async();              // the row is visible to the bulk copy
                if (row_ok) {
                    bulk_store(p.out + ((p.q_row0(pc.b) + i) * p.Hq + pc.g * G + m % G) * kD,
                               sh.base + kSmemStage + m * kStagePitch * 4, kD * 4);
                    bulk_commit();
                }
            } else {
                // a partial: rows contiguous in the workspace, staged unpadded
                // with chunk c of row m at position c ^ (m & 7) (conflict-free),
                // one bulk copy per warp; the merge reads the same swizzle
                stage_row(reinterpret_cast<float4 *>(smem + kSmemStage) + m * 32, m & 7);
                fence_proxy_async();              // the rows are visible to the bulk copy
                __syncwarp();
                if (lane == 0) {
                    const int r0 = warp * 32, nrow = rows - r0 < 32 ? rows - r0 : 32;
                    bulk_store(p.ws_o + (slot * rows + r0) * kD, sh.base + kSmemStage + r0 * kD * 4,
                               (uint32_t)nrow * kD * 4);
                    bulk_commit();
                }
                if (row_ok) p.ws_lse[slot * lse_pitch(rows) + m] = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sh.bar(B_OFREE));          // TMEM O may be overwritten
        ++qp;
        if (!sole && warp_ok && lane == 0) {
            // publish this warp's rows of the partial: written (with the warp's
            // log2-sum-exp values, ordered by the __syncwarp above), then its
            // flag += 1 (release); the partial is complete at ceil(rows / 32)
            bulk_wait_all();
            fence_proxy_async_global();
            counter_add_release(p.ws_sync + (last ? kSyncLast : kSyncFirst) * kMaxSyncUnits + cid, 1);
        }
        ++piece;
        if (last) break;                                      // (no next piece: nothing refills the rings)
        bulk_wait_read();                                     // the staging row has been read
        if (!epi_sync()) return false;
        if (threadIdx.x == 0) mbar_arrive(sh.bar(B_MERGED)); // the rings may be refilled
    }
    bulk_wait_all();                                          // rows written
    if (npend == 0) return true;

    // ---- split merge: this CTA's share of the rows of each shared segment
    // (split_merge); the gathers overwrite the staging area, which every
    // warp's copies have read by now (bulk_wait_all above, then this join)
    if (!epi_sync()) return false;
    const Plan plan = *reinterpret_cast<const Plan *>(smem + kSmemPlan);
    auto shared_piece = [&](int k) {
        const SharedPiece sp = reinterpret_cast<const SharedPiece *>(smem + kSmemPend)[k];
        SplitInfo si;
        si.b = sp.b;
        si.g = sp.g;
        si.s = sp.s;
        si.c_lo = plan_cta_of(plan, sp.s0);
        const int c_hi = plan_cta_of(plan, sp.s0 + sp.nbx - 1);
        si.n = c_hi - si.c_lo + 1;
        si.hi_last = plan_start(plan, c_hi + 1) <= sp.s0 + sp.nbx;
        si.row0 = p.q_row0(sp.b);
        return si;
    };
    for (int k = 0; k < npend; ++k) {
        if (k > 0 && !epi_sync()) return false;               // gather buffer free again
        const SplitInfo sp = shared_piece(k);
        const int used = split_merge(sh.base, sh.abort_flag, smem, p.ws_sync, p.ws_o, p.ws_lse, p.out,
                                     p.status, sp, cid, rows, G, p.K, p.Hq, gph);
        if (used < 0) return false;
        gph += used;
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t aligned = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (aligned - raw);
    Shared sh;
    sh.base = aligned;
    sh.abort_flag = reinterpret_cast<volatile int *>(base_ptr + kSmemMisc + 4);
    const int cid = blockIdx.x;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(base_ptr + kSmemMisc);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- prologue: touches nothing an earlier kernel in the stream may write
    pdl_trigger();
    if (threadIdx.x == 0) {
        mbar_init(sh.bar(B_QFULL), 1);
        mbar_init(sh.bar(B_QEMPTY), 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(sh.bar(B_KFULL + s), 1);
            mbar_init(sh.bar(B_KEMPTY + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(sh.bar(B_VFULL + s), 1);
            mbar_init(sh.bar(B_VEMPTY + s), 1);
        }
        for (int s = 0; s < kSBuf; ++s) {
            mbar_init(sh.bar(B_SFULL + s), 1);
            mbar_init(sh.bar(B_PFULL + s), 4);
            mbar_init(sh.bar(B_PVDONE + s), 1);
        }
        mbar_init(sh.bar(B_OFREE), 4);
        mbar_init(sh.bar(B_EPI), 128);
        mbar_init(sh.bar(B_MERGED), 1);
        mbar_init(sh.bar(B_GATHER), 1);
        mbar_init(sh.bar(B_DRAIN), 1);
        mbar_init(sh.bar(B_DRAIN2), 1);
        *sh.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 4 && lane == 0) {
        tma_prefetch(&tm_q);
        tma_prefetch(&tm_k);
        tma_prefetch(&tm_v);
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         aligned + kSmemMisc),
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
    Plan *plan_s = reinterpret_cast<Plan *>(base_ptr + kSmemPlan);
    if (warp == 4) {
        const PlanArgs pa = {p.ctx_lens, p.status, p.B, p.Hkv, p.K, p.S_max};
        plan_prologue(pa, p.ws_plan, gridDim.x, cid, p.min_keys > kBoxKeys ? p.min_keys / kBoxKeys : 1, plan_s);
    }
    __syncthreads();
    const Plan pl = *plan_s;
    if (pl.NB > 0 && cid < pl.P) {
        if (warp < 4) {
            softmax_epilogue(sh, base_ptr, p, pl, cid, tmem);
            bulk_wait_all();                      // (also after an abort)
        } else if (warp == 4) {
            if (lane == 0) producer(sh, p, pl, &tm_q, &tm_k, &tm_v);
            __syncwarp();
        } else if (warp == 5) {
            if (lane == 0) s_issuer(sh, p, pl, tmem);
            __syncwarp();
        } else {
            if (lane == 0) pv_issuer(sh, p, pl, tmem);
            __syncwarp();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace tc

// ---------------------------------------------------------------- host side
namespace {

bool encode_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2)
{
    const uint64_t dims[3] = {d0, d1, d2};
    const uint64_t strides[2] = {s1, s2};
    const uint32_t box[3] = {b0, b1, b2};
    return encode_bf16_sw128(m, 3, base, dims, strides, box);
}

bool device_is_sm100()
{
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    return major == 10 && minor == 0;
}

}  // namespace

bool attn_tc_supported(int dtype, int D, int rows)
{
    return dtype == ORTHRUS_BF16 && D == tc::kD && rows <= tc::kRows && device_is_sm100();
}

namespace {

// CTAs of the split for this device, chosen once per device (thread-safe):
// one CTA per SM (the kernel's shared memory admits no second one).  The
// launch is cooperative, so all of them are resident at once or the launch
// fails; the in-kernel split merge relies on that.
constexpr int kMaxDevices = 64;
std::once_flag g_ctas_once[kMaxDevices];
int g_ctas[kMaxDevices];

int resident_ctas()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::call_once(g_ctas_once[dev], [dev] {
        int sms = 0, per_sm = 0;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaFuncSetAttribute(tc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tc::kSmemAlloc) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tc::attn_tc_kernel, tc::kThreads,
                                                          tc::kSmemAlloc) != cudaSuccess ||
            per_sm < 1) {
            cudaGetLastError();
            return;
        }
        // (capped by the split-merge counter block of the workspace)
        g_ctas[dev] = sms * per_sm < kMaxSyncUnits ? sms * per_sm : kMaxSyncUnits;
    });
    return g_ctas[dev];
}

}  // namespace

bool attn_tc_plan(int *units, int *min_keys)
{
    const int n = resident_ctas();
    if (!n) return false;
    *units = n;
    *min_keys = 128;          // one tile
    return true;
}

cudaError_t launch_attn_tc(const AttnArgs &p, int units, cudaStream_t st)
{
    const int n = resident_ctas();
    if (!n || units < 1 || units > n) return cudaErrorInvalidValue;
    const int G = p.Hq / p.Hkv;
    CUtensorMap tq, tk, tv;
    const uint64_t row = tc::kD * 2;
    const uint64_t q_rows = (uint64_t)((p.B + p.cache_div - 1) / p.cache_div) * p.q_seq_rows;
    const uint64_t kv_seqs = (uint64_t)((p.B + p.cache_div - 1) / p.cache_div) * p.Hkv;
    if (!encode_3d(&tq, p.q, tc::kD, p.Hq, q_rows, row, (uint64_t)p.Hq * row, 64, G, p.K) ||
        !encode_3d(&tk, p.k_cache, tc::kD, p.S_max, kv_seqs, row, (uint64_t)p.S_max * row, 64, 64, 1) ||
        !encode_3d(&tv, p.v_cache, tc::kD, p.S_max, kv_seqs, row, (uint64_t)p.S_max * row, 64, 64, 1))
        return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(units);
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = tc::kSmemAlloc;
    cfg.stream = st;
    // cooperative: every CTA is resident at once (the split merge waits on
    // sibling CTAs), or the launch fails; programmatic dependent launch lets
    // the prologue overlap the previous kernel in the stream
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, tc::attn_tc_kernel, tq, tk, tv, p);
}

}  // namespace orthrus

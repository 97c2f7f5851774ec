// Tensor-core dual-view attention for sm_100a: TMA-staged bf16 K/V tiles,
// tcgen05.mma with TMEM accumulators, one query row per softmax thread.
//
// What it computes (Orthrus technical summary, gist.science, sections 2.2 and
// 2.3): for one KV head g of sequence b, the G*K block queries (G query heads
// per KV head, K block slots; row m = i*G + hl) attend over keys [0, C+K) of
// the shared cache (DIFF, mask M_diff) or keys [0, C+i] (AR, causal within the
// block).  Each CTA takes an equal share of the flattened key space (see
// common.cuh) and produces, per piece, either the final rows or a split
// partial merged by attn_combine_kernel.
//
// Per 128-key tile (two 64-row TMA boxes per tensor):
//   S  = Q K^T      tcgen05.mma kind::f16, M=128, N=64|128, K=128 (8 steps),
//                   A = Q (smem, K-major, 128B swizzle), B = K tile (smem, K-major)
//   softmax         4 warps, thread m owns TMEM lane m: mask, running max with
//                   lazy rescaling (threshold 2^8), exp2, row sum
//   P = P_hi + P_lo two bf16 terms (hi = bf16(p), lo = bf16(p - hi)) written to
//                   TMEM over the consumed S columns; the two-term split keeps
//                   the PV product accurate to ~2^-16 relative, where a single
//                   bf16 P (2^-9) would break the 2e-3 * RMS output tolerance
//   O += P V        tcgen05.mma kind::f16 with A from TMEM, B = V tile (smem,
//                   MN-major), N = 128 = head_dim, twice (hi, lo)
// Roles: warps 0-3 softmax + epilogue, warp 4 TMA producer, warp 5 MMA issuer
// (+ TMEM allocation).  S is triple-buffered in TMEM (3 x 128 columns) next to
// the O accumulator (128 columns); K and V have 3-stage smem rings.
// Every mbarrier wait is bounded (ORTHRUS_STATUS_TIMEOUT, then drain and exit).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace orthrus {
namespace tc {

constexpr int kD = 128;
constexpr int kRows = 128;                  // M of every MMA (G*K <= 128 used)
constexpr int kStages = 3;
constexpr int kSBuf = 3;
constexpr int kThreads = 192;
constexpr int kBoxKeys = 64;
constexpr uint32_t kHalfBytes = kRows * 128;            // 128 rows x 128 B = 16 KiB
constexpr uint32_t kQBytes = 2 * kHalfBytes;            // 32 KiB
constexpr uint32_t kStageBytes = 2 * kHalfBytes;        // 128 keys x 256 B
constexpr uint32_t kBoxBytes = kBoxKeys * 128;          // 8 KiB (64 keys x 64 dims)
constexpr uint32_t kSmemQ = 0;
constexpr uint32_t kSmemK = kSmemQ + kQBytes;
constexpr uint32_t kSmemV = kSmemK + kStages * kStageBytes;
constexpr uint32_t kSmemBar = kSmemV + kStages * kStageBytes;

enum : int {
    B_QFULL = 0,
    B_QEMPTY,
    B_KFULL,
    B_KEMPTY = B_KFULL + kStages,
    B_VFULL = B_KEMPTY + kStages,
    B_VEMPTY = B_VFULL + kStages,
    B_SFULL = B_VEMPTY + kStages,
    B_PFULL = B_SFULL + kSBuf,
    B_PVDONE = B_PFULL + kSBuf,
    B_OFREE = B_PVDONE + kSBuf,
    B_DRAIN,
    B_COUNT
};

constexpr uint32_t kSmemMisc = kSmemBar + B_COUNT * 8;
constexpr uint32_t kSmemUsed = kSmemMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;       // room to align the base to 1 KiB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = kSBuf * 128;                 // 384
constexpr unsigned long long kTimeoutNs = 2000000000ull;

static_assert(kSmemAlloc <= 232448, "shared memory budget");

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait: false when the CTA aborted or this wait ran out of time (the
// latter raises ORTHRUS_STATUS_TIMEOUT and sets the CTA's abort flag).
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                      int32_t *status)
{
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > kTimeoutNs) {
                *abort_flag = 1;
                raise_status(status, ORTHRUS_STATUS_TIMEOUT);
                return false;
            }
        }
    }
}

// Drain wait used on the abort path: bounded, no side effects.
__device__ __noinline__ void wait_bar_quiet(uint32_t bar, uint32_t parity)
{
    const unsigned long long t0 = global_ns();
    while (!mbar_try(bar, parity))
        if (global_ns() - t0 > kTimeoutNs) return;
}

__device__ __forceinline__ void tma_prefetch(const CUtensorMap *m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"((unsigned long long)m) : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                            int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"((unsigned long long)m), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tc_mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void tc_mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                          uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

#define ORTHRUS_R32(r)                                                                        \
    "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),     \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),          \
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),       \
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),       \
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),       \
        "=r"(r[31])

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : ORTHRUS_R32(r)
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float even, float odd)
{
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(odd), "f"(even));
    return d;
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor, 128-byte swizzle (layout code 2), version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, A K-major.
__host__ __device__ constexpr uint32_t instr_desc(int M, int N, bool b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- tiling
// A piece [a, e) is read in 64-key boxes; box k starts at a + 64k except the
// last, which is right-aligned to end at e (it may overlap the previous box or
// start below 0, where TMA fills zeros), so no key at or past e is ever read.
struct Tiling {
    int a, e, nbox, ntile, skip;   // skip: leading rows of the last box to mask
    __device__ __forceinline__ Tiling(int a_, int e_) : a(a_), e(e_)
    {
        nbox = (e - a + kBoxKeys - 1) / kBoxKeys;
        ntile = (nbox + 1) / 2;
        skip = a + kBoxKeys * nbox - e;
    }
    __device__ __forceinline__ int box_start(int k) const
    {
        return k < nbox - 1 ? a + kBoxKeys * k : e - kBoxKeys;
    }
    __device__ __forceinline__ int boxes_in_tile(int t) const
    {
        return nbox - 2 * t >= 2 ? 2 : 1;
    }
};

struct Shared {
    uint32_t base;                 // shared address of the 1 KiB-aligned window
    volatile int *abort_flag;
    __device__ __forceinline__ uint32_t bar(int i) const { return base + kSmemBar + 8u * i; }
};

// ---------------------------------------------------------------- roles
__device__ __forceinline__ void producer(const Shared &sh, const AttnArgs &p, const Decomp &d,
                                         const CUtensorMap *tq, const CUtensorMap *tk,
                                         const CUtensorMap *tv)
{
    const int G = p.Hq / p.Hkv;
    const uint32_t q_bytes = 2u * 128u * G * p.K;
    PieceIter it(p.ctx_lens, p.B, p.Hkv, p.K, p.S_max, d, blockIdx.x);
    Piece pc;
    uint32_t piece = 0, kv = 0;
    bool ok = true;
    while (ok && it.next(pc)) {
        if (piece > 0 && !wait_bar(sh.bar(B_QEMPTY), (piece - 1) & 1, sh.abort_flag, p.status)) {
            ok = false;
            break;
        }
        mbar_expect_tx(sh.bar(B_QFULL), q_bytes);
        tma_load_3d(sh.base + kSmemQ, tq, sh.bar(B_QFULL), 0, pc.g * G, pc.b * p.K);
        tma_load_3d(sh.base + kSmemQ + kHalfBytes, tq, sh.bar(B_QFULL), 64, pc.g * G, pc.b * p.K);
        const Tiling tl(pc.a, pc.e);
        const int z = pc.b * p.Hkv + pc.g;
        for (int t = 0; t < tl.ntile && ok; ++t, ++kv) {
            const int nb = tl.boxes_in_tile(t);
            const uint32_t st = kv % kStages, n = kv / kStages;
            for (int which = 0; which < 2; ++which) {
                const uint32_t full = sh.bar((which ? B_VFULL : B_KFULL) + st);
                const uint32_t empty = sh.bar((which ? B_VEMPTY : B_KEMPTY) + st);
                if (n > 0 && !wait_bar(empty, (n - 1) & 1, sh.abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(full, nb * 2u * kBoxBytes);
                const uint32_t dst = sh.base + (which ? kSmemV : kSmemK) + st * kStageBytes;
                const CUtensorMap *m = which ? tv : tk;
                for (int kb = 0; kb < nb; ++kb) {
                    const int y = tl.box_start(2 * t + kb);
                    tma_load_3d(dst + kb * kBoxBytes, m, full, 0, y, z);
                    tma_load_3d(dst + kHalfBytes + kb * kBoxBytes, m, full, 64, y, z);
                }
            }
        }
        ++piece;
    }
    if (!ok) {
        // abort: let every copy already issued land before the CTA exits
        for (uint32_t s = 0; s < kStages; ++s) {
            const uint32_t fills = kv / kStages + (s < kv % kStages ? 1u : 0u);
            if (fills) {
                wait_bar_quiet(sh.bar(B_KFULL + s), (fills - 1) & 1);
                wait_bar_quiet(sh.bar(B_VFULL + s), (fills - 1) & 1);
            }
        }
        if (piece > 0 || kv > 0) wait_bar_quiet(sh.bar(B_QFULL), piece & 1);
    }
}

__device__ __forceinline__ void mma_issuer(const Shared &sh, const AttnArgs &p, const Decomp &d,
                                           uint32_t tmem)
{
    const uint32_t idesc_pv = instr_desc(128, 128, true);
    PieceIter it(p.ctx_lens, p.B, p.Hkv, p.K, p.S_max, d, blockIdx.x);
    Piece pc;
    uint32_t piece = 0, kv = 0, gt = 0;
    bool ok = true;
    while (ok && it.next(pc)) {
        if (!wait_bar(sh.bar(B_QFULL), piece & 1, sh.abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const Tiling tl(pc.a, pc.e);
        for (int t = 0; t <= tl.ntile && ok; ++t) {
            if (t < tl.ntile) {        // S(t) = Q K(t)^T
                const int nb = tl.boxes_in_tile(t);
                const uint32_t st = (kv + t) % kStages, n = (kv + t) / kStages;
                const uint32_t g = gt + t, buf = g % kSBuf;
                if (!wait_bar(sh.bar(B_KFULL + st), n & 1, sh.abort_flag, p.status)) { ok = false; break; }
                if (g >= kSBuf &&
                    !wait_bar(sh.bar(B_PVDONE + buf), (g / kSBuf - 1) & 1, sh.abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t idesc_s = instr_desc(128, 64 * nb, false);
                const uint32_t kaddr = sh.base + kSmemK + st * kStageBytes;
                const uint32_t qaddr = sh.base + kSmemQ;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    tc_mma_ss(tmem + buf * 128, smem_desc(qaddr + off, 16, 1024),
                              smem_desc(kaddr + off, 16, 1024), idesc_s, kk > 0);
                }
                tc_commit(sh.bar(B_SFULL + buf));
                tc_commit(sh.bar(B_KEMPTY + st));
                if (t == tl.ntile - 1) tc_commit(sh.bar(B_QEMPTY));
            }
            if (t >= 1) {              // O += P(t-1) V(t-1)
                const int tp = t - 1;
                const int nb = tl.boxes_in_tile(tp);
                const uint32_t st = (kv + tp) % kStages, n = (kv + tp) / kStages;
                const uint32_t g = gt + tp, buf = g % kSBuf;
                if (!wait_bar(sh.bar(B_PFULL + buf), (g / kSBuf) & 1, sh.abort_flag, p.status) ||
                    !wait_bar(sh.bar(B_VFULL + st), n & 1, sh.abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                if (tp == 0 && piece > 0 &&
                    !wait_bar(sh.bar(B_OFREE), (piece - 1) & 1, sh.abort_flag, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t vaddr = sh.base + kSmemV + st * kStageBytes;
                const int steps = 4 * nb;
                for (int kk = 0; kk < steps; ++kk)
                    tc_mma_ts(tmem + kColO, tmem + buf * 128 + 8 * kk,
                              smem_desc(vaddr + kk * 2048, kHalfBytes, 1024), idesc_pv,
                              (tp == 0 && kk == 0) ? 0u : 1u);
                for (int kk = 0; kk < steps; ++kk)
                    tc_mma_ts(tmem + kColO, tmem + buf * 128 + 64 + 8 * kk,
                              smem_desc(vaddr + kk * 2048, kHalfBytes, 1024), idesc_pv, 1u);
                tc_commit(sh.bar(B_VEMPTY + st));
                tc_commit(sh.bar(B_PVDONE + buf));
            }
        }
        kv += tl.ntile;
        gt += tl.ntile;
        ++piece;
    }
    if (!ok) {                          // abort: wait for every MMA issued so far
        tc_commit(sh.bar(B_DRAIN));
        wait_bar_quiet(sh.bar(B_DRAIN), 0);
    }
}

__device__ __forceinline__ void softmax_epilogue(const Shared &sh, const AttnArgs &p,
                                                 const Decomp &d, uint32_t tmem)
{
    const int warp = threadIdx.x >> 5;          // 0..3 = TMEM lane quarter
    const int lane = threadIdx.x & 31;
    const int m = warp * 32 + lane;             // query row of this thread
    const int G = p.Hq / p.Hkv;
    const int rows = G * p.K;
    const bool row_ok = m < rows;
    const bool warp_ok = warp * 32 < rows;
    const int i = m / G, hl = m % G;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl2 = p.scale_log2;

    PieceIter it(p.ctx_lens, p.B, p.Hkv, p.K, p.S_max, d, blockIdx.x);
    Piece pc;
    uint32_t piece = 0, gt = 0;
    while (it.next(pc)) {
        const int C = pc.len - p.K;
        const int lim = p.view == ORTHRUS_AR ? C + i : 0x7FFFFFFF;   // last visible key
        const Tiling tl(pc.a, pc.e);
        float m_run = -INFINITY, l_run = 0.f;
        for (int t = 0; t < tl.ntile; ++t, ++gt) {
            const uint32_t buf = gt % kSBuf;
            if (!wait_bar(sh.bar(B_SFULL + buf), (gt / kSBuf) & 1, sh.abort_flag, p.status)) return;
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
                    const int k = 2 * t + kb;
                    const int ks = tl.box_start(k);
                    r_lo[kb] = (k == tl.nbox - 1) ? tl.skip : 0;
                    const long long hi = (long long)lim - ks;
                    r_hi[kb] = hi > 63 ? 63 : (int)hi;
                    if (!row_ok || kb >= nb) { r_lo[kb] = 64; r_hi[kb] = -1; }
                }
                const bool full = r_lo[0] == 0 && r_hi[0] == 63 && (nb == 1 || (r_lo[1] == 0 && r_hi[1] == 63));
                float mx = -INFINITY;
                if (full) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c < 64 * nb) mx = fmaxf(mx, __uint_as_float(s[c]));
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const int kb = c >> 6, r = c & 63;
                        const bool v = r >= r_lo[kb] && r <= r_hi[kb];
                        if (!v) s[c] = __float_as_uint(-INFINITY);
                        mx = fmaxf(mx, __uint_as_float(s[c]));
                    }
                }
                const float m_tile = mx * sl2;
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
                        return;
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
                float lsum = 0.f;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    if (ch < 2 * nb) {
                        uint32_t hi[16], lo[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float p0 = fast_exp2(fmaf(__uint_as_float(s[32 * ch + 2 * j]), sl2, -mb));
                            const float p1 = fast_exp2(fmaf(__uint_as_float(s[32 * ch + 2 * j + 1]), sl2, -mb));
                            lsum += p0 + p1;
                            const uint32_t h = pack_bf16x2(p0, p1);
                            hi[j] = h;
                            lo[j] = pack_bf16x2(p0 - __uint_as_float(h << 16),
                                                p1 - __uint_as_float(h & 0xFFFF0000u));
                        }
                        tmem_st16(lane_base + buf * 128 + 16 * ch, hi);
                        tmem_st16(lane_base + buf * 128 + 64 + 16 * ch, lo);
                    }
                }
                l_run += lsum;
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sh.bar(B_PFULL + buf));
        }
        // epilogue: O of this piece is final once PV(last) has completed
        {
            const uint32_t pg = gt - 1, pb = pg % kSBuf;
            if (!wait_bar(sh.bar(B_PVDONE + pb), (pg / kSBuf) & 1, sh.abort_flag, p.status)) return;
            tc_fence_after();
        }
        if (warp_ok) {
            const bool sole = pc.a == 0 && pc.e == pc.len;
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            float *dst;
            if (sole)
                dst = p.out + (((size_t)pc.b * p.K + i) * p.Hq + pc.g * G + hl) * kD;
            else
                dst = p.ws_o + ((size_t)(blockIdx.x + pc.s) * rows + m) * kD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t o[32];
                tmem_ld32(lane_base + kColO + 32 * ch, o);
                tmem_wait_ld();
                if (row_ok) {
                    float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * ch);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        d4[c] = make_float4(__uint_as_float(o[4 * c]) * inv, __uint_as_float(o[4 * c + 1]) * inv,
                                            __uint_as_float(o[4 * c + 2]) * inv, __uint_as_float(o[4 * c + 3]) * inv);
                }
            }
            if (row_ok && !sole)
                p.ws_lse[(size_t)(blockIdx.x + pc.s) * rows + m] =
                    l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sh.bar(B_OFREE));
        ++piece;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    const Decomp d = make_decomp(p.ctx_lens, p.B, p.Hkv, p.K, p.S_max, gridDim.x, p.min_keys);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int b = 0; b < p.B; ++b)
            if (seg_len(p.ctx_lens, b, p.K, p.S_max) == 0) raise_status(p.status, ORTHRUS_STATUS_CAPACITY);
    }
    if (d.W == 0 || (int)blockIdx.x >= d.P) return;      // uniform per CTA

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t aligned = (raw + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (aligned - raw);
    Shared sh;
    sh.base = aligned;
    sh.abort_flag = reinterpret_cast<volatile int *>(base_ptr + kSmemMisc + 4);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(base_ptr + kSmemMisc);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(sh.bar(B_QFULL), 1);
        mbar_init(sh.bar(B_QEMPTY), 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(sh.bar(B_KFULL + s), 1);
            mbar_init(sh.bar(B_KEMPTY + s), 1);
            mbar_init(sh.bar(B_VFULL + s), 1);
            mbar_init(sh.bar(B_VEMPTY + s), 1);
        }
        for (int s = 0; s < kSBuf; ++s) {
            mbar_init(sh.bar(B_SFULL + s), 1);
            mbar_init(sh.bar(B_PFULL + s), 4);
            mbar_init(sh.bar(B_PVDONE + s), 1);
        }
        mbar_init(sh.bar(B_OFREE), 4);
        mbar_init(sh.bar(B_DRAIN), 1);
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

    if (warp < 4) {
        softmax_epilogue(sh, p, d, tmem);
    } else if (warp == 4) {
        if (lane == 0) producer(sh, p, d, &tm_q, &tm_k, &tm_v);
        __syncwarp();
    } else {
        if (lane == 0) mma_issuer(sh, p, d, tmem);
        __syncwarp();
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool encode_3d(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

cudaError_t launch_attn_tc(const AttnArgs &p, int grid, cudaStream_t st)
{
    const int G = p.Hq / p.Hkv;
    CUtensorMap tq, tk, tv;
    const uint64_t row = tc::kD * 2;
    if (!encode_3d(&tq, p.q, tc::kD, p.Hq, (uint64_t)p.B * p.K, row, (uint64_t)p.Hq * row, 64, G, p.K) ||
        !encode_3d(&tk, p.k_cache, tc::kD, p.S_max, (uint64_t)p.B * p.Hkv, row,
                   (uint64_t)p.S_max * row, 64, 64, 1) ||
        !encode_3d(&tv, p.v_cache, tc::kD, p.S_max, (uint64_t)p.B * p.Hkv, row,
                   (uint64_t)p.S_max * row, 64, 64, 1))
        return cudaErrorInvalidValue;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(tc::attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)tc::kSmemAlloc);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    tc::attn_tc_kernel<<<grid, tc::kThreads, tc::kSmemAlloc, st>>>(tq, tk, tv, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_attn_combine(p, grid, st);
}

}  // namespace orthrus

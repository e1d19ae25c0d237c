// sm_100a decode kernel for sequences of at most 64 query rows (s_q * h_q <= 64): one CTA
// per SM, no cluster, nothing exchanged between SMs.
//
// The 2-CTA kernel (decode_pair.cuh) works on 128-row tiles split over two SMs. With 64
// rows or fewer, one of its CTAs computes padding only, yet the pair still runs its full
// per-page chain, including the post-QK reload of the other page. Here one CTA owns a
// work unit alone and reads every page exactly once:
//   QK:  S = Q K^T for one 64-token page: M = 128, N = 64 tokens, K = 576. The A operand
//        holds the R <= 64 query rows replicated: TMEM lane l (A row l) carries query row
//        l % 32 (kN <= 32: four copies, one per lane quarter) or l % 64 (kN = 64: two
//        copies). So every warp finds every row's scores in its own lane quarter, and
//        the four warps split each page's tokens between them: the softmax work of a
//        page is spread over all four SM sub-partitions instead of one or two.
//        Q's first kQtChunks x 64 dims come from TMEM, the rest from shared memory (the
//        replicated rows laid out as 128 A rows).
//   PV:  transposed, O^T = V^T P^T: M = 128 latent dims (four blocks for 512), N = kN
//        (the rows padded to 16, 32 or 64), K = 16 tokens per instruction. V^T is the page
//        tile itself, read MN-major from its stage (no copy); P is the B operand, K-major,
//        one 128-byte row of 64 bf16 probabilities per query row, each warp writing its
//        token slice. O^T needs 4 kN TMEM columns, which leaves room for Q in TMEM.
// Per CTA (224 threads; 480 over an FP8 cache):
//   warps 0-3  the row group. Warp w takes copy w / kRowWarps of the rows (token slice
//              [copy x kTok, +kTok) of every page) and rows (w % kRowWarps) x 32 + lane.
//              All 128 threads (TMEM lane = latent dim of an O^T block) also do the rare
//              O rescale, the epilogue, the move of each item's q rows into TMEM and
//              shared memory, and the zeroing of V rows past a sequence's end.
//   warp 4     TMA producer: a ring of kStages 72 KB stages. An item takes one slot for its
//              q rows (box {64, kN rows, 9 chunks}) and then one slot per page (box {64,
//              64 rows, 9 chunks}: 9 swizzled 8 KB tiles in one instruction), with the next
//              page prefetched into L2.
//   warp 5     TMEM owner and QK issuer: each page's QK as soon as its stage landed and
//              its score buffer was read out, so the next page's QK keeps the tensor pipe
//              busy while the row group turns S(j) into P(j).
//   warp 6     PV issuer: PV(j) as soon as P(j) is written. With one thread issuing both,
//              a P that became ready while the next QK's 36 instructions were being
//              issued (the issue queue is shallow, so that thread blocks) waited for all
//              of them, and its stage stayed held that much longer.
//   warps 7-14 FP8 cache only: widen each page's codes to bf16 in its stage.
// Scores stay in the log2 domain. A row's reference max is raised only when a score
// exceeds it by more than kRescaleLog2. Partial maxima of the token slices meet in shared
// memory once per page; every warp then tracks every row's reference itself, so the
// rescale factors of O^T columns need no second exchange.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "items.cuh"
#include "ptx.cuh"

namespace mla {
namespace solo {

constexpr int kThreads = 224;                         // bf16 cache: rows, producer, QK and PV issuers
constexpr int kWidenWarps = 8;                        // FP8 cache: warps that widen pages
constexpr int kThreadsF8 = kThreads + 32 * kWidenWarps;
constexpr int kRowThreads = 128;
constexpr int kWarpProducer = 4;
constexpr int kWarpMma = 5;                           // issues QK (and owns TMEM)
constexpr int kWarpPv = 6;                            // issues PV
constexpr int kWarpWiden = 7;                         // FP8 cache: the first widening warp
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kBoxBytes = 64 * 128;             // 64 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kStageBytes = 9 * kBoxBytes;      // one page: 64 tokens x 576 dims
constexpr uint32_t kSmemLimit = 232448;              // sm_100 per-block opt-in maximum
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 3;
// An FP8 page lands in its own stage and is widened there: its codes as 8 tiles of 64 rows
// x 64 bytes at [32, 64) KB (tile c = latent dims [64 c, 64 c + 64)), its scales as 64 rows
// x 16 bytes at [31, 32) KB, its rope dims (bf16) already in the rope tile at [64, 72) KB.
// The widened tile c takes [8 c, 8 c + 8) KB. 41,984 bytes land per page, the row format's.
constexpr uint32_t kF8CodeOff = 32 * 1024;
constexpr uint32_t kF8ScaleOff = 31 * 1024;
constexpr uint32_t kF8PageTx = 8 * 64 * 64 + 64 * 16 + kBoxBytes;

// Layout for kN padded query rows. TMEM columns: O^T [0, 4 kN), kSBufs score buffers of 64,
// then Q's first dims as bf16 pairs. Shared memory (from a 1 KB aligned base): Q's
// remaining chunks (128 replicated A rows each), one P buffer, the stages, then barriers
// and per-row arrays.
template <int N_, bool F8_ = false>
struct Cfg {
    static constexpr int kN = N_;
    static constexpr bool kF8 = F8_;                          // FP8 latent cache (656-byte rows)
    static constexpr int kBlockThreads = kF8 ? kThreadsF8 : kThreads;
    static constexpr int kRowWarps = kN <= 32 ? 1 : 2;        // warps holding one copy of the rows
    static constexpr int kCopies = 4 / kRowWarps;
    static constexpr int kTok = 64 / kCopies;                 // tokens of a page per warp
    static constexpr uint32_t kColO = 0;
    static constexpr uint32_t kColS = 4 * kN;
    static constexpr int kSBufs = (kColS + 2 * 64 + 288 <= kTmemCols) ? 2 : 1;
    static constexpr uint32_t kColQ = kColS + 64 * kSBufs;
    static constexpr int kQtChunksFit = (int)((kTmemCols - kColQ) * 2 / 64);
    static constexpr int kQtChunks = kQtChunksFit >= 9 ? 9 : kQtChunksFit;   // Q chunks in TMEM
    static constexpr int kQsChunks = 9 - kQtChunks;                          // in shared memory
    static constexpr uint32_t kTileBytes = kN * 128;          // kN rows x 64 dims, one chunk
    static constexpr uint32_t kARows = 128;                   // A rows of a Q chunk in smem
    static constexpr uint32_t kOffQs = 0;
    static constexpr uint32_t kOffP = kOffQs + kQsChunks * kARows * 128;
    static constexpr uint32_t kOffStage = kOffP + kTileBytes;
    static constexpr uint32_t kMiscBytes = 4096;
    static constexpr int kStagesFit = (int)((kSmemLimit - 1024 - kMiscBytes - kOffStage) / kStageBytes);
    static constexpr int kStages = kStagesFit > kMaxStages ? kMaxStages : kStagesFit;
    static constexpr uint32_t kOffMisc = kOffStage + kStages * kStageBytes;
    static constexpr uint32_t kSmemAlloc = kOffMisc + kMiscBytes + 1024;     // + base alignment
    static constexpr uint32_t kQSlotBytes = kN * 9 * 128;                    // the q rows' box
    static_assert(kN == 16 || kN == 32 || kN == 64, "kN must be 16, 32 or 64");
    static_assert(kStages >= 2, "the ring needs two stages");
    static_assert(kColQ + 32 * kQtChunks <= kTmemCols, "TMEM over budget");
    static_assert(kSmemAlloc <= kSmemLimit, "shared memory over the sm_100 per-block limit");
};

enum : uint32_t {
    kBarFull = 0,                        // [kMaxStages] a stage's copy landed
    kBarFree = kBarFull + kMaxStages,    // [kMaxStages] a stage may be refilled
    kBarQkDone = kBarFree + kMaxStages,  // [2] QK of a step done (score buffer step % kSBufs)
    kBarPvDone = kBarQkDone + 2,         // PV of a step done (one phase per step)
    kBarPReady = kBarPvDone + 1,         // the row group wrote P (4 warp arrivals)
    kBarSFree = kBarPReady + 1,          // [2] the row group read S out of score buffer i
    kBarQReady = kBarSFree + 2,          // the item's q rows are in TMEM and shared memory
    kBarOFree = kBarQReady + 1,          // the previous item's O^T was read out
    kBarDecide = kBarOFree + 1,          // the step's partial maxima are posted
    kBarEpi = kBarDecide + 1,            // the item's partial row sums / 1/l posted (2 per item)
    kBarDrain = kBarEpi + 1,             // [2] the QK and the PV issuer's last commits
    kBarStall = kBarDrain + 2,           // never completes (the timeout test hook waits on it)
    kBarWiden = kBarStall + 1,           // FP8 cache: the widening warps' syncs inside a page
    kBarDqFull = kBarWiden + 1,          // [kMaxStages] FP8 cache: a stage's page widened (kWidenWarps arrivals)
    kBarDqHalf = kBarDqFull + kMaxStages,  // [kMaxStages] FP8 cache: its tiles 0-2 widened
    kNumBars = kBarDqHalf + kMaxStages
};
// misc area: barriers [0, 256), tmem base at 256, abort flag at 260; partial maxima
// [2 parity][4 copies][64 rows] f32 at 512; partial row sums [2 sums][4 copies][64] at
// 2560; inverse row sums [64] at 3584
static_assert(kNumBars * 8 <= 256, "barrier area");
constexpr uint32_t kMiscPmax = 512, kMiscPsum = 2560, kMiscInvL = 3584;

template <class C>
struct Smem {
    uint8_t* base;
    uint32_t base_u32;
    uint64_t wait_limit;                 // ns a wait may last before the kernel gives up
    __device__ uint32_t bar(uint32_t i) const { return base_u32 + C::kOffMisc + 8 * i; }
    __device__ uint32_t stage(uint32_t s) const { return base_u32 + C::kOffStage + s * kStageBytes; }
    __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + C::kOffMisc + 256); }
    __device__ volatile int* abort_flag() const {
        return reinterpret_cast<volatile int*>(base + C::kOffMisc + 260);
    }
    __device__ float* pmax(uint32_t par, int copy) const {
        return reinterpret_cast<float*>(base + C::kOffMisc + kMiscPmax) + (par * 4 + copy) * 64;
    }
    __device__ float* psum(int which, int copy) const {
        return reinterpret_cast<float*>(base + C::kOffMisc + kMiscPsum) + (which * 4 + copy) * 64;
    }
    __device__ float* inv_l() const { return reinterpret_cast<float*>(base + C::kOffMisc + kMiscInvL); }
};

// Bounded wait: false if the phase does not complete within the limit or another role of
// the CTA already gave up (then the caller stops).
template <class C>
__device__ __forceinline__ bool wait_bar(const Smem<C>& sh, uint32_t bar, uint32_t parity,
                                         uint32_t where) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 0;; ++it) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u) {
            if (*sh.abort_flag()) return false;
            if (ptx::globaltimer() - t0 > sh.wait_limit) {
                *sh.abort_flag() = 1;
                record_error(kErrTimeout, where);
                return false;
            }
        }
    }
}

// Warp-uniform bounded wait: no lane leaves while its neighbours stay in .aligned code.
template <class C>
__device__ __forceinline__ bool warp_wait_bar(const Smem<C>& sh, uint32_t bar, uint32_t parity,
                                              uint32_t where) {
    const bool ok = wait_bar(sh, bar, parity, where);
    return __all_sync(0xffffffffu, ok);
}

// Wait for copies or MMAs this CTA issued before it may finish: bounded by the time limit
// only (the abort flag does not cut it short, so nothing lands after the CTA has exited
// unless the limit itself runs out).
template <class C>
__device__ __forceinline__ void drain_wait(const Smem<C>& sh, uint32_t bar, uint32_t parity,
                                           uint32_t where) {
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > sh.wait_limit) {
            record_error(kErrTimeout, where);
            return;
        }
    }
}

__device__ __forceinline__ void warp_arrive(uint32_t bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(bar);
}

// ------------------------------------------------------------------ producer (warp 4)
// Ring slot g uses stage g % kStages; its fill number g / kStages sets the parities.
// tm_page is the bf16 pool's page map, or for an FP8 cache its codes map; tm_scales and
// tm_rope are the FP8 cache's scale and rope maps (unused for bf16).
template <class C>
__device__ __forceinline__ void run_producer(const DecodeParams& p, const Smem<C>& sh,
                                             const CUtensorMap* tm_page, const CUtensorMap* tm_scales,
                                             const CUtensorMap* tm_rope, const CUtensorMap* tm_q) {
    if (g_mla_debug_stall) {
        // test hook: wait on a barrier nothing completes, before any copy is issued, so
        // every role gives up after the limit with nothing in flight
        wait_bar(sh, sh.bar(kBarStall), 0, 0x40u);
        return;
    }
    ItemIter iter(p, (int)blockIdx.x, (int)gridDim.x);
    Item it;
    uint32_t g = 0;
    auto acquire = [&](uint32_t gg) -> bool {
        if (gg < (uint32_t)C::kStages) return true;
        return wait_bar(sh, sh.bar(kBarFree + gg % C::kStages), ((gg / C::kStages) - 1u) & 1u, 0x41u);
    };
    bool ok = true;
    while (ok && iter.next(it)) {
        if (!(ok = acquire(g))) break;
        {
            const uint32_t s = g % C::kStages;
            ptx::mbar_arrive_expect_tx(sh.bar(kBarFull + s), C::kQSlotBytes);
            ptx::tma_load_3d(sh.stage(s), tm_q, sh.bar(kBarFull + s), 0,
                             it.b * p.rows + it.t * kTileRows, 0);
            ++g;
        }
        // the holder of a split sequence's first chunk clears the combine's counters
        if (it.chunk == 0 && it.n_chunks > 1 && it.v < p.max_chunks) {
            int* cnt = combine_counters(p) + (size_t)it.v * kCombineCounters;
#pragma unroll 1
            for (int i = 0; i < kCombineCounters; ++i) cnt[i] = 0;
        }
        for (int k = it.k_lo; k < it.k_hi; ++k) {
            if (!(ok = acquire(g))) break;
            const uint32_t s = g % C::kStages;
            const int row = page_row(p, it.b, k, it.k_hi);
            if constexpr (C::kF8) {
                const uint32_t st = sh.stage(s), bar = sh.bar(kBarFull + s);
                ptx::mbar_arrive_expect_tx(bar, kF8PageTx);
                ptx::tma_load_3d(st + kF8CodeOff, tm_page, bar, 0, row, 0);
                ptx::tma_load_2d(st + kF8ScaleOff, tm_scales, bar, 0, row);
                ptx::tma_load_2d(st + 8 * kBoxBytes, tm_rope, bar, 0, row);
            } else {
                ptx::mbar_arrive_expect_tx(sh.bar(kBarFull + s), kStageBytes);
                ptx::tma_load_3d(sh.stage(s), tm_page, sh.bar(kBarFull + s), 0, row, 0);
            }
            ++g;
            if (k + 1 < it.k_hi) {                   // warm L2 for the next page
                const int pid = p.block_table[(size_t)it.b * p.max_blocks + k + 1];
                if (pid >= 0 && pid < p.num_blocks) ptx::tma_prefetch_3d(tm_page, 0, pid * kBlock, 0);
            }
        }
    }
    // every copy issued must land before the CTA may finish
    const uint32_t first = g > (uint32_t)C::kStages ? g - C::kStages : 0u;
    for (uint32_t gg = first; gg < g; ++gg)
        drain_wait(sh, sh.bar(kBarFull + gg % C::kStages), (gg / C::kStages) & 1u, 0x42u);
}

// ------------------------------------------------------------------ MMA issuers (warps 5, 6)
// K-steps [k0, k1) of the 36 (16 dims each) of QK for the page in stage s into score
// buffer sb; the part that ends at 36 commits the buffer's QkDone.
template <class C, int k0, int k1>
__device__ __forceinline__ void issue_qk_range(const Smem<C>& sh, uint32_t tmem, uint32_t s, uint32_t sb) {
    constexpr uint32_t kIdesc = ptx::idesc_bf16(128, 64, false, false);
    ptx::tc_fence_after();
    const uint32_t d = tmem + C::kColS + 64 * sb;
    const uint32_t st = sh.stage(s);
#pragma unroll
    for (int k = k0; k < k1; ++k) {
        const uint64_t bdesc = ptx::smem_desc(st + (k >> 2) * kBoxBytes + (k & 3) * 32, 16, 1024, 2);
        if (k < 4 * C::kQtChunks) {
            ptx::mma_ts(d, tmem + C::kColQ + 8 * k, bdesc, kIdesc, k > 0 ? 1u : 0u);
        } else {
            const uint64_t adesc = ptx::smem_desc(
                sh.base_u32 + C::kOffQs + ((k >> 2) - C::kQtChunks) * (C::kARows * 128) + (k & 3) * 32,
                16, 1024, 2);
            ptx::mma_ss(d, adesc, bdesc, kIdesc, k > 0 ? 1u : 0u);
        }
    }
    if constexpr (k1 == 36) ptx::mma_commit(sh.bar(kBarQkDone + sb));
}

// O^T += V^T P^T for the page in stage s; `first` starts the item's accumulation.
template <class C>
__device__ __forceinline__ void issue_pv(const Smem<C>& sh, uint32_t tmem, uint32_t s, bool first) {
    constexpr int kN = C::kN;
    constexpr uint32_t kIdesc = ptx::idesc_bf16(128, kN, true, false);
    ptx::tc_fence_after();
    const uint32_t st = sh.stage(s);
    const uint32_t pb = sh.base_u32 + C::kOffP;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            // V^T block i: dims [128 i, 128 i + 128) = chunks 2i, 2i+1 (leading offset one
            // chunk), tokens [16 kk, 16 kk + 16) (8-token groups 1 KB apart)
            const uint64_t adesc = ptx::smem_desc(st + 2 * i * kBoxBytes + kk * 2048, kBoxBytes, 1024, 2);
            const uint64_t bdesc = ptx::smem_desc(pb + kk * 32, 16, 1024, 2);
            ptx::mma_ss(tmem + C::kColO + kN * i, adesc, bdesc, kIdesc, (!first || kk > 0) ? 1u : 0u);
        }
    }
    ptx::mma_commit(sh.bar(kBarFree + s));
    ptx::mma_commit(sh.bar(kBarPvDone));
}

// Bounded wait of an issuer thread: also gives up when another role has.
template <class C>
__device__ __forceinline__ bool issuer_wait(const Smem<C>& sh, uint32_t bar, uint32_t parity,
                                            uint32_t where) {
    return wait_bar(sh, bar, parity, where);
}

// QK issuer (warp 5, one thread): each page's QK as soon as its stage landed (and, for an
// FP8 cache, was widened) and its score buffer was read out. PVs come from their own
// thread (run_pv), so a P that is ready while a QK is being issued does not wait for the
// whole QK to be issued first.
template <class C>
__device__ __forceinline__ void run_qk(const DecodeParams& p, const Smem<C>& sh, uint32_t tmem) {
    ItemIter iter(p, (int)blockIdx.x, (int)gridDim.x);
    Item it;
    uint32_t g = 0, gs = 0, items = 0;
    uint32_t dq_par = 0;                   // FP8: bit s = parity of stage s's next widened page
    bool ok = true;
    while (ok && iter.next(it)) {
        // the item's q rows were moved out of their slot: free it
        if (!issuer_wait(sh, sh.bar(kBarQReady), items & 1u, 0x48u)) break;
        ptx::tc_fence_after();
        ptx::mbar_arrive(sh.bar(kBarFree + g % C::kStages));
        ++g;
        const uint32_t n = (uint32_t)it.pages();
        for (uint32_t qk = 0; qk < n && ok; ++qk) {
            const uint32_t gq = g + qk, Sq = gs + qk;
            const uint32_t st = gq % C::kStages, sb = Sq % C::kSBufs;
            // its score buffer must be free: S of step Sq - kSBufs read out
            if (Sq >= (uint32_t)C::kSBufs &&
                !issuer_wait(sh, sh.bar(kBarSFree + sb), ((Sq / C::kSBufs) - 1u) & 1u, 0x49u)) { ok = false; break; }
            if (!issuer_wait(sh, sh.bar(kBarFull + st), (gq / C::kStages) & 1u, 0x4bu)) { ok = false; break; }
            if constexpr (C::kF8) {
                // the K-steps of the first three tiles as soon as those are widened
                const uint32_t par = (dq_par >> st) & 1u;
                dq_par ^= 1u << st;
                if (!issuer_wait(sh, sh.bar(kBarDqHalf + st), par, 0x4du)) { ok = false; break; }
                issue_qk_range<C, 0, 12>(sh, tmem, st, sb);
                if (!issuer_wait(sh, sh.bar(kBarDqFull + st), par, 0x4cu)) { ok = false; break; }
                issue_qk_range<C, 12, 36>(sh, tmem, st, sb);
            } else {
                issue_qk_range<C, 0, 36>(sh, tmem, st, sb);
            }
        }
        g += n;
        gs += n;
        ++items;
    }
    // every MMA this thread issued is complete before the CTA may finish
    ptx::mma_commit(sh.bar(kBarDrain));
    drain_wait(sh, sh.bar(kBarDrain), 0, 0x4au);
}

// PV issuer (warp 6, one thread): each page's PV as soon as its P is written (and, for an
// item's first page, the previous item's O^T was read out).
template <class C>
__device__ __forceinline__ void run_pv(const DecodeParams& p, const Smem<C>& sh, uint32_t tmem) {
    ItemIter iter(p, (int)blockIdx.x, (int)gridDim.x);
    Item it;
    uint32_t g = 0, gs = 0, items = 0;
    bool ok = true;
    while (ok && iter.next(it)) {
        ++g;                                   // the item's q slot
        const uint32_t n = (uint32_t)it.pages();
        for (uint32_t pv = 0; pv < n; ++pv) {
            if (pv == 0 && items > 0 &&
                !issuer_wait(sh, sh.bar(kBarOFree), (items - 1) & 1u, 0x4du)) { ok = false; break; }
            if (!issuer_wait(sh, sh.bar(kBarPReady), (gs + pv) & 1u, 0x4eu)) { ok = false; break; }
            ptx::tc_fence_after();
            issue_pv(sh, tmem, (g + pv) % C::kStages, pv == 0);
        }
        g += n;
        gs += n;
        ++items;
    }
    ptx::mma_commit(sh.bar(kBarDrain + 1));
    drain_wait(sh, sh.bar(kBarDrain + 1), 0, 0x4fu);
}

// ------------------------------------------------------------------ row group (warps 0-3)
__device__ __forceinline__ float f32(uint32_t x) { return __uint_as_float(x); }

template <int kCols>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* v) {
    if constexpr (kCols == 16) ptx::tmem_ld16(taddr, v);
    else if constexpr (kCols == 32) ptx::tmem_ld32(taddr, v);
    else ptx::tmem_ld64(taddr, v);
}

template <class C>
struct RowCtx {
    uint32_t tmem, lane_base;
    int tid, warp, lane;
    int copy;             // which copy of the rows this warp holds: token slice copy x kTok
    int row;              // this thread's query row: (warp % kRowWarps) x 32 + lane
    int own;              // index of `row` among the rows this thread tracks (warp % kRowWarps)
};

// Per-row state every warp keeps for the rows lane, lane + 32 (kRowWarps of them): the
// reference max of the item so far.
template <class C>
struct Track {
    float m[C::kRowWarps];
};

// a[i] for a register array of one or two values, without dynamic indexing
template <int K>
__device__ __forceinline__ float pick(const float (&a)[K], int i) {
    if constexpr (K == 1) return a[0];
    else return i ? a[1] : a[0];
}

// The item's q rows, landed in stage s as kN rows x 9 chunks: dims [0, 64 kQtChunks) go
// to TMEM, every lane l holding query row l % (32 kRowWarps) (bf16 pairs), and the rest to
// shared memory as 128 A rows of the same replication (a byte copy of 128-byte rows:
// both sides are 1 KB aligned and row l keeps its row % 8, so the swizzle carries over).
template <class C>
__device__ __forceinline__ void move_q(const Smem<C>& sh, const RowCtx<C>& c, uint32_t s) {
    const uint32_t st = sh.stage(s);
    const int src_row = c.row;                     // < 32 kRowWarps; >= kN reads padding
#pragma unroll 1
    for (int ch = 0; ch < C::kQtChunks; ++ch) {
        uint32_t v[32];
        const uint32_t rowa = st + ch * C::kTileBytes + (uint32_t)src_row * 128;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            const uint4 x = ptx::ld_shared_v4(rowa + (((uint32_t)jj ^ (uint32_t)(src_row & 7)) * 16));
            v[4 * jj] = x.x; v[4 * jj + 1] = x.y; v[4 * jj + 2] = x.z; v[4 * jj + 3] = x.w;
        }
        ptx::tmem_st32(c.tmem + c.lane_base + C::kColQ + 32 * ch, v);
    }
    ptx::tmem_wait_st();
    if constexpr (C::kQsChunks > 0) {
        // A row a = tid (all 128 rows), source row a % (32 kRowWarps)
        const int a = c.tid;
        const int r = a % (32 * C::kRowWarps);
#pragma unroll 1
        for (int ch = 0; ch < C::kQsChunks; ++ch) {
            const uint32_t src = st + (C::kQtChunks + ch) * C::kTileBytes + (uint32_t)r * 128;
            const uint32_t dst = sh.base_u32 + C::kOffQs + ch * (C::kARows * 128) + (uint32_t)a * 128;
            // 16-byte units in an order rotated by row, so that a warp's 32 rows spread
            // over all banks (the copy keeps each unit in place)
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint32_t off = (uint32_t)((u ^ a) & 7) * 16;
                const uint4 x = ptx::ld_shared_v4(src + off);
                ptx::st_shared_v4(dst + off, x.x, x.y, x.z, x.w);
            }
        }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
}

// Row-group sync inside a widening: every warp arrives, every warp waits (bounded).
template <class C>
__device__ __forceinline__ bool widen_sync(const Smem<C>& sh, uint32_t& n_syncs) {
    warp_arrive(sh.bar(kBarWiden));
    return warp_wait_bar(sh, sh.bar(kBarWiden), (n_syncs++) & 1u, 0x5au);
}

// 16 kU codes of one row (kU 16-byte words) to bf16, as the format reads them back: E4M3
// -> f16 (exact), times the group scale in fp32, rounded to bf16 (both nearest-even);
// stored as the row's 16-byte units 2 kU part .. 2 kU part + 2 kU - 1 of its
// 128-byte-swizzled tile row.
template <int kU>
__device__ __forceinline__ void widen_units(uint32_t tile_row, int row, int part, float sc,
                                            const uint4 (&w)[kU], bool live) {
    uint32_t o[8 * kU];
    const float2 sc2 = make_float2(sc, sc);
#pragma unroll
    for (int k = 0; k < 4 * kU; ++k) {
        const uint4& wu = w[k >> 2];
        const uint32_t word = (k & 3) == 0 ? wu.x : (k & 3) == 1 ? wu.y : (k & 3) == 2 ? wu.z : wu.w;
        const uint32_t lo = ptx::e4m3x2_to_f16x2((uint16_t)(word & 0xffffu));
        const uint32_t hi = ptx::e4m3x2_to_f16x2((uint16_t)(word >> 16));
        const float2 a = ptx::mul_f32x2(__half22float2(*reinterpret_cast<const __half2*>(&lo)), sc2);
        const float2 b = ptx::mul_f32x2(__half22float2(*reinterpret_cast<const __half2*>(&hi)), sc2);
        const __nv_bfloat162 r0 = __floats2bfloat162_rn(a.x, a.y);
        const __nv_bfloat162 r1 = __floats2bfloat162_rn(b.x, b.y);
        o[2 * k] = live ? *reinterpret_cast<const uint32_t*>(&r0) : 0u;
        o[2 * k + 1] = live ? *reinterpret_cast<const uint32_t*>(&r1) : 0u;
    }
    const uint32_t sw = (uint32_t)(row & 7);
#pragma unroll
    for (int u = 0; u < 2 * kU; ++u)
        ptx::st_shared_v4(tile_row + ((((uint32_t)(2 * kU * part + u)) ^ sw) * 16), o[4 * u],
                          o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
}

// FP8 cache: widens the page in the stage of ring slot g in place, into the 9-tile
// swizzled bf16 layout QK and PV read (the rope tile arrived by TMA). The widening warps
// give each row kWidenWarps / 2 threads, each a contiguous share of each tile's 64 dims.
// Every thread first reads its scales and all its codes into registers; tiles 0-2 lie
// below every input and are written at once; tiles 3-7 cover the scales and the codes,
// so they follow one sync of the widening warps (all inputs read). Rows past the
// sequence end are written as zeros (their codes may be anything, NaN included).
template <class C>
__device__ __forceinline__ bool widen(const Smem<C>& sh, int tid, const Item& it, int page,
                                      uint32_t g, uint32_t& n_syncs) {
    const uint32_t s = g % C::kStages;
    if (!warp_wait_bar(sh, sh.bar(kBarFull + s), (g / C::kStages) & 1u, 0x58u)) return false;
    // kParts threads per row, each kU 16-byte words (16 kU codes) of each 64-code chunk
    constexpr int kParts = kWidenWarps * 32 / kBlock;
    constexpr int kU = 4 / kParts;
    static_assert(kParts * kU == 4 && kParts * kBlock == kWidenWarps * 32, "widening layout");
    const int row = tid / kParts, part = tid % kParts;
    const bool live = page * kBlock + row < it.L;
    const uint32_t st = sh.stage(s);
    const uint4 scv = ptx::ld_shared_v4(st + kF8ScaleOff + (uint32_t)row * 16);
    const float sc[4] = {__uint_as_float(scv.x), __uint_as_float(scv.y), __uint_as_float(scv.z),
                         __uint_as_float(scv.w)};
    uint4 w[8][kU];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint32_t a = st + kF8CodeOff + (uint32_t)ch * 4096 + (uint32_t)row * 64 + (uint32_t)part * 16 * kU;
#pragma unroll
        for (int u = 0; u < kU; ++u) w[ch][u] = ptx::ld_shared_v4(a + 16 * u);
    }
    auto tile = [&](int ch) {
        widen_units<kU>(st + (uint32_t)ch * kBoxBytes + (uint32_t)row * 128, row, part, sc[ch >> 1], w[ch], live);
    };
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) tile(ch);
    ptx::fence_proxy_async_smem();           // tiles 0-2 visible to the MMA: QK may start
    warp_arrive(sh.bar(kBarDqHalf + s));
    if (!widen_sync(sh, n_syncs)) return false;
#pragma unroll
    for (int ch = 3; ch < 8; ++ch) tile(ch);
    ptx::fence_proxy_async_smem();           // the widened tiles visible to the MMA
    warp_arrive(sh.bar(kBarDqFull + s));
    return true;
}

// One page step S (the item's j-th page) for this thread.
template <class C>
__device__ __forceinline__ bool row_step(const DecodeParams& p, const Smem<C>& sh, const RowCtx<C>& c,
                                         const Item& it, int n_vis, uint32_t j, uint32_t S,
                                         uint32_t s, Track<C>& tr, float& l_sum, float& l_rnd) {
    constexpr int kN = C::kN;
    constexpr int kTok = C::kTok;
    const uint32_t sb = S % C::kSBufs, par = S & 1u;
    const uint32_t qpar = C::kSBufs == 2 ? (S >> 1) & 1u : S & 1u;
    if (!warp_wait_bar(sh, sh.bar(kBarQkDone + sb), qpar, 0x51u)) return false;
    ptx::tc_fence_after();
    uint32_t sv[kTok];
    tmem_ld_cols<kTok>(c.tmem + c.lane_base + C::kColS + 64 * sb + c.copy * kTok, sv);
    ptx::tc_fence_before();                        // S read out before a later QK rewrites it
    warp_arrive(sh.bar(kBarSFree + sb));
    const int page = it.k_lo + (int)j;
    const int lim = n_vis - page * kBlock - c.copy * kTok;    // valid tokens of the slice [0, lim)
    const float m_own = pick(tr.m, c.own);
    const float base = m_own == -INFINITY ? 0.f : m_own;
    const float L2 = p.scale_log2;
    float x[kTok];
    if (__all_sync(0xffffffffu, lim >= kTok)) {
#pragma unroll
        for (int q = 0; q < kTok; ++q) x[q] = fmaf(f32(sv[q]), L2, -base);
    } else {
#pragma unroll
        for (int q = 0; q < kTok; ++q) x[q] = q < lim ? fmaf(f32(sv[q]), L2, -base) : -INFINITY;
    }
    float mx = x[0];
#pragma unroll
    for (int q = 1; q < kTok; ++q) mx = fmaxf(mx, x[q]);
    sh.pmax(par, c.copy)[c.row] = mx + base;
    warp_arrive(sh.bar(kBarDecide));
    if (!warp_wait_bar(sh, sh.bar(kBarDecide), par, 0x52u)) return false;
    // every tracked row's page max, reference update and O^T factor (identical in every
    // warp: the same maxima and the same history)
    float fac[C::kRowWarps];
    bool any = false;
#pragma unroll
    for (int k = 0; k < C::kRowWarps; ++k) {
        const int r = c.lane + 32 * k;
        float pm = -INFINITY;
#pragma unroll
        for (int cp = 0; cp < C::kCopies; ++cp)
            pm = fmaxf(pm, *reinterpret_cast<volatile float*>(&sh.pmax(par, cp)[r]));
        const float mo = tr.m[k];
        const bool raise = mo == -INFINITY ? pm > -INFINITY : pm > mo + kRescaleLog2;
        const float mn = raise ? pm : mo;
        const bool need = raise && mo != -INFINITY;           // O^T holds pages at mo
        fac[k] = need ? ptx::ex2_ftz(mo - mn) : 1.f;
        any |= need;
        tr.m[k] = mn;
    }
    const float m_new = pick(tr.m, c.own);
    if (m_new != base && m_new != -INFINITY) {
        const float d = m_new - base;
#pragma unroll
        for (int q = 0; q < kTok; ++q) x[q] -= d;
    }
    l_sum *= pick(fac, c.own);
    l_rnd *= pick(fac, c.own);
    any = __any_sync(0xffffffffu, any);
    if (any || S > 0) {
        // PV of step S-1 must be done: before O^T is rescaled, and before P is rewritten
        if (!warp_wait_bar(sh, sh.bar(kBarPvDone), (S - 1) & 1u, 0x53u)) return false;
        ptx::tc_fence_after();
    }
    if (any) {
        // scale O^T column r (query row r) by its row's factor; the factor of row r is
        // held by lane r % 32 (tracked index r / 32)
#pragma unroll 1
        for (int cc = 0; cc < kN; cc += 16) {
            float f[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int r = cc + e;
                f[e] = __shfl_sync(0xffffffffu, pick(fac, r >> 5), r & 31);
            }
#pragma unroll 1
            for (int i = 0; i < 4; ++i) {
                uint32_t v[16];
                const uint32_t a = c.tmem + c.lane_base + C::kColO + kN * i + cc;
                ptx::tmem_ld16(a, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(f32(v[e]) * f[e]);
                ptx::tmem_st16(a, v);
            }
        }
        ptx::tmem_wait_st();
    }
    {
        uint32_t pk[kTok / 2];
        float rs0 = 0.f, rs1 = 0.f, rr0 = 0.f, rr1 = 0.f;
#pragma unroll
        for (int q = 0; q < kTok / 2; ++q) {
            const float p0 = ptx::ex2_ftz(x[2 * q]);
            const float p1 = ptx::ex2_ftz(x[2 * q + 1]);
            rs0 += p0;
            rs1 += p1;
            // O is normalised by the sum of the bf16 values PV multiplies, so it is a
            // weighted mean of V rows whose weights sum to one: a dominant token's rounding
            // (its P may be up to 2^kRescaleLog2, not 1) then cancels instead of scaling
            // the output. The lse keeps the exact sum.
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            rr0 += __low2float(h2);
            rr1 += __high2float(h2);
            pk[q] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        l_sum += rs0 + rs1;
        l_rnd += rr0 + rr1;
        if (c.row < kN) {
            // this slice of the row of P: tokens [copy kTok, +kTok) = 16-byte units
            // [copy kTok / 8, +kTok / 8) of the 128-byte row, K-major, 128-byte swizzle
            const uint32_t prow = sh.base_u32 + C::kOffP + (uint32_t)c.row * 128;
#pragma unroll
            for (int u = 0; u < kTok / 8; ++u) {
                const uint32_t unit = (uint32_t)(c.copy * (kTok / 8) + u);
                ptx::st_shared_v4(prow + ((unit ^ (uint32_t)(c.row & 7)) * 16), pk[4 * u],
                                  pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
        }
    }
    // V rows past the sequence end (they may hold stale or NaN data, and P = 0 would not
    // cancel NaN): zero them in the stage. QK of this step, their only other reader, is done.
    const int tail = it.L - page * kBlock;
    if (!C::kF8 && tail < kBlock) {
        const uint32_t st = sh.stage(s);
        const int units = (kBlock - tail) * 64;                 // 8 chunks x 8 x 16 B per row
        for (int q = c.tid; q < units; q += kRowThreads) {
            const int rr = tail + (q >> 6), ch = (q >> 3) & 7, u = q & 7;
            ptx::st_shared_v4(st + ch * kBoxBytes + rr * 128 + u * 16, 0, 0, 0, 0);
        }
    }
    ptx::fence_proxy_async_smem();           // P and zeroed rows visible to the MMA
    ptx::tc_fence_before();
    warp_arrive(sh.bar(kBarPReady));
    return true;
}

// Epilogue of an item: the partial row sums of the token slices meet in shared memory;
// the threads of copy 0 post 1/l and write the lse; then every thread (TMEM lane = latent
// dim) writes its dim of each real row, normalised, as bf16 `out`, fp32 `out_f32` or the
// fp32 split partial.
template <class C>
__device__ __forceinline__ bool epilogue(const DecodeParams& p, const Smem<C>& sh, const RowCtx<C>& c,
                                         const Item& it, float m_row, float l_sum, float l_rnd,
                                         uint32_t last_step, uint32_t epi_index) {
    constexpr int kN = C::kN;
    const bool final_out = it.n_chunks == 1;
    const bool have_ws = it.part < p.max_chunks;
    sh.psum(0, c.copy)[c.row] = l_sum;
    sh.psum(1, c.copy)[c.row] = l_rnd;
    warp_arrive(sh.bar(kBarEpi));
    if (!warp_wait_bar(sh, sh.bar(kBarEpi), (2 * epi_index) & 1u, 0x54u)) return false;
    if (c.copy == 0) {
        float lt = 0.f, lr = 0.f;
#pragma unroll
        for (int cp = 0; cp < C::kCopies; ++cp) {
            lt += *reinterpret_cast<volatile float*>(&sh.psum(0, cp)[c.row]);
            lr += *reinterpret_cast<volatile float*>(&sh.psum(1, cp)[c.row]);
        }
        const bool empty = !(lt > 0.f);
        sh.inv_l()[c.row] = empty ? 0.f : 1.f / lr;
        if (c.row < p.rows) {
            const float lse2 = empty ? -INFINITY : m_row + __log2f(lt);
            if (final_out) {
                const int qi = c.row / p.h_q, h = c.row % p.h_q;
                p.lse[((size_t)it.b * p.h_q + h) * p.s_q + qi] = empty ? -INFINITY : lse2 * kLn2;
            } else if (have_ws) {
                p.ws_lse[(size_t)it.part * kTileRows + c.row] = lse2;
            }
        }
    }
    if (!final_out && !have_ws && c.tid == 0) record_error(kErrWorkspace, (uint32_t)it.v & 0xffffffu);

    warp_arrive(sh.bar(kBarEpi));
    if (!warp_wait_bar(sh, sh.bar(kBarEpi), (2 * epi_index + 1) & 1u, 0x56u)) return false;
    if (!warp_wait_bar(sh, sh.bar(kBarPvDone), last_step & 1u, 0x55u)) return false;
    ptx::tc_fence_after();
    const float* inv_l = sh.inv_l();
    const int rows = p.rows;
    const bool write_any = final_out || have_ws;
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
        uint32_t v[kN];
        tmem_ld_cols<kN>(c.tmem + c.lane_base + C::kColO + kN * i, v);
        if (!write_any) continue;
        const int dim = 128 * i + c.tid;
        if (final_out && p.out_f32 == nullptr) {
            uint16_t* dst = reinterpret_cast<uint16_t*>(p.out) + (size_t)it.b * rows * kHeadDimV + dim;
#pragma unroll
            for (int r = 0; r < kN; ++r)
                if (r < rows) {
                    const __nv_bfloat16 h = __float2bfloat16_rn(f32(v[r]) * inv_l[r]);
                    dst[(size_t)r * kHeadDimV] = *reinterpret_cast<const uint16_t*>(&h);
                }
        } else {
            float* dst = final_out ? p.out_f32 + (size_t)it.b * rows * kHeadDimV + dim
                                   : p.ws_o + (size_t)it.part * kTileRows * kHeadDimV + dim;
#pragma unroll
            for (int r = 0; r < kN; ++r)
                if (r < rows) dst[(size_t)r * kHeadDimV] = f32(v[r]) * inv_l[r];
        }
    }
    ptx::tc_fence_before();
    warp_arrive(sh.bar(kBarOFree));
    return true;
}

template <class C>
__device__ __forceinline__ void run_rows(const DecodeParams& p, const Smem<C>& sh, uint32_t tmem) {
    RowCtx<C> c;
    c.tmem = tmem;
    c.tid = (int)threadIdx.x;
    c.warp = c.tid >> 5;
    c.lane = c.tid & 31;
    c.lane_base = (uint32_t)(c.warp * 32) << 16;
    c.copy = c.warp / C::kRowWarps;
    c.own = c.warp % C::kRowWarps;
    c.row = c.own * 32 + c.lane;
    ItemIter iter(p, (int)blockIdx.x, (int)gridDim.x);
    Item it, prev;
    uint32_t g = 0, gs = 0, items = 0;
    Track<C> tr;
    float l_sum = 0.f, l_rnd = 0.f;
    float prev_m = -INFINITY, prev_l = 0.f, prev_r = 0.f;
    bool have_prev = false;
    while (iter.next(it)) {
        // the item's q rows: into TMEM and shared memory (QK of the previous item, their
        // only reader, finished before the last softmax step of that item began)
        const uint32_t s = g % C::kStages;
        if (!warp_wait_bar(sh, sh.bar(kBarFull + s), (g / C::kStages) & 1u, 0x50u)) return;
        move_q(sh, c, s);
        warp_arrive(sh.bar(kBarQReady));
        ++g;
        // the previous item's epilogue overlaps this item's first QK
        if (have_prev) {
            if (!epilogue(p, sh, c, prev, prev_m, prev_l, prev_r, gs - 1, items - 1)) return;
        }
        const bool row_valid = c.row < p.rows;
        const int qi = row_valid ? c.row / p.h_q : 0;
        const int n_vis = row_valid ? visible_tokens(it.L, p.s_q, qi, p.causal) : 0;
#pragma unroll
        for (int k = 0; k < C::kRowWarps; ++k) tr.m[k] = -INFINITY;
        l_sum = 0.f;
        l_rnd = 0.f;
        const uint32_t n = (uint32_t)it.pages();
        for (uint32_t j = 0; j < n; ++j) {
            if (!row_step(p, sh, c, it, n_vis, j, gs + j, (g + j) % C::kStages, tr, l_sum, l_rnd))
                return;
        }
        g += n;
        gs += n;
        prev = it;
        prev_m = pick(tr.m, c.own);
        prev_l = l_sum;
        prev_r = l_rnd;
        have_prev = true;
        ++items;
    }
    if (have_prev) epilogue(p, sh, c, prev, prev_m, prev_l, prev_r, gs - 1, items - 1);
}

// FP8 cache, warps 6-9: widen every page of this CTA's items as it lands, in ring order
// (an item's q slot comes first and is not theirs), so that neither the softmax warps
// nor the MMA issuer spend time on it.
template <class C>
__device__ __forceinline__ void run_widen(const DecodeParams& p, const Smem<C>& sh, int tid) {
    ItemIter iter(p, (int)blockIdx.x, (int)gridDim.x);
    Item it;
    uint32_t g = 0, n_syncs = 0;
    while (iter.next(it)) {
        ++g;                                   // the item's q slot
        const int n = it.pages();
        for (int j = 0; j < n; ++j, ++g)
            if (!widen(sh, tid, it, it.k_lo + j, g, n_syncs)) return;
    }
}

// tm_page: the bf16 pool's pages, or for an FP8 cache its rows' codes; tm_scales and
// tm_rope: FP8 cache only, its rows' scales and their rope dims as bf16 (unused otherwise).
template <class C>
__global__ void __launch_bounds__(C::kBlockThreads, 1)
decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_page,
              const __grid_constant__ CUtensorMap tm_scales, const __grid_constant__ CUtensorMap tm_rope,
              const __grid_constant__ CUtensorMap tm_q) {
    extern __shared__ uint8_t smem_raw[];
    Smem<C> sh;
    {
        const uint32_t raw = ptx::smem_u32(smem_raw);
        const uint32_t aligned = (raw + 1023u) & ~1023u;
        sh.base = smem_raw + (aligned - raw);
        sh.base_u32 = aligned;
        sh.wait_limit = g_mla_wait_limit_ns;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            ptx::mbar_init(sh.bar(kBarFull + i), 1);
            ptx::mbar_init(sh.bar(kBarFree + i), 1);
        }
        ptx::mbar_init(sh.bar(kBarQkDone + 0), 1);
        ptx::mbar_init(sh.bar(kBarQkDone + 1), 1);
        ptx::mbar_init(sh.bar(kBarPvDone), 1);
        ptx::mbar_init(sh.bar(kBarPReady), 4);
        ptx::mbar_init(sh.bar(kBarSFree + 0), 4);
        ptx::mbar_init(sh.bar(kBarSFree + 1), 4);
        ptx::mbar_init(sh.bar(kBarQReady), 4);
        ptx::mbar_init(sh.bar(kBarOFree), 4);
        ptx::mbar_init(sh.bar(kBarDecide), 4);
        ptx::mbar_init(sh.bar(kBarEpi), 4);
        ptx::mbar_init(sh.bar(kBarDrain + 0), 1);
        ptx::mbar_init(sh.bar(kBarDrain + 1), 1);
        ptx::mbar_init(sh.bar(kBarStall), 1);
        ptx::mbar_init(sh.bar(kBarWiden), kWidenWarps);
        for (int i = 0; i < kMaxStages; ++i) {
            ptx::mbar_init(sh.bar(kBarDqFull + i), kWidenWarps);
            ptx::mbar_init(sh.bar(kBarDqHalf + i), kWidenWarps);
        }
        *sh.abort_flag() = 0;
        ptx::fence_mbarrier_init_cluster();
        ptx::prefetch_tensormap(&tm_page);
        ptx::prefetch_tensormap(&tm_q);
        if (C::kF8) {
            ptx::prefetch_tensormap(&tm_scales);
            ptx::prefetch_tensormap(&tm_rope);
        }
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(ptx::smem_u32(sh.tmem_slot()), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *sh.tmem_slot();
    grid_dependency_wait();      // the schedule is written

    if (warp < 4) {
        run_rows<C>(p, sh, tmem);
    } else if (warp == kWarpProducer) {
        if (lane == 0) run_producer<C>(p, sh, &tm_page, &tm_scales, &tm_rope, &tm_q);
    } else if (warp == kWarpMma) {
        if (lane == 0) run_qk<C>(p, sh, tmem);
    } else if (warp == kWarpPv) {
        if (lane == 0) run_pv<C>(p, sh, tmem);
    } else if (C::kF8 && warp >= kWarpWiden) {
        run_widen<C>(p, sh, (int)threadIdx.x - 32 * kWarpWiden);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace solo
}  // namespace mla

// sm_100a split kernel for paged MLA decode: 2-CTA pairs that split the query rows.
//
// One cluster of two CTAs (one per SM) owns one work unit, a contiguous run of pages of
// one or more work sequences (128-row query tiles of a sequence, see sched.cuh). CTA c
// holds query rows [64c, 64c+64) of the tile, all 576 dims of them, and its 64 x 512
// fp32 output rows: each CTA ends with complete rows, and the pair never exchanges
// scores. The pages are taken two at a time ("steps"): page A = k_lo + 2j is loaded
// whole (64 tokens x 576 dims) by CTA 0 and page B = A + 1 by CTA 1.
//
// The tensor work is 2-CTA tcgen05 MMAs (cta_group::2, M = 128 = 2 x 64 rows) issued by
// one thread of CTA 0. Measured on B200, every MMA instruction costs at least ~45
// cycles, so a 64-row slice only runs the tensor pipe at full rate with N >= 256 and at
// 70% with N = 128; hence two pages per step:
//   QK:  S = Q K^T, M = 128, N = 128 (each CTA supplies its page's 64 tokens), K = 576.
//        The lower 256 latent dims of Q come from TMEM, the rest from shared memory.
//        Each CTA gets S for its 64 rows and all 128 tokens of the step, laid out over
//        its 128 TMEM lanes: lanes [0,64) hold page A's tokens, [64,128) page B's.
//   PV:  O += P V, M = 128, N = 256 per instruction (two for the 512 dims), K = 128.
//        The B operand of one instruction must sit at the same shared-memory address in
//        both CTAs, CTA 0 supplying dims [256j, 256j+128) and CTA 1 dims
//        [256j+128, 256j+256) of the same tokens. So once QK of the step is done, each
//        CTA reloads (an L2 hit) the other page's half of those dims into the boxes of its
//        own stage that only QK needed: in both CTAs, boxes {0,1,4,5} then hold page A
//        and boxes {2,3,6,7} page B, each CTA's share of the dims.
//        O per CTA is 64 rows x 512 dims = 256 TMEM columns (2 x 128, lanes [0,64) the
//        first half of each 256-dim block, lanes [64,128) the second).
//
// Per CTA (320 threads):
//   warps 0-7 softmax, correction, epilogue in two groups that take alternate steps. In a
//             group, warp q reads TMEM lanes [32q, 32q+32): row 32(q%2) + lane, page
//             half q/2. The two halves of a row meet through shared memory for the row
//             max; the lazy reference max passes from step to step between the groups.
//             P (bf16) goes to shared memory as the A operand of PV.
//   warp 8    TMA producer: whole pages into a 2-stage ring (the stage frees when PV of
//             its step is done), the post-QK reloads, and L2 prefetch of pages ahead.
//             The pool is seen as a 3-D tensor {64 elements, rows, 9 chunks of 128 B}, so
//             one instruction lands a page as its 9 swizzled tiles (the TMA unit streams
//             8 KB boxes at barely half the rate of whole pages) and a reload is two
//             2-tile instructions. It also brings each item's 64 q rows: dims
//             [256,576) straight into their tiles, dims [0,256) into the (then idle) P
//             buffers, from where the softmax warps move them into TMEM. So the next
//             item's QK overlaps the previous item's epilogue.
//   warp 9    TMEM owner (both CTAs) and, in CTA 0, the MMA issuer.
// CTA 1's warps tell CTA 0's barriers that their Q or P is ready with a 4-byte
// asynchronous store whose completion counts bytes on the barrier (release at cluster
// scope without stalling the warp; a remote mbarrier arrive stalls its thread for over
// a thousand cycles). CTA 0's MMA thread arms those barriers with the bytes to expect.
// Shared memory: 2 stages x 9 boxes (64 tokens x 64 dims, 128-byte swizzle), Q's upper
// 320 dims (5 boxes), 2 P buffers (64 rows x 128 tokens), small exchange arrays.
// TMEM columns: O [0,256) fp32, Q lower latent [256,384) bf16x2 (the 2-CTA A-from-TMEM
// layout: rows 0-63 in lanes [0,64) and again in [64,128)), S0 [384,448), S1 [448,512).
// Scores stay in the log2 domain (scale * log2 e folded in). A row's reference max is
// raised only when a score exceeds it by more than kRescaleLog2, so O is rescaled rarely.
#pragma once

#include "common.cuh"
#include "items.cuh"
#include "ptx.cuh"

namespace mla {
namespace pair {

constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr int kPrefetchSteps = 1;                    // L2 prefetch distance in steps (fastest of 0-4)
constexpr float kRescaleLog2 = 8.0f;

constexpr uint32_t kBoxBytes = 64 * 128;             // 64 rows x 64 bf16, SW128
constexpr int kBoxesPerPage = 9;                     // 8 latent + 1 rope
constexpr uint32_t kStageBytes = kBoxesPerPage * kBoxBytes;          // 72 KB
constexpr uint32_t kPageBytes = kStageBytes;                         // one CTA's page
constexpr uint32_t kReloadBytes = 4 * kBoxBytes;                     // 32 KB
constexpr int kQsBoxes = 5;                          // Q dims [256, 576)
constexpr uint32_t kPBytes = 2 * kBoxBytes;          // 64 rows x 128 tokens bf16

constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffQs = kOffK + 2 * kStageBytes;
constexpr uint32_t kOffP = kOffQs + kQsBoxes * kBoxBytes;
constexpr uint32_t kOffMax = kOffP + 2 * kPBytes;             // [2 grp][2 par][2 half][64] f32
constexpr uint32_t kOffMref = kOffMax + 2 * 2 * 2 * 64 * 4;   // [2 par][64] f32
constexpr uint32_t kOffLsum = kOffMref + 2 * 64 * 4;          // [2 sum][2 grp][2 half][64] f32
constexpr uint32_t kOffBar = kOffLsum + 2 * 2 * 2 * 64 * 4;
enum : uint32_t {
    kBarKFull = 0,                  // [2] both pages of the step landed (CTA 0's copy used)
    kBarQkDone = kBarKFull + 2,     // [2] QK of the step done (both CTAs)
    kBarVFull = kBarQkDone + 2,     // [2] this CTA's reload landed
    kBarPReady = kBarVFull + 2,     // [2] P written and V ready in both CTAs (CTA 0's used)
    kBarPvDone = kBarPReady + 2,    // [2] PV of the step done (both CTAs)
    kBarQReady = kBarPvDone + 2,    // Q of the item in place in both CTAs (CTA 0's used)
    kBarQLand = kBarQReady + 1,     // the item's q rows landed in shared memory
    kBarOFree = kBarQLand + 1,      // O of the previous item read out in both CTAs (CTA 0's)
    kBarMaxX = kBarOFree + 1,       // [2 groups] row-max halves posted
    kBarMref = kBarMaxX + 2,        // [2 groups] reference max of the step posted
    kBarLsum = kBarMref + 2,        // both groups posted their row sums
    kBarDrain = kBarLsum + 1,       // the MMA issuer's last commit
    kBarStall = kBarDrain + 1,      // never completes (the timeout test hook waits on it)
    kNumBars = kBarStall + 1
};
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort flag, sink word
// bytes CTA 1 signals per phase: one 4-byte store per softmax warp that arrives
constexpr uint32_t kPReadyTx = 4 * 4;
constexpr uint32_t kQReadyTx = 8 * 4;
constexpr uint32_t kOFreeTx = 8 * 4;
constexpr uint32_t kQBytes = 9 * kBoxBytes;             // 64 q rows x 576 dims
constexpr uint32_t kSmemBytes = kOffMisc + 24;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;      // room to align the base to 1 KB
static_assert(kSmemAlloc <= 232448, "shared memory over the sm_100 per-block limit");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColQ = 256;
constexpr uint32_t kColS = 384;                          // + 64 * buffer

constexpr uint32_t kIdescQK = ptx::idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = ptx::idesc_bf16(128, 256, false, true);
constexpr uint16_t kBothCtas = 3;

struct Shared {
    uint8_t* base;
    uint32_t base_u32;
    __device__ uint32_t bar(uint32_t i) const { return base_u32 + kOffBar + 8 * i; }
    __device__ uint32_t stage(uint32_t s) const { return base_u32 + kOffK + s * kStageBytes; }
    __device__ float* fptr(uint32_t off) const { return reinterpret_cast<float*>(base + off); }
    __device__ volatile int* abort_flag() const {
        return reinterpret_cast<volatile int*>(base + kOffMisc + 8);
    }
    __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + kOffMisc); }
    __device__ uint32_t sink() const { return base_u32 + kOffMisc + 12; }
    // ns a wait may last before the kernel gives up (read only on the slow path)
    __device__ uint64_t wait_limit() const {
        return *reinterpret_cast<volatile uint64_t*>(base + kOffMisc + 16);
    }
};

// Bounded wait (as in every kernel of the library): false if the phase does not complete
// within the limit or another role of this CTA already gave up.
template <bool kCluster>
__device__ __forceinline__ bool wait_bar(const Shared& sh, uint32_t bar, uint32_t parity,
                                         uint32_t where) {
    if (kCluster ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = ptx::globaltimer();
    for (uint32_t it = 0;; ++it) {
        if (kCluster ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity))
            return true;
        if ((it & 255u) == 255u) {
            if (*sh.abort_flag()) return false;
            if (ptx::globaltimer() - t0 > sh.wait_limit()) {
                *sh.abort_flag() = 1;
                record_error(kErrTimeout, where);
                return false;
            }
        }
    }
}

// Warp-uniform bounded wait (no lane leaves a loop holding .sync.aligned instructions
// while its neighbours stay).
template <bool kCluster>
__device__ __forceinline__ bool warp_wait_bar(const Shared& sh, uint32_t bar, uint32_t parity,
                                              uint32_t where) {
    const bool ok = wait_bar<kCluster>(sh, bar, parity, where);
    return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------------ producer (warp 8)
// tm_page: box {64, 64 rows, 9 chunks} (a whole page); tm_pair: box {64, 64 rows, 2}.
// Step S uses stage S % 2. This CTA's page of the step is loaded whole once PV of step
// S - 2 has freed the stage; both CTAs' loads complete on CTA 0's barrier. Once QK of
// the step is done, the other page's share of this CTA's PV dims is reloaded into the
// four boxes that only QK needed (CTA 0: boxes 2,3,6,7 <- page B's 0,1,4,5; CTA 1: boxes
// 0,1,4,5 <- page A's 2,3,6,7), completing on this CTA's own barrier.
__device__ __forceinline__ void run_producer(const DecodeParams& p, const Shared& sh,
                                             const CUtensorMap* tm_page, const CUtensorMap* tm_pair,
                                             const CUtensorMap* tm_q4, const CUtensorMap* tm_q5,
                                             uint32_t crank) {
    if (g_mla_debug_stall) {
        // test hook: wait on a barrier nothing completes, before any copy is issued; the
        // wait gives up after the limit, so every role of the CTA stops with nothing in
        // flight and the timeout is recorded
        wait_bar<false>(sh, sh.bar(kBarStall), 0, 0x13u);
        return;
    }
    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    bool have = iter.next(it);
    // q stream: item m's rows may land once PV of item m-1's last step is done (the q
    // tiles, Q in TMEM and the P buffers are then free)
    ItemIter qiter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item qit;
    bool qhave = qiter.next(qit);
    uint32_t qitems = 0;
    int64_t q_prev_last = -1;                      // global last step of the previous item
    uint32_t q_first = 0;                          // global first step of item qit
    auto q_row = [&](const Item& x) { return (x.b * p.rows + x.t * kTileRows) + 64 * (int)crank; };
    int j = 0;                                     // step within the current item
    ItemIter piter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item pit;
    bool phave = piter.next(pit);
    int pj = 0;
    // L2 prefetch cursor over this CTA's pages, kPrefetchSteps steps ahead of the loads.
    // The first two steps are loaded at once, so the prefetches start only after them:
    // at launch every SM's first loads then reach HBM before any prefetch traffic.
    auto prefetch_next = [&](bool issue) {
        if (!phave) return;
        const int k = pit.k_lo + 2 * pj + (int)crank;
        if (issue && k < pit.k_hi) {
            const int pid = p.block_table[(size_t)pit.b * p.max_blocks + k];
            if (pid >= 0 && pid < p.num_blocks) ptx::tma_prefetch_3d(tm_page, 0, pid * kBlock, 0);
        }
        if (++pj >= pit.steps()) {
            phave = piter.next(pit);
            pj = 0;
        }
    };
    prefetch_next(false);
    prefetch_next(false);
    const uint32_t kfull_leader = ptx::mapa(sh.bar(kBarKFull), 0);
    int reload_row[4];                             // pool row of the other page, per step % 4
    uint32_t gk = 0, gv = 0;                       // steps loaded / reloaded
    // PV completions are observed strictly in step order: PV of step pv_seen + 2 needs
    // that step's page, which is only loaded after PV of step pv_seen was seen, so the
    // phase tested below can never be confused with an older one of the same parity
    uint32_t pv_seen = 0;
    uint64_t t0 = 0;
    uint32_t idle = 0;
    for (;;) {
        if (pv_seen < gk &&
            ptx::mbar_test_wait(sh.bar(kBarPvDone + (pv_seen & 1u)), (pv_seen >> 1) & 1u))
            ++pv_seen;
        if (qhave && (int64_t)pv_seen > q_prev_last) {
            const uint32_t land = sh.bar(kBarQLand);
            ptx::mbar_arrive_expect_tx(land, kQBytes);
            const int y = q_row(qit);
            ptx::tma_load_3d(sh.base_u32 + kOffQs, tm_q5, land, 0, y, 4);
            ptx::tma_load_3d(sh.base_u32 + kOffP, tm_q4, land, 0, y, 0);
            q_first += (uint32_t)qit.steps();
            q_prev_last = (int64_t)q_first - 1;
            ++qitems;
            qhave = qiter.next(qit);
            if (qhave) {                           // warm L2 for the next item's rows
                ptx::tma_prefetch_3d(tm_q5, 0, q_row(qit), 4);
                ptx::tma_prefetch_3d(tm_q4, 0, q_row(qit), 0);
            }
            idle = 0;
        } else if (gv < gk && ptx::mbar_test_wait(sh.bar(kBarQkDone + (gv & 1u)), (gv >> 1) & 1u)) {
            const uint32_t full = sh.bar(kBarVFull + (gv & 1u));
            ptx::mbar_arrive_expect_tx(full, kReloadBytes);
            const uint32_t st = sh.stage(gv & 1u);
            const int y = reload_row[gv & 3u];
            // CTA 0 fills boxes 2,3,6,7 from page B's 0,1,4,5; CTA 1 fills 0,1,4,5 from
            // page A's 2,3,6,7 (two boxes per instruction)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int src = 4 * i + 2 * (int)crank;                     // 0,4 (+2)
                const int dst = 4 * i + 2 * (int)(crank ^ 1u);
                ptx::tma_load_3d(st + dst * kBoxBytes, tm_pair, full, 0, y, src);
            }
            ++gv;
            idle = 0;
        } else if (have && gk < gv + 2 && gk < pv_seen + 2) {
            const int ka = it.k_lo + 2 * j;
            const int own = page_row(p, it.b, ka + (int)crank, it.k_hi);
            reload_row[gk & 3u] = page_row(p, it.b, ka + (int)(crank ^ 1u), it.k_hi);
            if (crank == 0) ptx::mbar_arrive_expect_tx(sh.bar(kBarKFull + (gk & 1u)), 2 * kPageBytes);
            const uint32_t st = sh.stage(gk & 1u);
            ptx::tma_load_3d_pair(st, tm_page, kfull_leader + 8 * (gk & 1u), 0, own, 0);
            // the holder of a split sequence's first chunk clears the combine's counters
            if (j == 0 && crank == 0 && it.chunk == 0 && it.n_chunks > 1 && it.v < p.max_chunks) {
                int* cnt = combine_counters(p) + (size_t)it.v * kCombineCounters;
#pragma unroll 1
                for (int i = 0; i < kCombineCounters; ++i) cnt[i] = 0;
            }
            ++gk;
            if (gk == 2)
                for (int i = 0; i < kPrefetchSteps; ++i) prefetch_next(true);
            else if (gk > 2)
                prefetch_next(true);
            if (++j >= it.steps()) {
                have = iter.next(it);
                j = 0;
            }
            idle = 0;
        } else if (!have && gv == gk && !qhave) {
            break;
        } else if ((++idle & 1023u) == 0) {
            if (*sh.abort_flag()) return;
            const uint64_t now = ptx::globaltimer();
            if (idle == 1024u) t0 = now;
            else if (now - t0 > sh.wait_limit()) {
                *sh.abort_flag() = 1;
                record_error(kErrTimeout, 0x10u);
                return;
            }
        }
    }
    // the last copies must land before this CTA may finish
    if (qitems > 0) wait_bar<false>(sh, sh.bar(kBarQLand), (qitems - 1) & 1u, 0x12u);
    for (uint32_t i = 0; i < 2 && i < gv; ++i) {
        const uint32_t g = gv - 1 - i;
        wait_bar<false>(sh, sh.bar(kBarVFull + (g & 1u)), (g >> 1) & 1u, 0x11u);
    }
}

// ------------------------------------------------------------------ MMA issuer (CTA 0)
// S of step S goes to TMEM buffer S % 2, free once PV of step S - 2 was issued (its P
// was written after the softmax had read that S).
// K-steps [k0, k1) of the 36 (16 dims each) of QK for step S; the part that ends at 36
// commits the step's QkDone.
template <int k0, int k1>
__device__ __forceinline__ void issue_qk(const Shared& sh, uint32_t tmem, uint32_t S) {
    const uint32_t b = S & 1u;
    ptx::tc_fence_after();
    const uint32_t d = tmem + kColS + 64 * b;
    const uint32_t st = sh.stage(b);
    const uint32_t qs = sh.base_u32 + kOffQs;
#pragma unroll
    for (int k = k0; k < k1; ++k) {
        const uint64_t bdesc = ptx::smem_desc(st + (k >> 2) * kBoxBytes + (k & 3) * 32, 16, 1024, 2);
        if (k < 16) {                              // latent dims [0,256): Q from TMEM
            ptx::mma_ts_pair(d, tmem + kColQ + 8 * k, bdesc, kIdescQK, k > 0 ? 1u : 0u);
        } else {                                   // dims [256,576): Q from shared memory
            const uint64_t adesc =
                ptx::smem_desc(qs + ((k - 16) >> 2) * kBoxBytes + (k & 3) * 32, 16, 1024, 2);
            ptx::mma_ss_pair(d, adesc, bdesc, kIdescQK, 1u);
        }
    }
    if constexpr (k1 == 36) ptx::mma_commit_pair(sh.bar(kBarQkDone + b), kBothCtas);
}

// O += P V for step S; `first` starts the item's accumulation.
__device__ __forceinline__ void issue_pv(const Shared& sh, uint32_t tmem, uint32_t S, bool first) {
    const uint32_t b = S & 1u;
    ptx::tc_fence_after();
    const uint32_t st = sh.stage(b);
    const uint32_t pa = sh.base_u32 + kOffP + b * kPBytes;
#pragma unroll
    for (int jd = 0; jd < 2; ++jd) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t adesc =
                ptx::smem_desc(pa + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024, 2);
            const uint32_t box = 4 * jd + 2 * (kk >> 2);       // page A: 4jd, page B: 4jd+2
            const uint64_t bdesc =
                ptx::smem_desc(st + box * kBoxBytes + (kk & 3) * 2048, kBoxBytes, 1024, 2);
            ptx::mma_ss_pair(tmem + kColO + 128 * jd, adesc, bdesc, kIdescPV,
                             (!first || kk > 0) ? 1u : 0u);
        }
    }
    ptx::mma_commit_pair(sh.bar(kBarPvDone + b), kBothCtas);
}

__device__ __forceinline__ void run_mma(const DecodeParams& p, const Shared& sh, uint32_t tmem) {
    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t S0 = 0;       // global index of the item's first step
    uint32_t items = 0;
    while (iter.next(it)) {
        if (!wait_bar<true>(sh, sh.bar(kBarQReady), items & 1u, 0x20u)) break;
        ptx::mbar_arrive_expect_tx(sh.bar(kBarQReady), kQReadyTx);      // the next item's
        ptx::tc_fence_after();
        bool o_free = items == 0;        // the previous item's O must be read out first
        const uint32_t n = (uint32_t)it.steps();
        uint32_t qk = 0, pv = 0;
        uint64_t t0 = 0;
        uint32_t idle = 0;
        bool ok = true;
        while (pv < n) {
            const uint32_t Sv = S0 + pv, Sq = S0 + qk;
            if (!o_free &&
                ptx::mbar_test_wait_cluster(sh.bar(kBarOFree), (items - 1) & 1u)) {
                ptx::mbar_arrive_expect_tx(sh.bar(kBarOFree), kOFreeTx);   // this item's
                ptx::tc_fence_after();
                o_free = true;
            }
            if (pv < qk && (pv > 0 || o_free) &&
                ptx::mbar_test_wait_cluster(sh.bar(kBarPReady + (Sv & 1u)), (Sv >> 1) & 1u)) {
                issue_pv(sh, tmem, Sv, pv == 0);
                ptx::mbar_arrive_expect_tx(sh.bar(kBarPReady + (Sv & 1u)), kPReadyTx);  // step Sv+2
                ++pv;
                idle = 0;
            } else if (qk < n && qk < pv + 2 &&
                       ptx::mbar_test_wait_cluster(sh.bar(kBarKFull + (Sq & 1u)), (Sq >> 1) & 1u)) {
                issue_qk<0, 36>(sh, tmem, Sq);
                ++qk;
                idle = 0;
            } else if ((++idle & 1023u) == 0) {
                if (*sh.abort_flag()) { ok = false; break; }
                const uint64_t now = ptx::globaltimer();
                if (idle == 1024u) t0 = now;
                else if (now - t0 > sh.wait_limit()) {
                    *sh.abort_flag() = 1;
                    record_error(kErrTimeout, 0x24u);
                    ok = false;
                    break;
                }
            }
        }
        if (!ok) break;
        S0 += n;
        ++items;
    }
    // every MMA this thread issued is complete before the CTA may finish
    ptx::mma_commit_pair(sh.bar(kBarDrain), 1);
    wait_bar<false>(sh, sh.bar(kBarDrain), 0, 0x25u);
}

// ------------------------------------------------------------------ softmax (warps 0-7)
__device__ __forceinline__ float f32(uint32_t x) { return __uint_as_float(x); }

struct SoftmaxCtx {
    uint32_t tmem, lane_base, crank;
    int row;          // query row within this CTA's 64 (TMEM lane mod 64)
    int half;         // page half of the step this thread scores (0: page A, 1: page B)
    int grp;          // group (0 or 1): takes the steps S with S % 2 == grp
};

struct RowState {
    float m_used;     // reference the sums are relative to (-inf: nothing yet)
    float l_sum;      // sum of 2^(s - m_used) over this thread's tokens (for the lse)
    float l_rnd;      // the same sum of the bf16-rounded values PV multiplies (normalises O)
};

__device__ __forceinline__ void rebase(RowState& st, float m) {
    if (m != st.m_used) {
        const float f = st.m_used == -INFINITY ? 0.f : ptx::ex2_ftz(st.m_used - m);
        st.l_sum *= f;
        st.l_rnd *= f;
        st.m_used = m;
    }
}

// Softmax of step S (the item's j-th) for this thread's row and page half.
__device__ __forceinline__ bool softmax_step(const DecodeParams& p, const Shared& sh,
                                             const SoftmaxCtx& c, const Item& it, int n_vis,
                                             uint32_t j, uint32_t S, RowState& st) {
    const uint32_t b = S & 1u;
    const int row = c.row;
    if (!warp_wait_bar<false>(sh, sh.bar(kBarQkDone + b), (S >> 1) & 1u, 0x30u)) return false;
    ptx::tc_fence_after();
    uint32_t sv[64];
    ptx::tmem_ld64(c.tmem + c.lane_base + kColS + 64 * b, sv);

    // scores in the log2 domain relative to the current reference, masked past the end
    const int page = it.k_lo + 2 * (int)j + c.half;
    const int lim = page < it.k_hi ? n_vis - page * kBlock : 0;   // valid: [0, lim)
    const float base = st.m_used == -INFINITY ? 0.f : st.m_used;
    const float L = p.scale_log2;
    float s[64];
    if (__all_sync(0xffffffffu, lim >= 64)) {
#pragma unroll
        for (int q = 0; q < 64; ++q) s[q] = fmaf(f32(sv[q]), L, -base);
    } else {
#pragma unroll
        for (int q = 0; q < 64; ++q) s[q] = q < lim ? fmaf(f32(sv[q]), L, -base) : -INFINITY;
    }
    float mx;
    {
        float m8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a)
            m8[a] = fmaxf(fmaxf(fmaxf(s[a], s[a + 8]), fmaxf(s[a + 16], s[a + 24])),
                          fmaxf(fmaxf(s[a + 32], s[a + 40]), fmaxf(s[a + 48], s[a + 56])));
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    }
    // the row's other half (same group, warp q ^ 2)
    const uint32_t par = (S >> 1) & 1u;
    float* mxbuf = sh.fptr(kOffMax) + ((c.grp * 2 + par) * 2) * 64;
    mxbuf[c.half * 64 + row] = mx;
    ptx::mbar_arrive(sh.bar(kBarMaxX + c.grp));
    if (!warp_wait_bar<false>(sh, sh.bar(kBarMaxX + c.grp), par, 0x31u)) return false;
    mx = fmaxf(mx, *reinterpret_cast<volatile float*>(&mxbuf[(c.half ^ 1) * 64 + row]));
    const float mx_abs = mx + base;

    // reference after step S-1 (the other group), then this step's decision: raise only
    // when a score exceeds it by more than the threshold. Both halves decide alike.
    float* mref = sh.fptr(kOffMref);
    float m_prev = -INFINITY;
    if (j > 0) {
        if (!warp_wait_bar<false>(sh, sh.bar(kBarMref + (c.grp ^ 1)), ((S - 1) >> 1) & 1u, 0x36u))
            return false;
        m_prev = *reinterpret_cast<volatile float*>(&mref[((S - 1) & 1u) * 64 + row]);
    }
    const bool raise = m_prev == -INFINITY ? mx_abs > -INFINITY : mx_abs > m_prev + kRescaleLog2;
    const float m_new = raise ? mx_abs : m_prev;
    if (c.half == 0) mref[(S & 1u) * 64 + row] = m_new;
    ptx::mbar_arrive(sh.bar(kBarMref + c.grp));

    if (m_new != base && m_new != -INFINITY) {
        const float d = m_new - base;
#pragma unroll
        for (int q = 0; q < 64; ++q) s[q] -= d;
    }
    rebase(st, m_new);
    // O follows a raise: after PV of step S-1, scale this lane's 256 O columns
    const bool need_o = raise && j > 0 && m_prev != -INFINITY;
    if (__any_sync(0xffffffffu, need_o)) {
        if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (b ^ 1u)), ((S - 1) >> 1) & 1u, 0x33u))
            return false;
        ptx::tc_fence_after();
        const float f = need_o ? ptx::ex2_ftz(m_prev - m_new) : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
            uint32_t ov[32];
            const uint32_t oaddr = c.tmem + c.lane_base + kColO + 32 * cc;
            ptx::tmem_ld32(oaddr, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(f32(ov[e]) * f);
            ptx::tmem_st32(oaddr, ov);
        }
        ptx::tmem_wait_st();
    }
    uint32_t pk[32];
    float rs0 = 0.f, rs1 = 0.f, rr0 = 0.f, rr1 = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const float p0 = ptx::ex2_ftz(s[2 * q]);
        const float p1 = ptx::ex2_ftz(s[2 * q + 1]);
        rs0 += p0;
        rs1 += p1;
        // O is normalised by the sum of the bf16 values PV multiplies, so it is a weighted
        // mean of V rows whose weights sum to one: a dominant token's rounding (its P may
        // be up to 2^kRescaleLog2, not 1) then cancels instead of scaling the output. The
        // lse keeps the exact sum.
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        rr0 += __low2float(h2);
        rr1 += __high2float(h2);
        pk[q] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    st.l_sum += rs0 + rs1;
    st.l_rnd += rr0 + rr1;

    // P buffer b is free once PV of step S-2 has completed
    if (S >= 2 && !warp_wait_bar<false>(sh, sh.bar(kBarPvDone + b), ((S - 2) >> 1) & 1u, 0x35u))
        return false;
    {
        // row of P: this half's 64 tokens = 8 chunks of 16 B in box `half`, K-major SW128
        const uint32_t prow = sh.base_u32 + kOffP + b * kPBytes + (uint32_t)c.half * kBoxBytes +
                              (uint32_t)row * 128;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
            ptx::st_shared_v4(prow + (((uint32_t)cc ^ (uint32_t)(row & 7)) * 16), pk[4 * cc],
                              pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
    }
    // this CTA's reload must have landed; then zero V rows past the sequence end on a
    // partial page (they may hold stale or NaN data, and P = 0 would not cancel NaN)
    if (!warp_wait_bar<false>(sh, sh.bar(kBarVFull + b), (S >> 1) & 1u, 0x39u)) return false;
    {
        const uint32_t stg = sh.stage(b);
        const int gtid = c.half * 64 + row;      // 0..127 within the step's group
#pragma unroll
        for (int pg = 0; pg < 2; ++pg) {
            const int pidx = it.k_lo + 2 * (int)j + pg;
            if (pidx >= it.k_hi) continue;
            const int tail = it.L - pidx * kBlock;
            if (tail >= kBlock) continue;
            const int nbad = kBlock - tail;
            // boxes 4jd + 2pg + (0,1), jd = 0,1: 4 boxes x nbad rows x 8 chunks
            for (int q = gtid; q < nbad * 32; q += 128) {
                const int rr = tail + (q >> 5);
                const int bx = (q >> 3) & 3;
                const int box = (bx & 1) + 4 * (bx >> 1) + 2 * pg;
                const int ch = q & 7;
                ptx::st_shared_v4(stg + box * kBoxBytes + rr * 128 + ch * 16, 0, 0, 0, 0);
            }
        }
    }
    ptx::fence_proxy_async_smem();            // P and zeroed rows visible to the MMA
    ptx::tc_fence_before();                   // S read before QK of step S+2 overwrites it
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        if (c.crank == 0) ptx::mbar_arrive(sh.bar(kBarPReady + b));
        else ptx::st_async_signal(ptx::mapa(sh.sink(), 0), ptx::mapa(sh.bar(kBarPReady + b), 0));
    }
    return true;
}

// Where one item's rows stand once its steps are done: what its epilogue needs.
struct ItemEnd {
    Item it;
    int r, qi;
    bool row_valid;
    uint32_t last_step;      // global index of the item's last step
    RowState st;
};

// Epilogue of an item for this thread's row: merge the four row sums (two groups x two
// page halves), then write this lane's 128 output dims (dims block `grp`, half `half`)
// normalised, with the lse, or the fp32 partial for the combine.
__device__ __forceinline__ bool epilogue(const DecodeParams& p, const Shared& sh,
                                         const SoftmaxCtx& c, ItemEnd& e, uint32_t epi_index) {
    const int row = c.row;
    const uint32_t Sl = e.last_step;
    if (!warp_wait_bar<false>(sh, sh.bar(kBarMref + (Sl & 1u)), (Sl >> 1) & 1u, 0x38u)) return false;
    const float m_fin = *reinterpret_cast<volatile float*>(&sh.fptr(kOffMref)[(Sl & 1u) * 64 + row]);
    rebase(e.st, m_fin);
    float* lsum = sh.fptr(kOffLsum);
    lsum[(c.grp * 2 + c.half) * 64 + row] = e.st.l_sum;
    lsum[256 + (c.grp * 2 + c.half) * 64 + row] = e.st.l_rnd;
    ptx::mbar_arrive(sh.bar(kBarLsum));
    if (!warp_wait_bar<false>(sh, sh.bar(kBarLsum), epi_index & 1u, 0x37u)) return false;
    if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (Sl & 1u)), (Sl >> 1) & 1u, 0x34u)) return false;
    ptx::tc_fence_after();
    volatile float* vl = lsum;
    const float l_tot = (vl[row] + vl[64 + row]) + (vl[128 + row] + vl[192 + row]);
    const float l_rnd = (vl[256 + row] + vl[320 + row]) + (vl[384 + row] + vl[448 + row]);
    const bool empty = !(l_tot > 0.f);
    const float inv = empty ? 0.f : 1.f / l_rnd;
    const float lse2 = empty ? -INFINITY : m_fin + __log2f(l_tot);
    const Item& it = e.it;
    const bool final_out = it.n_chunks == 1;
    const bool have_ws = it.part < p.max_chunks;
    if (!final_out && !have_ws && row == 0 && c.grp == 0 && c.half == 0)
        record_error(kErrWorkspace, (uint32_t)it.v & 0xffffffu);
    const int tile_row = (int)c.crank * 64 + row;
    // The rows leave through shared memory, so that each store instruction writes whole
    // row segments instead of 16 bytes of 32 different rows. A warp stages its 32 rows x
    // 32 columns in its own 4 KB of the P region: exactly the bytes that only this warp
    // writes P into (warp 4g + q holds P rows of buffer g, page half q / 2, rows
    // 32 (q % 2) ..), and every warp moved its q rows out of the region before the row-sum
    // barrier above. The P buffers are idle here: PV of the item's last step is done and
    // the next item's first P comes after this epilogue.
    const int lane = (int)(threadIdx.x & 31);
    const uint32_t stg = sh.base_u32 + kOffP + (threadIdx.x >> 5) * 4096u;
    const int row0 = row - lane;                              // the warp's first row
    const bool fp32_out = !final_out || p.out_f32 != nullptr;
    float* const f32_base = final_out ? p.out_f32 : p.ws_o;
    const bool write_any = final_out || have_ws;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
        uint32_t ov[32];
        ptx::tmem_ld32(c.tmem + c.lane_base + kColO + 128 * c.grp + 32 * cc, ov);
        if (!write_any) continue;
        const int col = 256 * c.grp + 128 * c.half + 32 * cc;
        if (fp32_out) {
            // stage: lane i's 128-byte row, 16-byte chunks XOR-swizzled by i % 8
#pragma unroll
            for (int k = 0; k < 8; ++k)
                ptx::st_shared_v4(stg + lane * 128 + ((k ^ (lane & 7)) * 16),
                                  __float_as_uint(f32(ov[4 * k]) * inv),
                                  __float_as_uint(f32(ov[4 * k + 1]) * inv),
                                  __float_as_uint(f32(ov[4 * k + 2]) * inv),
                                  __float_as_uint(f32(ov[4 * k + 3]) * inv));
            __syncwarp();
            // write: 4 rows x 128 bytes per instruction (8 lanes per row)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 4 * i + (lane >> 3), k = lane & 7;
                const uint4 v = ptx::ld_shared_v4(stg + r * 128 + ((k ^ (r & 7)) * 16));
                const int lr = row0 + r;                          // row within this CTA's 64
                const int qr = it.t * kTileRows + (int)c.crank * 64 + lr;
                if (qr < p.rows) {
                    const size_t grow = final_out ? (size_t)it.b * p.rows + qr
                                                  : (size_t)it.part * kTileRows + (int)c.crank * 64 + lr;
                    *reinterpret_cast<uint4*>(f32_base + grow * kHeadDimV + col + 4 * k) = v;
                }
            }
        } else {
            // stage: lane i's 64-byte bf16 row, chunks XOR-swizzled by (i / 2) % 4
            uint32_t w[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(f32(ov[2 * h]) * inv, f32(ov[2 * h + 1]) * inv);
                w[h] = *reinterpret_cast<uint32_t*>(&b2);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k)
                ptx::st_shared_v4(stg + lane * 64 + ((k ^ ((lane >> 1) & 3)) * 16),
                                  w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
            __syncwarp();
            // write: 8 rows x 64 bytes per instruction (4 lanes per row)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 8 * i + (lane >> 2), k = lane & 3;
                const uint4 v = ptx::ld_shared_v4(stg + r * 64 + ((k ^ ((r >> 1) & 3)) * 16));
                const int qr = it.t * kTileRows + (int)c.crank * 64 + row0 + r;
                if (qr < p.rows)
                    *reinterpret_cast<uint4*>(p.out + ((size_t)it.b * p.rows + qr) * kHeadDimV + col + 8 * k) = v;
            }
        }
        __syncwarp();                      // staging reads done before the next chunk's writes
    }
    if (e.row_valid && c.grp == 0 && c.half == 0) {
        if (final_out) {
            const int h = e.r % p.h_q;
            p.lse[((size_t)it.b * p.h_q + h) * p.s_q + e.qi] = empty ? -INFINITY : lse2 * kLn2;
        } else if (have_ws) {
            p.ws_lse[(size_t)it.part * kTileRows + tile_row] = lse2;
        }
    }

    ptx::tc_fence_before();
    return true;
}

// Tell CTA 0's barrier `bar` that this warp is done (local arrive in CTA 0; in CTA 1 a
// 4-byte store whose completion counts on that barrier).
__device__ __forceinline__ void signal_leader(const Shared& sh, uint32_t crank, uint32_t bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) {
        if (crank == 0) ptx::mbar_arrive(sh.bar(bar));
        else ptx::st_async_signal(ptx::mapa(sh.sink(), 0), ptx::mapa(sh.bar(bar), 0));
    }
}

__device__ __forceinline__ void run_softmax(const DecodeParams& p, const Shared& sh, uint32_t tmem,
                                            uint32_t crank, int warp, int lane) {
    SoftmaxCtx c;
    const int q = warp & 3;
    c.tmem = tmem;
    c.crank = crank;
    c.lane_base = (uint32_t)(q * 32) << 16;
    c.row = (q & 1) * 32 + lane;
    c.half = q >> 1;
    c.grp = warp >> 2;
    const int row = c.row;
    (void)lane;

    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t S = 0;
    uint32_t items = 0;
    ItemEnd prev;
    bool have_prev = false;
    while (iter.next(it)) {
        const int r = it.t * kTileRows + (int)crank * 64 + row;   // query row in the sequence
        const bool row_valid = r < p.rows;
        const int qi = row_valid ? r / p.h_q : 0;
        const int n_vis = row_valid ? visible_tokens(it.L, p.s_q, qi, p.causal) : 0;

        // ---- q of this row, dims [0,256): from the P buffers (where the producer landed
        // them) into TMEM, both lane halves (group g moves dims [128g, 128g+128))
        if (!warp_wait_bar<false>(sh, sh.bar(kBarQLand), items & 1u, 0x3au)) return;
        {
            const uint32_t qaddr = tmem + c.lane_base + kColQ + 64 * c.grp;
            const uint32_t stg = sh.base_u32 + kOffP + (uint32_t)row * 128;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t v[32];
                const uint32_t tile = stg + (uint32_t)(2 * c.grp + cc) * kBoxBytes;
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const uint32_t a = tile + (((uint32_t)jj ^ (uint32_t)(row & 7)) * 16);
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(v[4 * jj]), "=r"(v[4 * jj + 1]), "=r"(v[4 * jj + 2]),
                                   "=r"(v[4 * jj + 3])
                                 : "r"(a) : "memory");
                }
                ptx::tmem_st32(qaddr + 32 * cc, v);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            signal_leader(sh, crank, kBarQReady);
        }

        // ---- the previous item's epilogue overlaps this item's first QK
        if (have_prev) {
            if (!epilogue(p, sh, c, prev, items - 1)) return;
            signal_leader(sh, crank, kBarOFree);
        }

        RowState st{-INFINITY, 0.f, 0.f};
        const uint32_t n = (uint32_t)it.steps();
        const uint32_t S0 = S;
        bool ok = true;
        for (uint32_t j = (S0 & 1u) == (uint32_t)c.grp ? 0u : 1u; j < n; j += 2) {
            if (!softmax_step(p, sh, c, it, n_vis, j, S0 + j, st)) { ok = false; break; }
        }
        if (!ok) return;
        S = S0 + n;
        prev.it = it;
        prev.r = r;
        prev.qi = qi;
        prev.row_valid = row_valid;
        prev.last_step = S - 1;
        prev.st = st;
        have_prev = true;
        ++items;
    }
    if (have_prev) epilogue(p, sh, c, prev, items - 1);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_page,
              const __grid_constant__ CUtensorMap tm_pair, const __grid_constant__ CUtensorMap tm_q4,
              const __grid_constant__ CUtensorMap tm_q5) {
    extern __shared__ uint8_t smem_raw[];
    Shared sh;
    {
        const uint32_t raw = ptx::smem_u32(smem_raw);
        const uint32_t aligned = (raw + 1023u) & ~1023u;
        sh.base = smem_raw + (aligned - raw);
        sh.base_u32 = aligned;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = ptx::cluster_ctarank();

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(sh.bar(kBarKFull + i), 1);
            ptx::mbar_init(sh.bar(kBarQkDone + i), 1);
            ptx::mbar_init(sh.bar(kBarVFull + i), 1);
            ptx::mbar_init(sh.bar(kBarPReady + i), 4 + 1);      // CTA 0's warps + arming
            ptx::mbar_init(sh.bar(kBarPvDone + i), 1);
            ptx::mbar_init(sh.bar(kBarMaxX + i), 128);
            ptx::mbar_init(sh.bar(kBarMref + i), 128);
        }
        ptx::mbar_init(sh.bar(kBarQReady), 8 + 1);              // CTA 0's warps + arming
        ptx::mbar_init(sh.bar(kBarQLand), 1);
        ptx::mbar_init(sh.bar(kBarOFree), 8 + 1);               // CTA 0's warps + arming
        ptx::mbar_init(sh.bar(kBarLsum), kSoftmaxThreads);
        ptx::mbar_init(sh.bar(kBarDrain), 1);
        ptx::mbar_init(sh.bar(kBarStall), 1);
        *sh.abort_flag() = 0;
        *reinterpret_cast<volatile uint64_t*>(sh.base + kOffMisc + 16) = g_mla_wait_limit_ns;
        ptx::fence_mbarrier_init_cluster();
        // arm the first phases of the barriers CTA 1 signals with byte counts
        ptx::mbar_arrive_expect_tx(sh.bar(kBarPReady + 0), kPReadyTx);
        ptx::mbar_arrive_expect_tx(sh.bar(kBarPReady + 1), kPReadyTx);
        ptx::mbar_arrive_expect_tx(sh.bar(kBarQReady), kQReadyTx);
        ptx::mbar_arrive_expect_tx(sh.bar(kBarOFree), kOFreeTx);
        ptx::prefetch_tensormap(&tm_page);
        ptx::prefetch_tensormap(&tm_pair);
        ptx::prefetch_tensormap(&tm_q4);
        ptx::prefetch_tensormap(&tm_q5);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc_pair(ptx::smem_u32(sh.tmem_slot()), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();            // peer barriers initialised before any remote access
    ptx::tc_fence_after();
    const uint32_t tmem = *sh.tmem_slot();
    grid_dependency_wait();         // the schedule is written

    if (warp < kWarpProducer) {
        run_softmax(p, sh, tmem, crank, warp, lane);
    } else if (warp == kWarpProducer) {
        if (lane == 0) run_producer(p, sh, &tm_page, &tm_pair, &tm_q4, &tm_q5, crank);
    } else if (warp == kWarpMma) {
        if (lane == 0 && crank == 0) run_mma(p, sh, tmem);
    }

    // after a failure some copies may still be in flight: give them time to land
    if (*sh.abort_flag()) {
        const uint64_t t0 = ptx::globaltimer();
        while (ptx::globaltimer() - t0 < 50000ull) {}
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();            // no remote access may target an exited CTA
    if (warp == kWarpMma) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace pair
}  // namespace mla

// sm_100a split kernel for paged MLA decode.
//
// One 2-CTA cluster owns one work unit (a contiguous run of pages, see sched.cuh) and
// processes 128 query rows against one 64-token page at a time. Per SM the 128 x 512
// fp32 output accumulator alone would fill all of TMEM (128 lanes x 512 columns), and
// the 128 x 576 bf16 query tile plus a 64 x 576 page would crowd shared memory. So
// the pair splits the 576 dims: CTA c holds latent dims [256c, 256c+256) and rope dims
// [512+32c, 512+32c+32) of q and of every page, computes the partial scores over its
// 288 dims, and owns output columns [256c, 256c+256). The two partial score tiles are
// exchanged through distributed shared memory, so no FLOP or HBM byte is duplicated.
// Shared-memory traffic between SMs is slow (about 15 B/clock/SM for bulk copies), so
// each row's 64 partial scores travel as 16-bit fixed point with a per-row scale (the
// row's largest magnitude over its visible tokens maps to 32767): 16.5 KB per page
// instead of 32 KB, error at most 2^-16 of that magnitude. Each CTA's softmax adds its
// own quantised partial (the staging buffer it just shipped) to the peer's, so both CTAs
// see the same scores and take the same decisions.
//
// Per CTA (512 threads, four warpgroups whose registers are rebalanced at start):
//   warps 0-7 softmax / correction / epilogue in two warpgroups that take alternate
//             pages (page G goes to group G % 2), one thread per query row (TMEM lane):
//             while one group exponentiates its page, the other combines the next. The
//             lazy reference max of each row is handed from page G-1 to page G through
//             shared memory, so both groups scale P identically; each group keeps its
//             own row sum and the two are merged at the end of the item.
//   warps 8-11 senders: the only readers of S in TMEM. They quantise each page's
//             partial scores into a local staging buffer (read by this CTA's softmax) and
//             bulk-copy it into the peer's exchange buffer. S is free again right after,
//             so QK runs up to three pages ahead of PV and hides the exchange latency.
//   warp 12   TMA producer: page ids from the block table. Each page is loaded twice:
//             its 288 dims (4 SW128 latent boxes + 1 SW64 rope box) into a 2-stage QK
//             ring that frees as soon as QK completes, and its 256 latent dims again into
//             a 2-stage V ring just in time for PV (an L2 hit by then; pages are also
//             prefetched into L2 ahead of the QK stream). A page's bytes thus never sit in
//             shared memory through the score exchange and softmax.
//   warp 13   TMEM owner and MMA issuer (one thread): S = Q K^T (M=128, N=64, K=288;
//             the latent part reads Q from TMEM, the rope part from shared memory) into
//             S, and O += P V (M=128, N=256, K=64; P from one of two TMEM buffers, V the
//             page's latent boxes read MN-major). Whichever MMA is ready is
//             issued, so QK of later pages overlaps the exchange of earlier ones.
//   warp 14   relay: tells the peer when this CTA's softmax has read an exchange buffer
//             (a remote mbarrier arrive, whose release fence would otherwise stall the
//             senders). Warp 15 idles to complete the last warpgroup.
// TMEM columns: O [0,256) fp32, Q latent [256,384) bf16x2, S [384,448) fp32,
// P0 [448,480) and P1 [480,512) bf16x2.
// Scores stay in the log2 domain (scale * log2 e folded in). The running max is only
// raised when a new score exceeds it by more than kRescaleLog2, so O is rescaled rarely.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kThreads = 512;
constexpr int kSoftmaxThreads = 256;
constexpr int kWarpSender0 = 8;
constexpr int kWarpControl0 = 12;
constexpr int kWarpProducer = 12;
constexpr int kWarpMma = 13;
constexpr int kWarpRelay = 14;
// Registers per thread after rebalancing: 256 * 160 + 128 * (104 + 72) = 63488, within
// the 512 * 128 = 65536 the CTA is launched with.
constexpr uint32_t kRegsSoftmax = 160;
constexpr uint32_t kRegsSender = 104;
constexpr uint32_t kRegsControl = 72;
constexpr uint32_t kRegsNeeded =
    kSoftmaxThreads * kRegsSoftmax + 128 * kRegsSender + 128 * kRegsControl;
constexpr int kQkStages = 2;
constexpr int kVStages = 2;
constexpr int kPidRing = 16;                         // page ids issued to QK, kept for V
constexpr int kPrefetchPages = 6;                    // L2 prefetch distance of the QK stream
constexpr int kLatentHalf = 256;                     // latent dims per CTA
constexpr int kRopeHalf = 32;                        // rope dims per CTA
constexpr uint32_t kBoxBytes = 64 * 64 * 2;          // one SW128 box: 64 tokens x 64 dims
constexpr uint32_t kRopeBoxBytes = 64 * 32 * 2;      // one SW64 box: 64 tokens x 32 dims
constexpr uint32_t kQkStageBytes = 4 * kBoxBytes + kRopeBoxBytes;   // 36 KB
constexpr uint32_t kVStageBytes = 4 * kBoxBytes;                    // 32 KB
constexpr uint32_t kQropeBytes = 128 * kRopeHalf * 2;             // 8 KB
// Exchange buffer (and its staging twin): 128 rows x 64 biased 16-bit scores (128 B per
// row, 16-byte chunks XOR-swizzled by row % 8 so row-per-thread access is conflict-free)
// followed by the 128 per-row fp32 scales.
constexpr uint32_t kXDataBytes = 128 * 128;
constexpr uint32_t kXBytes = kXDataBytes + 128 * 4;  // 16896
constexpr uint32_t kXPayload = kXBytes;              // bytes the peer sends per page
constexpr float kQuantMax = 32767.f;

constexpr uint32_t kOffQk = 0;
constexpr uint32_t kOffV = kOffQk + kQkStages * kQkStageBytes;
constexpr uint32_t kOffQrope = kOffV + kVStages * kVStageBytes;
constexpr uint32_t kOffX = kOffQrope + kQropeBytes;          // [2] receive buffers
constexpr uint32_t kOffXStage = kOffX + 2 * kXBytes;         // [2] staging buffers
constexpr uint32_t kOffMref = kOffXStage + 2 * kXBytes;      // [128] fp32 reference max per row
constexpr uint32_t kOffLsum = kOffMref + 128 * 4;            // [2 groups][128] fp32
constexpr uint32_t kOffBar = kOffLsum + 2 * 128 * 4;
// barriers (8 B each)
enum : uint32_t {
    kBarQkFull = 0,                   // [kQkStages] page landed -> MMA (QK)
    kBarQkEmpty = kBarQkFull + 2,     // [kQkStages] QK done -> TMA
    kBarVFull = kBarQkEmpty + 2,      // [kVStages] latent dims landed -> MMA (PV), softmax
    kBarVEmpty = kBarVFull + 2,       // [kVStages] PV done -> TMA
    kBarSFull = kBarVEmpty + 2,       // [2] QK of page G done (G % 2) -> senders
    kBarSFree = kBarSFull + 2,        // senders read S -> MMA
    kBarPReady = kBarSFree + 1,       // [2] P written -> MMA
    kBarPvDone = kBarPReady + 2,      // [2] PV done -> softmax
    kBarXFull = kBarPvDone + 2,       // [2] peer scores landed (tx count)
    kBarXRead = kBarXFull + 2,        // [2] softmax read exchange buffer -> senders
    kBarXFree = kBarXRead + 2,        // [2] peer's softmax read what we sent
    kBarQReady = kBarXFree + 2,       // query tile in TMEM / smem
    kBarStage = kBarQReady + 1,       // [2] staging buffer written -> sending thread, softmax
    kBarMref = kBarStage + 2,         // [2] page G's reference max published (G % 2)
    kBarLsum = kBarMref + 2,          // both groups posted their row sums
    kNumBars = kBarLsum + 1
};
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;      // room to align the base to 1 KB

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColQ = 256;
constexpr uint32_t kColS = 384;
constexpr uint32_t kColP = 448;                          // + 32 * buffer

constexpr float kRescaleLog2 = 8.0f;

constexpr uint32_t kIdescQK = ptx::idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescPV = ptx::idesc_bf16(128, 256, false, true);

constexpr uint64_t kWaitLimitNs = 2000000000ull;         // 2 s per wait, then give up

struct Shared {
    uint8_t* base;
    uint32_t base_u32;
    __device__ uint32_t bar(uint32_t i) const { return base_u32 + kOffBar + 8 * i; }
    __device__ uint32_t qk_stage(uint32_t s) const { return base_u32 + kOffQk + s * kQkStageBytes; }
    __device__ uint32_t v_stage(uint32_t s) const { return base_u32 + kOffV + s * kVStageBytes; }
    __device__ volatile int* abort_flag() const {
        return reinterpret_cast<volatile int*>(base + kOffMisc + 8);
    }
    __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + kOffMisc); }
};

// Bounded wait. Returns false (and records a timeout) if the phase does not complete
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
            if (ptx::globaltimer() - t0 > kWaitLimitNs) {
                *sh.abort_flag() = 1;
                record_error(kErrTimeout, where);
                return false;
            }
        }
    }
}

// Warp-uniform bounded wait: every lane waits, and the warp proceeds only if all lanes
// saw the phase complete, so no lane can leave a loop whose body holds .sync.aligned
// tcgen05 instructions while its neighbours stay in it.
template <bool kCluster>
__device__ __forceinline__ bool warp_wait_bar(const Shared& sh, uint32_t bar, uint32_t parity,
                                              uint32_t where) {
    const bool ok = wait_bar<kCluster>(sh, bar, parity, where);
    return __all_sync(0xffffffffu, ok);
}

// One piece of work: pages [k_lo, k_hi) of work sequence v.
struct Item {
    int v, b, t, L, k_lo, k_hi, chunk, n_chunks, part;
};

// Iterates the items of every unit this cluster owns, in the same order for all roles.
struct ItemIter {
    const DecodeParams& p;
    int u, num_units, V, step;
    int v, v_end, k_begin, k_end, chunk_begin, v_begin;
    __device__ ItemIter(const DecodeParams& pp, int first_unit, int unit_step)
        : p(pp), u(first_unit - unit_step), step(unit_step) {
        num_units = p.metadata[0];
        V = p.batch * p.tiles;
        v = 1;
        v_end = 0;
    }
    __device__ bool next(Item& it) {
        for (;;) {
            if (v > v_end || v >= V) {
                u += step;
                if (u >= num_units) return false;
                const int32_t* m = p.metadata + kMetaInts * (u + 1);
                v_begin = m[0]; k_begin = m[1]; v_end = m[2]; k_end = m[3]; chunk_begin = m[4];
                v = v_begin;
                continue;
            }
            const int vv = v++;
            it.v = vv;
            it.b = vv % p.batch;
            it.t = vv / p.batch;
            it.L = checked_seqlen(p, it.b);
            const int nblk = pages_of(it.L);
            it.k_lo = vv == v_begin ? k_begin : 0;
            it.k_hi = vv == v_end ? k_end : nblk;
            if (it.k_hi > nblk) it.k_hi = nblk;
            if (it.k_lo >= it.k_hi) continue;
            it.chunk = vv == v_begin ? chunk_begin : 0;
            it.n_chunks = p.num_splits[vv + 1] - p.num_splits[vv];
            it.part = p.num_splits[vv] + it.chunk;
            return true;
        }
    }
};

// ------------------------------------------------------------------ producer (warp 12)
// One thread drives two TMA streams: the QK stream walks the pages in order, loading each
// page's 288 dims into the QK ring as soon as a QK stage frees; the V stream follows it,
// loading the same pages' 256 latent dims into the V ring as soon as a V stage frees (PV
// of the page two earlier is done). Whichever stream can move does, V first. Pages
// kPrefetchPages ahead of the QK stream are prefetched into L2, so that HBM latency is
// paid outside the shared-memory rings.
__device__ __forceinline__ void run_producer(const DecodeParams& p, const Shared& sh,
                                             const CUtensorMap* tm_lat, const CUtensorMap* tm_rope,
                                             uint32_t crank) {
    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    bool have = iter.next(it);
    int k = have ? it.k_lo : 0;
    // prefetch cursor: the same page sequence, kPrefetchPages ahead
    ItemIter piter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item pit;
    bool phave = piter.next(pit);
    int pk = phave ? pit.k_lo : 0;
    const int x_lat0 = (int)crank * kLatentHalf;
    const int x_rope0 = 512 + (int)crank * kRopeHalf;
    auto prefetch_next = [&]() {
        if (!phave) return;
        const int pid = p.block_table[(size_t)pit.b * p.max_blocks + pk];
        if (pid >= 0 && pid < p.num_blocks) {
#pragma unroll
            for (int i = 0; i < 4; ++i) ptx::tma_prefetch_2d(tm_lat, x_lat0 + 64 * i, pid * kBlock);
            ptx::tma_prefetch_2d(tm_rope, x_rope0, pid * kBlock);
        }
        if (++pk >= pit.k_hi) {
            phave = piter.next(pit);
            pk = phave ? pit.k_lo : 0;
        }
    };
    for (int i = 0; i < kPrefetchPages; ++i) prefetch_next();
    int pid_ring[kPidRing];
    uint32_t gq = 0, gv = 0;                          // pages issued on each stream
    const int x_lat = (int)crank * kLatentHalf;
    const int x_rope = 512 + (int)crank * kRopeHalf;
    uint64_t t0 = 0;
    uint32_t idle = 0;
    for (;;) {
        if (gv < gq && (gv < (uint32_t)kVStages ||
                        ptx::mbar_test_wait(sh.bar(kBarVEmpty + gv % kVStages),
                                           ((gv / kVStages) - 1) & 1u))) {
            const uint32_t full = sh.bar(kBarVFull + gv % kVStages);
            ptx::mbar_arrive_expect_tx(full, kVStageBytes);
            const uint32_t dst = sh.v_stage(gv % kVStages);
            const int y = pid_ring[gv % kPidRing] * kBlock;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ptx::tma_load_2d(dst + i * kBoxBytes, tm_lat, full, x_lat + 64 * i, y);
            ++gv;
            idle = 0;
        } else if (have && gq < gv + kPidRing &&
                   (gq < (uint32_t)kQkStages ||
                    ptx::mbar_test_wait(sh.bar(kBarQkEmpty + gq % kQkStages),
                                       ((gq / kQkStages) - 1) & 1u))) {
            int pid = p.block_table[(size_t)it.b * p.max_blocks + k];
            if (pid < 0 || pid >= p.num_blocks) {
                record_error(kErrBadInput, 0x800000u | ((uint32_t)it.b & 0x7fffffu));
                pid = 0;
            }
            pid_ring[gq % kPidRing] = pid;
            const uint32_t full = sh.bar(kBarQkFull + gq % kQkStages);
            ptx::mbar_arrive_expect_tx(full, kQkStageBytes);
            const uint32_t dst = sh.qk_stage(gq % kQkStages);
            const int y = pid * kBlock;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ptx::tma_load_2d(dst + i * kBoxBytes, tm_lat, full, x_lat + 64 * i, y);
            ptx::tma_load_2d(dst + 4 * kBoxBytes, tm_rope, full, x_rope, y);
            prefetch_next();
            ++gq;
            if (++k >= it.k_hi) {
                have = iter.next(it);
                k = have ? it.k_lo : 0;
            }
            idle = 0;
        } else if (!have && gv == gq) {
            break;
        } else if ((++idle & 1023u) == 0) {
            if (*sh.abort_flag()) return;
            const uint64_t now = ptx::globaltimer();
            if (idle == 1024u) t0 = now;
            else if (now - t0 > kWaitLimitNs) {
                *sh.abort_flag() = 1;
                record_error(kErrTimeout, 0x10u);
                return;
            }
        }
    }
    // drain: wait until the loads still in flight have landed
    for (uint32_t i = 0; i < (uint32_t)kQkStages && i < gq; ++i) {
        const uint32_t g = gq - 1 - i;
        wait_bar<false>(sh, sh.bar(kBarQkFull + g % kQkStages), (g / kQkStages) & 1u, 0x11u);
    }
    for (uint32_t i = 0; i < (uint32_t)kVStages && i < gv; ++i) {
        const uint32_t g = gv - 1 - i;
        wait_bar<false>(sh, sh.bar(kBarVFull + g % kVStages), (g / kVStages) & 1u, 0x12u);
    }
}

// ------------------------------------------------------------------ MMA issuer (warp 9)
// QK of page G may start once its page has landed and the senders have read S of G - 1.
__device__ __forceinline__ bool qk_ready(const Shared& sh, uint32_t G) {
    return ptx::mbar_test_wait(sh.bar(kBarQkFull + G % kQkStages), (G / kQkStages) & 1u) &&
           (G == 0 || ptx::mbar_test_wait(sh.bar(kBarSFree), (G - 1) & 1u));
}

// PV of page G may start once its P is in TMEM and its latent dims are in the V ring.
__device__ __forceinline__ bool pv_ready(const Shared& sh, uint32_t G) {
    return ptx::mbar_test_wait(sh.bar(kBarPReady + (G & 1u)), (G >> 1) & 1u) &&
           ptx::mbar_test_wait(sh.bar(kBarVFull + G % kVStages), (G / kVStages) & 1u);
}

// S = Q K^T for global page index G (QK stage G % kQkStages); qk_ready(G) has been seen.
__device__ __forceinline__ void issue_qk(const Shared& sh, uint32_t tmem, uint32_t G) {
    const uint32_t s = G % kQkStages;
    ptx::tc_fence_after();
    const uint32_t d = tmem + kColS;
    const uint32_t st = sh.qk_stage(s);
    const uint32_t qrope = sh.base_u32 + kOffQrope;
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
        const uint64_t bdesc =
            ptx::smem_desc(st + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024, 2);
        ptx::mma_ts(d, tmem + kColQ + 8 * kk, bdesc, kIdescQK, kk > 0);
    }
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        const uint64_t adesc = ptx::smem_desc(qrope + 32 * kk, 16, 512, 4);
        const uint64_t bdesc = ptx::smem_desc(st + 4 * kBoxBytes + 32 * kk, 16, 512, 4);
        ptx::mma_ss(d, adesc, bdesc, kIdescQK, 1);
    }
    ptx::mma_commit(sh.bar(kBarSFull + (G & 1u)));
    ptx::mma_commit(sh.bar(kBarQkEmpty + s));
}

// O += P V for global page index G; `first` starts a new accumulation; pv_ready(G) has
// been observed.
__device__ __forceinline__ void issue_pv(const Shared& sh, uint32_t tmem, uint32_t G, bool first) {
    const uint32_t pb = G & 1u;
    ptx::tc_fence_after();
    const uint32_t st = sh.v_stage(G % kVStages);
    const uint32_t a = tmem + kColP + 32 * pb;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bdesc = ptx::smem_desc(st + kk * 2048, kBoxBytes, 1024, 2);
        ptx::mma_ts(tmem + kColO, a + 8 * kk, bdesc, kIdescPV, (!first || kk > 0) ? 1u : 0u);
    }
    ptx::mma_commit(sh.bar(kBarPvDone + pb));
    ptx::mma_commit(sh.bar(kBarVEmpty + G % kVStages));
}

__device__ __forceinline__ void run_mma(const DecodeParams& p, const Shared& sh, uint32_t tmem) {
    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t G = 0;        // global page index (stage ring and S/P buffers)
    uint32_t items = 0;
    while (iter.next(it)) {
        if (!wait_bar<false>(sh, sh.bar(kBarQReady), items & 1u, 0x20u)) return;
        ptx::tc_fence_after();
        const uint32_t n = (uint32_t)(it.k_hi - it.k_lo);
        // Issue whichever MMA is ready, PV first (it frees a stage and a P buffer); QK of
        // later pages goes ahead as soon as their pages have landed and S is free, so
        // neither waits behind the other. Waits are bounded as everywhere else.
        uint32_t qk = 0, pv = 0;
        uint64_t t0 = 0;
        uint32_t idle = 0;
        while (pv < n) {
            if (pv < qk && pv_ready(sh, G + pv)) {
                issue_pv(sh, tmem, G + pv, pv == 0);
                ++pv;
                idle = 0;
            } else if (qk < n && qk_ready(sh, G + qk)) {
                issue_qk(sh, tmem, G + qk);
                ++qk;
                idle = 0;
            } else if ((++idle & 1023u) == 0) {
                if (*sh.abort_flag()) return;
                const uint64_t now = ptx::globaltimer();
                if (idle == 1024u) t0 = now;
                else if (now - t0 > kWaitLimitNs) {
                    *sh.abort_flag() = 1;
                    record_error(kErrTimeout, 0x24u);
                    return;
                }
            }
        }
        G += n;
        ++items;
    }
}

// ------------------------------------------------------------------ senders (warps 4-7)
// For every page G: read this CTA's partial scores (one TMEM lane per thread), release S,
// quantise the row to 16-bit fixed point, write it into staging buffer G % 2 and (one
// thread) bulk-copy the buffer into the peer's exchange buffer G % 2, completing tx bytes
// on the peer's kBarXFull. Before reusing buffer G % 2, wait until the peer's softmax has
// read what was sent into it two pages earlier (kBarXFree, arrived by the peer's
// senders; the copy out of our staging buffer is then complete too), and forward this
// CTA's own "buffer read" signal to the peer in the same way.
__device__ __forceinline__ void run_sender(const DecodeParams& p, const Shared& sh, uint32_t tmem,
                                           uint32_t crank, int quarter, int lane) {
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t peer = crank ^ 1u;
    const uint32_t x_peer = ptx::mapa(sh.base_u32 + kOffX, peer);
    const uint32_t xfull_peer = ptx::mapa(sh.bar(kBarXFull), peer);
    const bool leader = row == 0;

    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t G = 0;
    while (iter.next(it)) {
        const int r = it.t * kTileRows + row;
        const int n_vis = r < p.rows ? visible_tokens(it.L, p.s_q, r / p.h_q, p.causal) : 0;
        const uint32_t n = (uint32_t)(it.k_hi - it.k_lo);
        for (uint32_t j = 0; j < n; ++j, ++G) {
            const uint32_t xb = G & 1u;
            if (!warp_wait_bar<false>(sh, sh.bar(kBarSFull + (G & 1u)), (G >> 1) & 1u, 0x40u)) return;
            ptx::tc_fence_after();
            uint32_t sv[64];
            ptx::tmem_ld64(tmem + lane_base + kColS, sv);
            ptx::tc_fence_before();
            ptx::mbar_arrive(sh.bar(kBarSFree));

            // per-row scale over the visible tokens of this page
            const int lim = n_vis - (it.k_lo + (int)j) * kBlock;
            float mx = 0.f;
            if (__all_sync(0xffffffffu, lim >= 64)) {
#pragma unroll
                for (int q = 0; q < 64; ++q) mx = fmaxf(mx, fabsf(__uint_as_float(sv[q])));
            } else {
#pragma unroll
                for (int q = 0; q < 64; ++q)
                    if (q < lim) mx = fmaxf(mx, fabsf(__uint_as_float(sv[q])));
            }
            const float inv = mx > 0.f ? kQuantMax / mx : 0.f;
            // round to the nearest integer on the FMA pipe: adding 1.5 * 2^23 + 32768 leaves
            // 32768 + round(x) (in [1, 65535] for |x| <= 32767) in the low 16 mantissa bits;
            // masked columns may carry any code, the softmax never uses them
            uint32_t pk[32];
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const uint32_t ua = __float_as_uint(fmaf(__uint_as_float(sv[2 * q]), inv, 12615680.f));
                const uint32_t ub = __float_as_uint(fmaf(__uint_as_float(sv[2 * q + 1]), inv, 12615680.f));
                pk[q] = __byte_perm(ua, ub, 0x5410);
            }

            // staging buffer xb held page G-2: our softmax must have read it (kBarXRead) and
            // the peer must have read the copy of it (kBarXFree), which also means the copy
            // out of it is complete
            if (G >= 2) {
                if (!warp_wait_bar<false>(sh, sh.bar(kBarXRead + xb), ((G - 2) >> 1) & 1u, 0x44u))
                    return;
                if (!warp_wait_bar<true>(sh, sh.bar(kBarXFree + xb), ((G - 2) >> 1) & 1u, 0x42u))
                    return;
            }
            const uint32_t stg = sh.base_u32 + kOffXStage + xb * kXBytes;
            const uint32_t rowp = stg + (uint32_t)row * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t phys = (uint32_t)(c ^ (row & 7));
                ptx::st_shared_v4(rowp + phys * 16, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                                  pk[4 * c + 3]);
            }
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(stg + kXDataBytes + 4 * row),
                         "f"(mx * (1.f / kQuantMax)) : "memory");
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(sh.bar(kBarStage + xb));
            if (leader) {
                if (!wait_bar<false>(sh, sh.bar(kBarStage + xb), (G >> 1) & 1u, 0x43u)) return;
                ptx::bulk_copy_to_peer(x_peer + xb * kXBytes, stg, kXBytes, xfull_peer + 8 * xb);
            }
        }
    }
}

// ------------------------------------------------------------------ relay (warp 10, one thread)
// For every page G: once this CTA's softmax has read exchange buffer G % 2, tell the
// peer's senders (kBarXFree of the peer) that they may write page G + 2 into it.
__device__ __forceinline__ void run_relay(const DecodeParams& p, const Shared& sh, uint32_t crank) {
    const uint32_t xfree_peer = ptx::mapa(sh.bar(kBarXFree), crank ^ 1u);
    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t G = 0;
    while (iter.next(it)) {
        const uint32_t n = (uint32_t)(it.k_hi - it.k_lo);
        for (uint32_t j = 0; j < n; ++j, ++G) {
            const uint32_t xb = G & 1u;
            if (!wait_bar<false>(sh, sh.bar(kBarXRead + xb), (G >> 1) & 1u, 0x41u)) return;
            ptx::mbar_arrive_remote(xfree_peer + 8 * xb);
        }
    }
}

// ------------------------------------------------------------------ softmax (warps 0-7)
__device__ __forceinline__ float f32(uint32_t x) { return __uint_as_float(x); }

struct SoftmaxCtx {
    uint32_t tmem, lane_base, crank;
    int row, wg;            // query row (TMEM lane) and warpgroup (0 or 1)
};

// Row state of one group: the reference max its sum is relative to, and the sum of
// 2^(s - m_used) over the tokens of its pages.
struct RowState {
    float m_used;
    float l_sum;
};

// Brings the group's sum to reference m (m >= m_used, or m_used = -inf with l = 0).
__device__ __forceinline__ void rebase(RowState& st, float m) {
    if (m != st.m_used) {
        st.l_sum = st.m_used == -INFINITY ? 0.f : st.l_sum * ptx::ex2_ftz(st.m_used - m);
        st.m_used = m;
    }
}

// Softmax of page G (j-th page of the item) for this group's row.
__device__ __forceinline__ bool softmax_page(const DecodeParams& p, const Shared& sh,
                                             const SoftmaxCtx& c, const Item& it, int n_vis,
                                             uint32_t j, uint32_t G, RowState& st) {
    const uint32_t xb = G & 1u;                         // == c.wg
    const int row = c.row;
    // own quantised scores of page G (staging buffer xb) and the peer's (exchange buffer xb)
    if (!warp_wait_bar<false>(sh, sh.bar(kBarStage + xb), (G >> 1) & 1u, 0x30u)) return false;
    if (!warp_wait_bar<true>(sh, sh.bar(kBarXFull + xb), (G >> 1) & 1u, 0x32u)) return false;
    // s = (part0 + part1) * scale_log2 - base, part_c the partial of CTA rank c, each
    // (v - 32768) * row_scale with v its biased 16-bit code. 2^23 + v is formed by OR-ing
    // v into the bits of 2^23, so (2^23 + v) * a + k with a = row_scale * scale_log2 and
    // k = -(2^23 + 32768) * a gives a partial; rounding k costs at most half a
    // quantisation step. Both CTAs evaluate the same expression in rank order, so they
    // obtain bit-identical scores.
    float s[64];
    const uint32_t xbuf = sh.base_u32 + kOffX + xb * kXBytes;        // the peer's partial
    const uint32_t sbuf = sh.base_u32 + kOffXStage + xb * kXBytes;   // this CTA's partial
    const uint32_t buf0 = c.crank == 0 ? sbuf : xbuf;
    const uint32_t buf1 = c.crank == 0 ? xbuf : sbuf;
    float sc0, sc1;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc0) : "r"(buf0 + kXDataBytes + 4 * row) : "memory");
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(sc1) : "r"(buf1 + kXDataBytes + 4 * row) : "memory");
    const float L = p.scale_log2;
    const float a0 = sc0 * L;
    const float a1 = sc1 * L;
    const float base = st.m_used == -INFINITY ? 0.f : st.m_used;
    const float k0 = fmaf(-8421376.f, a1, fmaf(-8421376.f, a0, -base));
    // raw codes first (the buffers are released before the arithmetic): w[0..31] from
    // rank 0's partial, w[32..63] from rank 1's
    uint32_t w[64];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
        const uint32_t off = (uint32_t)row * 128 + (((uint32_t)cc ^ (uint32_t)(row & 7)) * 16);
        ptx::ld_shared_v4(buf0 + off, w[4 * cc], w[4 * cc + 1], w[4 * cc + 2], w[4 * cc + 3]);
        ptx::ld_shared_v4(buf1 + off, w[32 + 4 * cc], w[33 + 4 * cc], w[34 + 4 * cc],
                          w[35 + 4 * cc]);
    }
    // buffers xb are consumed: tell the relay and the senders, and re-arm the exchange
    // buffer for page G + 2 (the peer cannot send that page before every thread of this
    // group has passed the wait above)
    ptx::mbar_arrive(sh.bar(kBarXRead + xb));
    if (row == 0) ptx::mbar_arrive_expect_tx(sh.bar(kBarXFull + xb), kXPayload);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        s[2 * e] = fmaf(__uint_as_float(0x4B000000u | (w[32 + e] & 0xffffu)), a1,
                        fmaf(__uint_as_float(0x4B000000u | (w[e] & 0xffffu)), a0, k0));
        s[2 * e + 1] = fmaf(__uint_as_float(0x4B000000u | (w[32 + e] >> 16)), a1,
                            fmaf(__uint_as_float(0x4B000000u | (w[e] >> 16)), a0, k0));
    }

    // mask tokens past this row's visible end
    const int t0 = (it.k_lo + (int)j) * kBlock;
    const int lim = n_vis - t0;                         // valid columns: [0, lim)
    if (!__all_sync(0xffffffffu, lim >= 64)) {
#pragma unroll
        for (int q = 0; q < 64; ++q) s[q] = q < lim ? s[q] : -INFINITY;
    }
    float mx;
    {
        float m8[8];
#pragma unroll
        for (int a8 = 0; a8 < 8; ++a8)
            m8[a8] = fmaxf(fmaxf(fmaxf(s[a8], s[a8 + 8]), fmaxf(s[a8 + 16], s[a8 + 24])),
                           fmaxf(fmaxf(s[a8 + 32], s[a8 + 40]), fmaxf(s[a8 + 48], s[a8 + 56])));
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    }
    const float mx_abs = mx + base;

    // reference max after page G-1 (from the other group), then this page's decision:
    // raise the reference only when a score exceeds it by more than the threshold
    float* mref_sh = reinterpret_cast<float*>(sh.base + kOffMref);
    float m_prev = -INFINITY;
    if (j > 0) {
        if (!warp_wait_bar<false>(sh, sh.bar(kBarMref + (xb ^ 1u)), ((G - 1) >> 1) & 1u, 0x36u))
            return false;
        m_prev = *reinterpret_cast<volatile float*>(&mref_sh[row]);
    }
    const bool raise = m_prev == -INFINITY ? mx_abs > -INFINITY : mx_abs > m_prev + kRescaleLog2;
    const float m_new = raise ? mx_abs : m_prev;
    // publish before any wait below, so the next page's group never waits on this one
    mref_sh[row] = m_new;
    ptx::mbar_arrive(sh.bar(kBarMref + xb));

    // re-express this page's scores and the group's sum relative to m_new
    if (m_new != base && m_new != -INFINITY) {
        const float d = m_new - base;
#pragma unroll
        for (int q = 0; q < 64; ++q) s[q] -= d;
    }
    rebase(st, m_new);
    // O must follow the raise: after PV of page G-1 (which used m_prev), scale it by
    // 2^(m_prev - m_new); only rows that were already accumulating need it
    const bool need_o = raise && j > 0 && m_prev != -INFINITY;
    if (__any_sync(0xffffffffu, need_o)) {
        if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (xb ^ 1u)), ((G - 1) >> 1) & 1u, 0x33u))
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
    }
    uint32_t pk[32];
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const float p0 = ptx::ex2_ftz(s[2 * q]);
        const float p1 = ptx::ex2_ftz(s[2 * q + 1]);
        rs0 += p0;
        rs1 += p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[q] = *reinterpret_cast<uint32_t*>(&h2);
    }
    st.l_sum += rs0 + rs1;
    // P buffer G % 2 is free once PV of page G - 2 has completed; that PV also saw the
    // V load of page G - 2 land in the stage this page's V uses, so the wait on that
    // stage below cannot match an earlier phase
    if (G >= 2 && !warp_wait_bar<false>(sh, sh.bar(kBarPvDone + xb), ((G - 2) >> 1) & 1u, 0x35u))
        return false;
    ptx::tc_fence_after();
    ptx::tmem_st32(c.tmem + c.lane_base + kColP + 32 * xb, pk);

    // zero V rows past the sequence end on its last, partial page (they may hold stale
    // or NaN data, and P = 0 would not cancel NaN in the MMA)
    const int tail = it.L - t0;
    if (tail < kBlock) {
        // the V load of this page must have landed before its tail is overwritten
        if (!warp_wait_bar<false>(sh, sh.bar(kBarVFull + G % kVStages), (G / kVStages) & 1u, 0x39u))
            return false;
        const uint32_t stg = sh.v_stage(G % kVStages);
        const int nbad = kBlock - tail;
        for (int q = row; q < nbad * 32; q += 128) {
            const int rr = tail + (q >> 5);
            const int box = (q >> 3) & 3;
            const int ch = q & 7;
            ptx::st_shared_v4(stg + box * kBoxBytes + rr * 128 + ch * 16, 0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();       // zeroed V rows visible to the MMA
    }
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(sh.bar(kBarPReady + xb));
    return true;
}

__device__ __forceinline__ void run_softmax(const DecodeParams& p, const Shared& sh, uint32_t tmem,
                                            uint32_t crank, int warp, int lane) {
    SoftmaxCtx c;
    const int quarter = warp & 3;
    c.tmem = tmem;
    c.crank = crank;
    c.lane_base = (uint32_t)(quarter * 32) << 16;
    c.row = quarter * 32 + lane;                           // TMEM lane == query row in tile
    c.wg = warp >> 2;
    const int row = c.row;
    float* mref_sh = reinterpret_cast<float*>(sh.base + kOffMref);

    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t G = 0;
    uint32_t items = 0;
    while (iter.next(it)) {
        const int r = it.t * kTileRows + row;               // query row within the sequence
        const bool row_valid = r < p.rows;
        const int qi = row_valid ? r / p.h_q : 0;
        const int n_vis = row_valid ? visible_tokens(it.L, p.s_q, qi, p.causal) : 0;

        // ---- load the group's part of the row of q: a quarter of the latent dims into
        // TMEM and half of the rope dims into shared memory
        {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((size_t)it.b * p.rows + (row_valid ? r : 0)) * kHeadDim);
            const uint32_t qaddr = tmem + c.lane_base + kColQ + 64 * c.wg;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                uint32_t v[32];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    uint4 x = row_valid ? __ldg(src + crank * 32 + c.wg * 16 + cc * 8 + jj)
                                        : make_uint4(0, 0, 0, 0);
                    v[4 * jj + 0] = x.x; v[4 * jj + 1] = x.y; v[4 * jj + 2] = x.z; v[4 * jj + 3] = x.w;
                }
                ptx::tmem_st32(qaddr + 32 * cc, v);
            }
            // rope: 32 dims = 4 chunks of 16 B per row; K-major SW64 layout, 8-row atoms
            const uint32_t qr = sh.base_u32 + kOffQrope + (uint32_t)(row >> 3) * 512 +
                                (uint32_t)(row & 7) * 64;
#pragma unroll
            for (int cc = 2 * c.wg; cc < 2 * c.wg + 2; ++cc) {
                uint4 x = row_valid ? __ldg(src + 64 + crank * 4 + cc) : make_uint4(0, 0, 0, 0);
                const uint32_t phys = (uint32_t)(cc ^ ((row & 7) >> 1));
                ptx::st_shared_v4(qr + phys * 16, x.x, x.y, x.z, x.w);
            }
            ptx::fence_proxy_async_smem();
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(sh.bar(kBarQReady));
        }

        RowState st{-INFINITY, 0.f};
        const uint32_t n = (uint32_t)(it.k_hi - it.k_lo);
        const uint32_t G0 = G;
        bool ok = true;
        for (uint32_t j = (G0 & 1u) == (uint32_t)c.wg ? 0u : 1u; j < n; j += 2) {
            if (!softmax_page(p, sh, c, it, n_vis, j, G0 + j, st)) { ok = false; break; }
        }
        if (!ok) return;
        G = G0 + n;

        // ---- epilogue: O / l for this group's 128 of the CTA's 256 output columns
        const uint32_t Gl = G - 1;
        if (!warp_wait_bar<false>(sh, sh.bar(kBarMref + (Gl & 1u)), (Gl >> 1) & 1u, 0x38u)) return;
        const float m_fin = *reinterpret_cast<volatile float*>(&mref_sh[row]);
        rebase(st, m_fin);
        float* lsum = reinterpret_cast<float*>(sh.base + kOffLsum);
        lsum[c.wg * 128 + row] = st.l_sum;
        ptx::mbar_arrive(sh.bar(kBarLsum));
        if (!warp_wait_bar<false>(sh, sh.bar(kBarLsum), items & 1u, 0x37u)) return;
        if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (Gl & 1u)), (Gl >> 1) & 1u, 0x34u)) return;
        ptx::tc_fence_after();
        const float l_tot = *reinterpret_cast<volatile float*>(&lsum[row]) +
                            *reinterpret_cast<volatile float*>(&lsum[128 + row]);
        const bool empty = !(l_tot > 0.f);
        const float inv = empty ? 0.f : 1.f / l_tot;
        const float lse2 = empty ? -INFINITY : m_fin + __log2f(l_tot);
        const bool final_out = it.n_chunks == 1;
        const bool have_ws = it.part < p.max_chunks;
        if (!final_out && !have_ws && row == 0 && c.wg == 0)
            record_error(kErrWorkspace, (uint32_t)it.v & 0xffffffu);
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            ptx::tmem_ld32(tmem + c.lane_base + kColO + 128 * c.wg + 32 * cc, ov);
            if (!row_valid) continue;
            const int col = (int)crank * kLatentHalf + 128 * c.wg + 32 * cc;
            if (final_out) {
                uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)it.b * p.rows + r) * kHeadDimV + col);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    uint32_t w[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(f32(ov[8 * e + 2 * h]) * inv,
                                                                  f32(ov[8 * e + 2 * h + 1]) * inv);
                        w[h] = *reinterpret_cast<uint32_t*>(&b2);
                    }
                    dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            } else if (have_ws) {
                float4* dst = reinterpret_cast<float4*>(
                    p.ws_o + ((size_t)it.part * kTileRows + row) * kHeadDimV + col);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(f32(ov[4 * e]) * inv, f32(ov[4 * e + 1]) * inv,
                                         f32(ov[4 * e + 2]) * inv, f32(ov[4 * e + 3]) * inv);
            }
        }
        if (row_valid && crank == 0 && c.wg == 0) {
            if (final_out) {
                const int h = r % p.h_q;
                p.lse[((size_t)it.b * p.h_q + h) * p.s_q + qi] = empty ? -INFINITY : lse2 * kLn2;
            } else if (have_ws) {
                p.ws_lse[(size_t)it.part * kTileRows + row] = lse2;
            }
        }
        ptx::tc_fence_before();
        ++items;
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_lat,
              const __grid_constant__ CUtensorMap tm_rope) {
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
        for (int s = 0; s < kQkStages; ++s) {
            ptx::mbar_init(sh.bar(kBarQkFull + s), 1);
            ptx::mbar_init(sh.bar(kBarQkEmpty + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            ptx::mbar_init(sh.bar(kBarVFull + s), 1);
            ptx::mbar_init(sh.bar(kBarVEmpty + s), 1);
        }
        ptx::mbar_init(sh.bar(kBarSFull + 0), 1);
        ptx::mbar_init(sh.bar(kBarSFull + 1), 1);
        ptx::mbar_init(sh.bar(kBarSFree), 128);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(sh.bar(kBarPReady + i), 128);
            ptx::mbar_init(sh.bar(kBarPvDone + i), 1);
            ptx::mbar_init(sh.bar(kBarXFull + i), 1);
            ptx::mbar_init(sh.bar(kBarXRead + i), 128);
            ptx::mbar_init(sh.bar(kBarXFree + i), 1);
            ptx::mbar_init(sh.bar(kBarStage + i), 128);
            ptx::mbar_init(sh.bar(kBarMref + i), 128);
        }
        ptx::mbar_init(sh.bar(kBarQReady), kSoftmaxThreads);
        ptx::mbar_init(sh.bar(kBarLsum), kSoftmaxThreads);
        *sh.abort_flag() = 0;
        ptx::fence_mbarrier_init_cluster();
        // arm both exchange buffers for the first two pages
        ptx::mbar_arrive_expect_tx(sh.bar(kBarXFull + 0), kXPayload);
        ptx::mbar_arrive_expect_tx(sh.bar(kBarXFull + 1), kXPayload);
        ptx::prefetch_tensormap(&tm_lat);
        ptx::prefetch_tensormap(&tm_rope);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(ptx::smem_u32(sh.tmem_slot()), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();            // peer barriers initialised before any remote access
    ptx::tc_fence_after();
    const uint32_t tmem = *sh.tmem_slot();

    if (warp < kWarpSender0) {
        ptx::setmaxnreg_inc<kRegsSoftmax>();
        run_softmax(p, sh, tmem, crank, warp, lane);
    } else if (warp < kWarpControl0) {
        ptx::setmaxnreg_dec<kRegsSender>();
        run_sender(p, sh, tmem, crank, warp - kWarpSender0, lane);
    } else {
        ptx::setmaxnreg_dec<kRegsControl>();
        if (warp == kWarpProducer && lane == 0) run_producer(p, sh, &tm_lat, &tm_rope, crank);
        if (warp == kWarpMma && lane == 0) run_mma(p, sh, tmem);
        if (warp == kWarpRelay && lane == 0) run_relay(p, sh, crank);
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();            // no remote store or arrive may target an exited CTA
    if (warp == kWarpMma) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace sm100
}  // namespace mla

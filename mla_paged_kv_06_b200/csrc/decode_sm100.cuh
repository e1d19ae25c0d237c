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
// instead of 32 KB, error at most 2^-16 of that magnitude. Each CTA adds the peer's
// dequantised partial to its own exact fp32 partial.
//
// Per CTA (384 threads, three warpgroups whose registers are rebalanced at start):
//   warps 0-3 softmax / correction / epilogue, one thread per query row (TMEM lane).
//             While page j is combined and exponentiated, page j+1's scores are already
//             read (and, by the senders, on their way to the peer).
//   warps 4-7 senders: read each page's partial scores from TMEM, quantise them into a
//             local staging buffer and bulk-copy it into the peer's exchange buffer;
//             relay to the peer when this CTA's softmax has finished reading an exchange
//             buffer. Remote traffic never stalls the softmax warps.
//   warp 8    TMA producer: page ids from the block table, 4 SW128 latent boxes + 1 SW64
//             rope box per page into a 4-stage ring.
//   warp 9    TMEM owner and MMA issuer (one thread): S = Q K^T (M=128, N=64, K=288;
//             the latent part reads Q from TMEM, the rope part from shared memory) and
//             O += P V (M=128, N=256, K=64; P from TMEM, V = the page's latent boxes
//             read MN-major). QK runs two pages ahead of PV.
//   warps 10-11 idle (they complete the third warpgroup).
// TMEM columns: O [0,256) fp32, Q latent [256,384) bf16x2, S [384,448) fp32,
// P0 [448,480) and P1 [480,512) bf16x2. S is released as soon as both groups read it.
// Scores stay in the log2 domain (scale * log2 e folded in). The running max is only
// raised when a new score exceeds it by more than kRescaleLog2, so O is rescaled rarely.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kThreads = 384;
constexpr int kWarpSender0 = 4;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
// Registers per thread after rebalancing: 128 * (240 + 104 + 56) = 51200, within the
// 384 * 168 = 64512 the CTA is launched with (ptxas reports 168 for this kernel).
constexpr uint32_t kRegsSoftmax = 240;
constexpr uint32_t kRegsSender = 104;
constexpr uint32_t kRegsControl = 56;
constexpr int kStages = 4;
constexpr int kLatentHalf = 256;                     // latent dims per CTA
constexpr int kRopeHalf = 32;                        // rope dims per CTA
constexpr uint32_t kBoxBytes = 64 * 64 * 2;          // one SW128 box: 64 tokens x 64 dims
constexpr uint32_t kRopeBoxBytes = 64 * 32 * 2;      // one SW64 box: 64 tokens x 32 dims
constexpr uint32_t kStageBytes = 4 * kBoxBytes + kRopeBoxBytes;   // 36 KB
constexpr uint32_t kQropeBytes = 128 * kRopeHalf * 2;             // 8 KB
// Exchange buffer (and its staging twin): 128 rows x 64 biased 16-bit scores (128 B per
// row, 16-byte chunks XOR-swizzled by row % 8 so row-per-thread access is conflict-free)
// followed by the 128 per-row fp32 scales.
constexpr uint32_t kXDataBytes = 128 * 128;
constexpr uint32_t kXBytes = kXDataBytes + 128 * 4;  // 16896
constexpr uint32_t kXPayload = kXBytes;              // bytes the peer sends per page
constexpr float kQuantMax = 32767.f;

constexpr uint32_t kOffStage = 0;
constexpr uint32_t kOffQrope = kStages * kStageBytes;
constexpr uint32_t kOffX = kOffQrope + kQropeBytes;          // [2] receive buffers
constexpr uint32_t kOffXStage = kOffX + 2 * kXBytes;         // [2] staging buffers
constexpr uint32_t kOffBar = kOffXStage + 2 * kXBytes;
// barriers (8 B each)
enum : uint32_t {
    kBarFull = 0,                     // [kStages] TMA -> MMA
    kBarEmpty = kBarFull + kStages,   // [kStages] MMA (PV done) -> TMA
    kBarSFull = kBarEmpty + kStages,  // QK done -> softmax and senders
    kBarSFree = kBarSFull + 1,        // softmax and senders read S -> MMA
    kBarPReady = kBarSFree + 1,       // [2] P written -> MMA
    kBarPvDone = kBarPReady + 2,      // [2] PV done -> softmax
    kBarXFull = kBarPvDone + 2,       // [2] peer scores landed (tx count)
    kBarXRead = kBarXFull + 2,        // [2] softmax read exchange buffer -> senders
    kBarXFree = kBarXRead + 2,        // [2] peer's softmax read what we sent
    kBarQReady = kBarXFree + 2,       // query tile in TMEM / smem
    kBarStage = kBarQReady + 1,       // [2] staging buffer written -> sending thread
    kNumBars = kBarStage + 2
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
    __device__ uint32_t stage(uint32_t s) const { return base_u32 + kOffStage + s * kStageBytes; }
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

// ------------------------------------------------------------------ producer (warp 8)
__device__ __forceinline__ void run_producer(const DecodeParams& p, const Shared& sh,
                                             const CUtensorMap* tm_lat, const CUtensorMap* tm_rope,
                                             uint32_t crank) {
    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t g = 0;                                   // pages issued so far
    const int x_lat = (int)crank * kLatentHalf;
    const int x_rope = 512 + (int)crank * kRopeHalf;
    while (iter.next(it)) {
        const int32_t* bt = p.block_table + (size_t)it.b * p.max_blocks;
        for (int k = it.k_lo; k < it.k_hi; ++k, ++g) {
            const uint32_t s = g % kStages;
            if (g >= (uint32_t)kStages &&
                !wait_bar<false>(sh, sh.bar(kBarEmpty + s), ((g / kStages) - 1) & 1u, 0x10u))
                return;
            int pid = bt[k];
            if (pid < 0 || pid >= p.num_blocks) {
                record_error(kErrBadInput, 0x800000u | ((uint32_t)it.b & 0x7fffffu));
                pid = 0;
            }
            const uint32_t full = sh.bar(kBarFull + s);
            ptx::mbar_arrive_expect_tx(full, kStageBytes);
            const uint32_t dst = sh.stage(s);
            const int y = pid * kBlock;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ptx::tma_load_2d(dst + i * kBoxBytes, tm_lat, full, x_lat + 64 * i, y);
            ptx::tma_load_2d(dst + 4 * kBoxBytes, tm_rope, full, x_rope, y);
        }
    }
    // drain: wait until the loads still in flight have landed
    for (uint32_t i = 0; i < (uint32_t)kStages && i < g; ++i) {
        const uint32_t gg = g - 1 - i;
        wait_bar<false>(sh, sh.bar(kBarFull + gg % kStages), (gg / kStages) & 1u, 0x11u);
    }
}

// ------------------------------------------------------------------ MMA issuer (warp 9)
// S = Q K^T for global page index G (stage G % kStages).
__device__ __forceinline__ bool issue_qk(const Shared& sh, uint32_t tmem, uint32_t G) {
    const uint32_t s = G % kStages;
    if (!wait_bar<false>(sh, sh.bar(kBarFull + s), (G / kStages) & 1u, 0x21u)) return false;
    if (G >= 1 && !wait_bar<false>(sh, sh.bar(kBarSFree), (G - 1) & 1u, 0x22u)) return false;
    ptx::tc_fence_after();
    const uint32_t d = tmem + kColS;
    const uint32_t st = sh.stage(s);
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
    ptx::mma_commit(sh.bar(kBarSFull));
    return true;
}

// O += P V for global page index G; `first` starts a new accumulation.
__device__ __forceinline__ bool issue_pv(const Shared& sh, uint32_t tmem, uint32_t G, bool first) {
    const uint32_t pb = G & 1u;
    if (!wait_bar<false>(sh, sh.bar(kBarPReady + pb), (G >> 1) & 1u, 0x23u)) return false;
    ptx::tc_fence_after();
    const uint32_t st = sh.stage(G % kStages);
    const uint32_t a = tmem + kColP + 32 * pb;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bdesc = ptx::smem_desc(st + kk * 2048, kBoxBytes, 1024, 2);
        ptx::mma_ts(tmem + kColO, a + 8 * kk, bdesc, kIdescPV, (!first || kk > 0) ? 1u : 0u);
    }
    ptx::mma_commit(sh.bar(kBarPvDone + pb));
    ptx::mma_commit(sh.bar(kBarEmpty + G % kStages));
    return true;
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
        // QK runs two pages ahead of PV: S of page j+1 is read (freeing the single S
        // buffer) before P of page j exists, so QK(j+2) can be issued ahead of PV(j).
        if (!issue_qk(sh, tmem, G)) return;
        if (n > 1 && !issue_qk(sh, tmem, G + 1)) return;
        for (uint32_t j = 0; j < n; ++j) {
            if (j + 2 < n && !issue_qk(sh, tmem, G + j + 2)) return;
            if (!issue_pv(sh, tmem, G + j, j == 0)) return;
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
    const uint32_t xfree_peer = ptx::mapa(sh.bar(kBarXFree), peer);
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
            if (!warp_wait_bar<false>(sh, sh.bar(kBarSFull), G & 1u, 0x40u)) return;
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

            if (G >= 2) {
                // relay: our softmax has read buffer xb (page G-2); the peer may refill it
                if (leader) {
                    if (!wait_bar<false>(sh, sh.bar(kBarXRead + xb), ((G - 2) >> 1) & 1u, 0x41u))
                        return;
                    ptx::mbar_arrive_remote(xfree_peer + 8 * xb);
                }
                // and the peer must have read our previous send into its buffer xb
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

// ------------------------------------------------------------------ softmax (warps 0-3)
__device__ __forceinline__ float f32(uint32_t x) { return __uint_as_float(x); }

struct RowState {
    float m_ref;     // reference max (log2 domain); -inf until a visible token is seen
    float l_sum;     // sum of 2^(s - m_ref) over the tokens seen
};

// Waits for S of page G, reads it into `sv` and releases the S buffer.
__device__ __forceinline__ bool load_scores(const Shared& sh, uint32_t tmem, uint32_t lane_base,
                                            uint32_t G, uint32_t* sv) {
    if (!warp_wait_bar<false>(sh, sh.bar(kBarSFull), G & 1u, 0x30u)) return false;
    ptx::tc_fence_after();
    ptx::tmem_ld64(tmem + lane_base + kColS, sv);
    ptx::tc_fence_before();
    ptx::mbar_arrive(sh.bar(kBarSFree));
    return true;
}

// Softmax of page G of the current item: combines the own partial scores `sv` with the
// peer's, updates the row state, writes P into TMEM and hands it to the MMA warp.
__device__ __forceinline__ bool softmax_page(const DecodeParams& p, const Shared& sh, uint32_t tmem,
                                             uint32_t lane_base, int row,
                                             const Item& it, int n_vis, uint32_t j, uint32_t G,
                                             const uint32_t* sv, RowState& st) {
    const uint32_t xb = G & 1u;
    if (!warp_wait_bar<true>(sh, sh.bar(kBarXFull + xb), (G >> 1) & 1u, 0x32u)) return false;
    // s = (own + peer) * scale_log2, peer = (v - 32768) * peer_scale where v is the biased
    // 16-bit code: 2^23 + v is formed by OR-ing v into the bits of 2^23, and subtracting
    // 2^23 + 32768 from it is exact, so dequantising rounds only once
    float s[64];
    const uint32_t buf = sh.base_u32 + kOffX + xb * kXBytes;
    float pscale;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(pscale) : "r"(buf + kXDataBytes + 4 * row) : "memory");
    const float a = pscale * p.scale_log2;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
        ptx::ld_shared_v4(buf + (uint32_t)row * 128 + (uint32_t)((c ^ (row & 7)) * 16), w[0], w[1],
                          w[2], w[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(0x4B000000u | (w[e] & 0xffffu));
            const float hi = __uint_as_float(0x4B000000u | (w[e] >> 16));
            const int q = 8 * c + 2 * e;
            s[q] = fmaf(lo - 8421376.f, a, f32(sv[q]) * p.scale_log2);
            s[q + 1] = fmaf(hi - 8421376.f, a, f32(sv[q + 1]) * p.scale_log2);
        }
    }
    // buffer xb is consumed: tell the senders, and re-arm it for page G + 2 (the peer
    // cannot send that page before every row here has passed the wait above)
    ptx::mbar_arrive(sh.bar(kBarXRead + xb));
    if (row == 0) ptx::mbar_arrive_expect_tx(sh.bar(kBarXFull + xb), kXPayload);

    // mask tokens past this row's visible end
    const int t0 = (it.k_lo + (int)j) * kBlock;
    const int lim = n_vis - t0;                        // valid columns: [0, lim)
    float mx = -INFINITY;
    if (!__all_sync(0xffffffffu, lim >= 64)) {
#pragma unroll
        for (int q = 0; q < 64; ++q) s[q] = q < lim ? s[q] : -INFINITY;
    }
    {
        float m8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            m8[a] = fmaxf(fmaxf(fmaxf(s[a], s[a + 8]), fmaxf(s[a + 16], s[a + 24])),
                          fmaxf(fmaxf(s[a + 32], s[a + 40]), fmaxf(s[a + 48], s[a + 56])));
        }
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
    }
    // raise the reference max only when it grows past the threshold
    const bool raise = mx > st.m_ref + kRescaleLog2 || (st.m_ref == -INFINITY && mx > -INFINITY);
    float factor = 1.f;
    if (raise) {
        factor = st.m_ref == -INFINITY ? 0.f : ptx::ex2_ftz(st.m_ref - mx);
        st.m_ref = mx;
        st.l_sum *= factor;
    }
    const bool need_o = raise && j > 0 && factor != 1.f;
    if (__any_sync(0xffffffffu, need_o)) {
        // O must hold the previous page's PV before it is rescaled
        if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (xb ^ 1u)), ((G - 1) >> 1) & 1u, 0x33u))
            return false;
        ptx::tc_fence_after();
        const float f = need_o ? factor : 1.f;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
            uint32_t ov[32];
            const uint32_t oaddr = tmem + lane_base + kColO + 32 * cc;
            ptx::tmem_ld32(oaddr, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(f32(ov[e]) * f);
            ptx::tmem_st32(oaddr, ov);
        }
    }
    const float mb = st.m_ref == -INFINITY ? 0.f : st.m_ref;
    uint32_t pk[32];
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
        const float p0 = ptx::ex2_ftz(s[2 * q] - mb);
        const float p1 = ptx::ex2_ftz(s[2 * q + 1] - mb);
        rs0 += p0;
        rs1 += p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[q] = *reinterpret_cast<uint32_t*>(&h2);
    }
    st.l_sum += rs0 + rs1;
    // P buffer G % 2 is free once PV of page G - 2 has completed
    if (G >= 2 && !warp_wait_bar<false>(sh, sh.bar(kBarPvDone + xb), ((G - 2) >> 1) & 1u, 0x35u))
        return false;
    ptx::tc_fence_after();
    ptx::tmem_st32(tmem + lane_base + kColP + 32 * xb, pk);

    // zero V rows past the sequence end on its last, partial page (they may hold stale
    // or NaN data, and P = 0 would not cancel NaN in the MMA)
    const int tail = it.L - t0;
    if (tail < kBlock) {
        const uint32_t stg = sh.stage(G % kStages);
        const int nbad = kBlock - tail;
        for (int q = row; q < nbad * 32; q += 128) {
            const int rr = tail + (q >> 5);
            const int box = (q >> 3) & 3;
            const int ch = q & 7;
            ptx::st_shared_v4(stg + box * kBoxBytes + rr * 128 + ch * 16, 0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
    }
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    ptx::mbar_arrive(sh.bar(kBarPReady + xb));
    return true;
}

__device__ __forceinline__ void run_softmax(const DecodeParams& p, const Shared& sh, uint32_t tmem,
                                            uint32_t crank, int quarter, int lane) {
    const int row = quarter * 32 + lane;                   // TMEM lane == query row in tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;

    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t G = 0;
    while (iter.next(it)) {
        const int r = it.t * kTileRows + row;               // query row within the sequence
        const bool row_valid = r < p.rows;
        const int qi = row_valid ? r / p.h_q : 0;
        const int n_vis = row_valid ? visible_tokens(it.L, p.s_q, qi, p.causal) : 0;

        // ---- load this row of q: latent half into TMEM, rope half into shared memory
        {
            const uint4* src = reinterpret_cast<const uint4*>(
                p.q + ((size_t)it.b * p.rows + (row_valid ? r : 0)) * kHeadDim);
            const uint32_t qaddr = tmem + lane_base + kColQ;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 x = row_valid ? __ldg(src + crank * 32 + cc * 8 + j) : make_uint4(0, 0, 0, 0);
                    v[4 * j + 0] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                ptx::tmem_st32(qaddr + 32 * cc, v);
            }
            // rope half: 32 dims = 4 chunks of 16 B; K-major SW64 layout, 8-row atoms
            const uint32_t qr = sh.base_u32 + kOffQrope + (uint32_t)(row >> 3) * 512 +
                                (uint32_t)(row & 7) * 64;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
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
        // page j is finished while page j+1's scores have already been read
        uint32_t sv[64], sn[64];
        if (!load_scores(sh, tmem, lane_base, G, sv)) return;
        bool ok = true;
        for (uint32_t j = 0; j < n; ++j, ++G) {
            if (j + 1 < n && !load_scores(sh, tmem, lane_base, G + 1, sn)) { ok = false; break; }
            if (!softmax_page(p, sh, tmem, lane_base, row, it, n_vis, j, G, sv, st)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int q = 0; q < 64; ++q) sv[q] = sn[q];
        }
        if (!ok) return;

        // ---- epilogue: O / l for this row's 256 output columns
        const uint32_t Gl = G - 1;
        if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (Gl & 1u)), (Gl >> 1) & 1u, 0x34u)) return;
        ptx::tc_fence_after();
        const bool empty = !(st.l_sum > 0.f);
        const float inv = empty ? 0.f : 1.f / st.l_sum;
        const float lse2 = empty ? -INFINITY : st.m_ref + __log2f(st.l_sum);
        const bool final_out = it.n_chunks == 1;
        const bool have_ws = it.part < p.max_chunks;
        if (!final_out && !have_ws && row == 0)
            record_error(kErrWorkspace, (uint32_t)it.v & 0xffffffu);
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
            uint32_t ov[32];
            ptx::tmem_ld32(tmem + lane_base + kColO + 32 * cc, ov);
            if (!row_valid) continue;
            const int col = (int)crank * kLatentHalf + 32 * cc;
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
        if (row_valid && crank == 0) {
            if (final_out) {
                const int h = r % p.h_q;
                p.lse[((size_t)it.b * p.h_q + h) * p.s_q + qi] = empty ? -INFINITY : lse2 * kLn2;
            } else if (have_ws) {
                p.ws_lse[(size_t)it.part * kTileRows + row] = lse2;
            }
        }
        ptx::tc_fence_before();
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
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(sh.bar(kBarFull + s), 1);
            ptx::mbar_init(sh.bar(kBarEmpty + s), 1);
        }
        ptx::mbar_init(sh.bar(kBarSFull), 1);
        ptx::mbar_init(sh.bar(kBarSFree), 256);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(sh.bar(kBarPReady + i), 128);
            ptx::mbar_init(sh.bar(kBarPvDone + i), 1);
            ptx::mbar_init(sh.bar(kBarXFull + i), 1);
            ptx::mbar_init(sh.bar(kBarXRead + i), 128);
            ptx::mbar_init(sh.bar(kBarXFree + i), 1);
            ptx::mbar_init(sh.bar(kBarStage + i), 128);
        }
        ptx::mbar_init(sh.bar(kBarQReady), 128);
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
    } else if (warp < kWarpProducer) {
        ptx::setmaxnreg_dec<kRegsSender>();
        run_sender(p, sh, tmem, crank, warp - kWarpSender0, lane);
    } else {
        ptx::setmaxnreg_dec<kRegsControl>();
        if (warp == kWarpProducer && lane == 0) run_producer(p, sh, &tm_lat, &tm_rope, crank);
        if (warp == kWarpMma && lane == 0) run_mma(p, sh, tmem);
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

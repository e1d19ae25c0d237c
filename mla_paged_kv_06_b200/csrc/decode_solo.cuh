// sm_100a decode kernel for sequences of at most 64 query rows (s_q * h_q <= 64): one CTA
// per SM, no cluster, nothing exchanged between SMs.
//
// The 2-CTA kernel (decode_pair.cuh) works on 128-row tiles split over two SMs. With 64
// rows or fewer, one of its CTAs computes padding only, yet the pair still runs its full
// per-page chain, including the post-QK reload of the other page. Here one CTA owns a
// work unit alone and reads every page exactly once:
//   QK:  S = Q K^T for one 64-token page: M = 128 (the R <= 64 real query rows; the rows
//        beyond are never read), N = 64 tokens, K = 576. Q's first kQtChunks x 64 dims
//        come from TMEM, the rest from shared memory. S lands one query row per TMEM
//        lane, so one thread owns a whole row: the row max needs no exchange.
//   PV:  transposed, O^T = V^T P^T: M = 128 latent dims (four blocks for 512), N = kN
//        (the rows padded to 16, 32 or 64), K = 16 tokens per instruction. V^T is the page
//        tile itself, read MN-major from its stage (no copy); P is the B operand, K-major,
//        one 128-byte row of 64 bf16 probabilities per query row. O^T needs 4 kN TMEM
//        columns, which leaves room for Q in TMEM and two score buffers.
// Per CTA (192 threads):
//   warps 0-3  the row group. Thread r (TMEM lane r) does the softmax of query row r < R.
//              All 128 threads (TMEM lane = latent dim of an O^T block) do the rare O
//              rescale, the epilogue, the move of each item's q rows into TMEM and shared
//              memory, and the zeroing of V rows past a sequence's end.
//   warp 4     TMA producer: a ring of kStages 72 KB stages. An item takes one slot for its
//              q rows (box {64, kN rows, 9 chunks}) and then one slot per page (box {64,
//              64 rows, 9 chunks}: 9 swizzled 8 KB tiles in one instruction), with the next
//              page prefetched into L2.
//   warp 5     TMEM owner and MMA issuer. Issue order QK(j), QK(j+1), PV(j), QK(j+2), ...
//              keeps the tensor pipe busy while the row group computes P(j).
// Scores stay in the log2 domain. A row's reference max is raised only when a score
// exceeds it by more than kRescaleLog2; O^T columns are then rescaled in TMEM by all four
// warps (a column spans all 128 lanes).
#pragma once

#include "common.cuh"
#include "items.cuh"
#include "ptx.cuh"

namespace mla {
namespace solo {

constexpr int kThreads = 192;
constexpr int kRowThreads = 128;
constexpr int kWarpProducer = 4;
constexpr int kWarpMma = 5;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kBoxBytes = 64 * 128;             // 64 rows x 64 bf16, 128-byte swizzle
constexpr uint32_t kStageBytes = 9 * kBoxBytes;      // one page: 64 tokens x 576 dims
constexpr uint32_t kSmemLimit = 232448;              // sm_100 per-block opt-in maximum
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 3;

// Layout for kN padded query rows. TMEM columns: O^T [0, 4 kN), two score buffers of 64,
// then Q's first dims as bf16 pairs. Shared memory (from a 1 KB aligned base): Q's
// remaining chunks, one P buffer, the stages, then barriers and per-row arrays.
template <int N_>
struct Cfg {
    static constexpr int kN = N_;
    static constexpr uint32_t kColO = 0;
    static constexpr uint32_t kColS = 4 * kN;
    static constexpr uint32_t kColQ = kColS + 128;
    static constexpr int kQtChunksFit = (int)((kTmemCols - kColQ) * 2 / 64);
    static constexpr int kQtChunks = kQtChunksFit >= 9 ? 9 : kQtChunksFit;   // Q chunks in TMEM
    static constexpr int kQsChunks = 9 - kQtChunks;                          // in shared memory
    static constexpr uint32_t kTileBytes = kN * 128;          // kN rows x 64 dims, one chunk
    static constexpr uint32_t kOffQs = 0;
    static constexpr uint32_t kOffP = kOffQs + kQsChunks * kTileBytes;
    static constexpr uint32_t kOffStage = kOffP + kTileBytes;
    static constexpr uint32_t kMiscBytes = 1024;
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
    kBarQkDone = kBarFree + kMaxStages,  // [2] QK of a step done (score buffer step % 2)
    kBarPvDone = kBarQkDone + 2,         // PV of a step done (one phase per step)
    kBarPReady = kBarPvDone + 1,         // the row group wrote P (4 warp arrivals)
    kBarQReady = kBarPReady + 1,         // the item's q rows are in TMEM and shared memory
    kBarOFree = kBarQReady + 1,          // the previous item's O^T was read out
    kBarDecide = kBarOFree + 1,          // the step's rescale decision is posted
    kBarEpi = kBarDecide + 1,            // the item's row sums are posted
    kBarDrain = kBarEpi + 1,             // the MMA issuer's last commit
    kBarStall = kBarDrain + 1,           // never completes (the timeout test hook waits on it)
    kNumBars = kBarStall + 1
};
// misc area: barriers [0, 128), tmem base at 128, abort flag at 132, rescale tags at 136
// and 140, rescale factors [2][64] at 256, inverse row sums [64] at 768
static_assert(kNumBars * 8 <= 128, "barrier area");

template <int kN>
struct Smem {
    using C = Cfg<kN>;
    uint8_t* base;
    uint32_t base_u32;
    uint64_t wait_limit;                 // ns a wait may last before the kernel gives up
    __device__ uint32_t bar(uint32_t i) const { return base_u32 + C::kOffMisc + 8 * i; }
    __device__ uint32_t stage(uint32_t s) const { return base_u32 + C::kOffStage + s * kStageBytes; }
    __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(base + C::kOffMisc + 128); }
    __device__ volatile int* abort_flag() const {
        return reinterpret_cast<volatile int*>(base + C::kOffMisc + 132);
    }
    __device__ volatile int* resc_tag(uint32_t par) const {
        return reinterpret_cast<volatile int*>(base + C::kOffMisc + 136 + 4 * par);
    }
    __device__ float* facs(uint32_t par) const {
        return reinterpret_cast<float*>(base + C::kOffMisc + 256 + 256 * par);
    }
    __device__ float* inv_l() const { return reinterpret_cast<float*>(base + C::kOffMisc + 768); }
};

// Bounded wait: false if the phase does not complete within the limit or another role of
// the CTA already gave up (then the caller stops).
template <int kN>
__device__ __forceinline__ bool wait_bar(const Smem<kN>& sh, uint32_t bar, uint32_t parity,
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
template <int kN>
__device__ __forceinline__ bool warp_wait_bar(const Smem<kN>& sh, uint32_t bar, uint32_t parity,
                                              uint32_t where) {
    const bool ok = wait_bar(sh, bar, parity, where);
    return __all_sync(0xffffffffu, ok);
}

// Wait for copies or MMAs this CTA issued before it may finish: bounded by the time limit
// only (the abort flag does not cut it short, so nothing lands after the CTA has exited
// unless the limit itself runs out).
template <int kN>
__device__ __forceinline__ void drain_wait(const Smem<kN>& sh, uint32_t bar, uint32_t parity,
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
template <int kN>
__device__ __forceinline__ void run_producer(const DecodeParams& p, const Smem<kN>& sh,
                                             const CUtensorMap* tm_page, const CUtensorMap* tm_q) {
    using C = Cfg<kN>;
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
        for (int k = it.k_lo; k < it.k_hi; ++k) {
            if (!(ok = acquire(g))) break;
            const uint32_t s = g % C::kStages;
            const int row = page_row(p, it.b, k, it.k_hi);
            ptx::mbar_arrive_expect_tx(sh.bar(kBarFull + s), kStageBytes);
            ptx::tma_load_3d(sh.stage(s), tm_page, sh.bar(kBarFull + s), 0, row, 0);
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

// ------------------------------------------------------------------ MMA issuer (warp 5)
// QK of the page in stage s into score buffer sb, K-steps [k0, k1) of the 36 (16 dims
// each); the half that ends at 36 commits the buffer's QkDone.
template <int kN, int k0, int k1>
__device__ __forceinline__ void issue_qk(const Smem<kN>& sh, uint32_t tmem, uint32_t s, uint32_t sb) {
    using C = Cfg<kN>;
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
                sh.base_u32 + C::kOffQs + ((k >> 2) - C::kQtChunks) * C::kTileBytes + (k & 3) * 32,
                16, 1024, 2);
            ptx::mma_ss(d, adesc, bdesc, kIdesc, k > 0 ? 1u : 0u);
        }
    }
    if constexpr (k1 == 36) ptx::mma_commit(sh.bar(kBarQkDone + sb));
}

// O^T += V^T P^T for the page in stage s; `first` starts the item's accumulation.
template <int kN>
__device__ __forceinline__ void issue_pv(const Smem<kN>& sh, uint32_t tmem, uint32_t s, bool first) {
    using C = Cfg<kN>;
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

template <int kN>
__device__ __forceinline__ void run_mma(const DecodeParams& p, const Smem<kN>& sh, uint32_t tmem) {
    using C = Cfg<kN>;
    ItemIter iter(p, (int)blockIdx.x, (int)gridDim.x);
    Item it;
    uint32_t g = 0, gs = 0, items = 0;
    bool ok = true;
    while (ok && iter.next(it)) {
        // the item's q rows were moved out of their slot: free it
        if (!wait_bar(sh, sh.bar(kBarQReady), items & 1u, 0x48u)) break;
        ptx::tc_fence_after();
        ptx::mbar_arrive(sh.bar(kBarFree + g % C::kStages));
        ++g;
        const uint32_t n = (uint32_t)it.pages();
        // Tensor-pipe order QK(0) QK(1) PV(0) QK(2) PV(1) ...: the next page's QK keeps the
        // pipe busy while the row group turns S(j) into P(j).
        uint32_t qk = 0, pv = 0;
        bool o_free = items == 0;          // the previous item's O^T must be read out first
        uint64_t t0 = 0;
        uint32_t idle = 0;
        while (pv < n) {
            if (!o_free && ptx::mbar_test_wait(sh.bar(kBarOFree), (items - 1) & 1u)) {
                ptx::tc_fence_after();
                o_free = true;
            }
            const uint32_t gq = g + qk;
            if (pv < qk && (pv > 0 || o_free) &&
                ptx::mbar_test_wait(sh.bar(kBarPReady), (gs + pv) & 1u)) {
                issue_pv(sh, tmem, (g + pv) % C::kStages, pv == 0);
                ++pv;
                idle = 0;
            } else if (qk < n && qk < pv + 2 &&
                       ptx::mbar_test_wait(sh.bar(kBarFull + gq % C::kStages), (gq / C::kStages) & 1u)) {
                issue_qk<kN, 0, 36>(sh, tmem, gq % C::kStages, (gs + qk) & 1u);
                ++qk;
                idle = 0;
            } else if ((++idle & 1023u) == 0) {
                if (*sh.abort_flag()) { ok = false; break; }
                const uint64_t now = ptx::globaltimer();
                if (idle == 1024u) t0 = now;
                else if (now - t0 > sh.wait_limit) {
                    *sh.abort_flag() = 1;
                    record_error(kErrTimeout, 0x49u);
                    ok = false;
                    break;
                }
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

// ------------------------------------------------------------------ row group (warps 0-3)
__device__ __forceinline__ float f32(uint32_t x) { return __uint_as_float(x); }

template <int kCols>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* v) {
    if constexpr (kCols == 16) ptx::tmem_ld16(taddr, v);
    else if constexpr (kCols == 32) ptx::tmem_ld32(taddr, v);
    else ptx::tmem_ld64(taddr, v);
}

struct RowCtx {
    uint32_t tmem, lane_base;
    int tid, warp, lane;
    bool row_warp;        // the warp holds query rows (warp-uniform)
};

// The item's q rows, landed in stage s as kN rows x 9 chunks: dims [0, 64 kQtChunks) go
// to TMEM (lane r = row r, bf16 pairs), the rest to their tiles in shared memory (a byte
// copy: both sides are 1 KB aligned, so the 128-byte swizzle carries over).
template <int kN>
__device__ __forceinline__ void move_q(const Smem<kN>& sh, const RowCtx& c, uint32_t s) {
    using C = Cfg<kN>;
    const uint32_t st = sh.stage(s);
    if (c.warp * 32 < kN) {
#pragma unroll 1
        for (int ch = 0; ch < C::kQtChunks; ++ch) {
            uint32_t v[32];
            const uint32_t rowa = st + ch * C::kTileBytes + (uint32_t)c.tid * 128;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const uint4 x = ptx::ld_shared_v4(rowa + (((uint32_t)jj ^ (uint32_t)(c.tid & 7)) * 16));
                v[4 * jj] = x.x; v[4 * jj + 1] = x.y; v[4 * jj + 2] = x.z; v[4 * jj + 3] = x.w;
            }
            ptx::tmem_st32(c.tmem + c.lane_base + C::kColQ + 32 * ch, v);
        }
        ptx::tmem_wait_st();
    }
    if constexpr (C::kQsChunks > 0) {
        constexpr uint32_t bytes = C::kQsChunks * C::kTileBytes;
        const uint32_t src = st + C::kQtChunks * C::kTileBytes;
        const uint32_t dst = sh.base_u32 + C::kOffQs;
#pragma unroll 4
        for (uint32_t o = (uint32_t)c.tid * 16; o < bytes; o += kRowThreads * 16)
            { const uint4 x = ptx::ld_shared_v4(src + o); ptx::st_shared_v4(dst + o, x.x, x.y, x.z, x.w); }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
}

// One page step S (the item's j-th page) for this thread.
template <int kN>
__device__ __forceinline__ bool row_step(const DecodeParams& p, const Smem<kN>& sh, const RowCtx& c,
                                         const Item& it, int n_vis, uint32_t j, uint32_t S,
                                         uint32_t s, float& m_ref, float& l_sum, float& l_rnd) {
    using C = Cfg<kN>;
    const uint32_t sb = S & 1u, par = S & 1u;
    if (!warp_wait_bar(sh, sh.bar(kBarQkDone + sb), (S >> 1) & 1u, 0x51u)) return false;
    ptx::tc_fence_after();
    const int page = it.k_lo + (int)j;
    float x[64];
    float fac = 1.f;
    bool need = false;
    if (c.row_warp) {
        uint32_t sv[64];
        ptx::tmem_ld64(c.tmem + c.lane_base + C::kColS + 64 * sb, sv);
        const int lim = n_vis - page * kBlock;                  // valid tokens [0, lim)
        const float base = m_ref == -INFINITY ? 0.f : m_ref;
        const float L2 = p.scale_log2;
        if (__all_sync(0xffffffffu, lim >= 64)) {
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] = fmaf(f32(sv[q]), L2, -base);
        } else {
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] = q < lim ? fmaf(f32(sv[q]), L2, -base) : -INFINITY;
        }
        float m8[8];
#pragma unroll
        for (int a = 0; a < 8; ++a)
            m8[a] = fmaxf(fmaxf(fmaxf(x[a], x[a + 8]), fmaxf(x[a + 16], x[a + 24])),
                          fmaxf(fmaxf(x[a + 32], x[a + 40]), fmaxf(x[a + 48], x[a + 56])));
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        const float mx_abs = mx + base;
        const bool raise = m_ref == -INFINITY ? mx_abs > -INFINITY : mx_abs > m_ref + kRescaleLog2;
        const float m_new = raise ? mx_abs : m_ref;
        if (m_new != base && m_new != -INFINITY) {
            const float d = m_new - base;
#pragma unroll
            for (int q = 0; q < 64; ++q) x[q] -= d;
        }
        need = raise && m_ref != -INFINITY;        // O^T holds earlier pages at m_ref
        if (need) {
            fac = ptx::ex2_ftz(m_ref - m_new);
            l_sum *= fac;
            l_rnd *= fac;
        }
        m_ref = m_new;
        if (c.tid < 64) sh.facs(par)[c.tid] = fac;
        if (need) *sh.resc_tag(par) = (int)(S + 1);
    }
    warp_arrive(sh.bar(kBarDecide));
    if (!warp_wait_bar(sh, sh.bar(kBarDecide), par, 0x52u)) return false;
    const bool resc = *sh.resc_tag(par) == (int)(S + 1);
    if (resc || S > 0) {
        // PV of step S-1 must be done: before O^T is rescaled, and before P is rewritten
        if (!warp_wait_bar(sh, sh.bar(kBarPvDone), (S - 1) & 1u, 0x53u)) return false;
        ptx::tc_fence_after();
    }
    if (resc) {
        // scale the O^T columns of rows that raised their reference (factor 1 elsewhere)
        const float* f = sh.facs(par);
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
#pragma unroll 1
            for (int cc = 0; cc < kN; cc += 16) {
                uint32_t v[16];
                const uint32_t a = c.tmem + c.lane_base + C::kColO + kN * i + cc;
                ptx::tmem_ld16(a, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(f32(v[e]) * f[cc + e]);
                ptx::tmem_st16(a, v);
            }
        }
        ptx::tmem_wait_st();
    }
    if (c.row_warp) {
        uint32_t pk[32];
        float rs0 = 0.f, rs1 = 0.f, rr0 = 0.f, rr1 = 0.f;
#pragma unroll
        for (int q = 0; q < 32; ++q) {
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
        if (c.tid < kN) {
            // row of P: 64 tokens = 8 chunks of 16 B, K-major, 128-byte swizzle
            const uint32_t prow = sh.base_u32 + C::kOffP + (uint32_t)c.tid * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                ptx::st_shared_v4(prow + (((uint32_t)cc ^ (uint32_t)(c.tid & 7)) * 16), pk[4 * cc],
                                  pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        }
    }
    // V rows past the sequence end (they may hold stale or NaN data, and P = 0 would not
    // cancel NaN): zero them in the stage. QK of this step, their only other reader, is done.
    const int tail = it.L - page * kBlock;
    if (tail < kBlock) {
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

// Epilogue of an item: the row threads post 1/l and write the lse; then every thread (TMEM
// lane = latent dim) writes its dim of each real row, normalised, as bf16 `out`, fp32
// `out_f32` or the fp32 split partial.
template <int kN>
__device__ __forceinline__ bool epilogue(const DecodeParams& p, const Smem<kN>& sh, const RowCtx& c,
                                         const Item& it, float m_ref, float l_sum, float l_rnd,
                                         uint32_t last_step, uint32_t epi_index) {
    using C = Cfg<kN>;
    const bool final_out = it.n_chunks == 1;
    const bool have_ws = it.part < p.max_chunks;
    if (c.row_warp && c.tid < 64) {
        const bool empty = !(l_sum > 0.f);
        sh.inv_l()[c.tid] = empty ? 0.f : 1.f / l_rnd;
        if (c.tid < p.rows) {
            const float lse2 = empty ? -INFINITY : m_ref + __log2f(l_sum);
            if (final_out) {
                const int qi = c.tid / p.h_q, h = c.tid % p.h_q;
                p.lse[((size_t)it.b * p.h_q + h) * p.s_q + qi] = empty ? -INFINITY : lse2 * kLn2;
            } else if (have_ws) {
                p.ws_lse[(size_t)it.part * kTileRows + c.tid] = lse2;
            }
        }
    }
    if (!final_out && !have_ws && c.tid == 0) record_error(kErrWorkspace, (uint32_t)it.v & 0xffffffu);
    warp_arrive(sh.bar(kBarEpi));
    if (!warp_wait_bar(sh, sh.bar(kBarEpi), epi_index & 1u, 0x54u)) return false;
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

template <int kN>
__device__ __forceinline__ void run_rows(const DecodeParams& p, const Smem<kN>& sh, uint32_t tmem) {
    using C = Cfg<kN>;
    RowCtx c;
    c.tmem = tmem;
    c.tid = (int)threadIdx.x;
    c.warp = c.tid >> 5;
    c.lane = c.tid & 31;
    c.lane_base = (uint32_t)(c.warp * 32) << 16;
    c.row_warp = c.warp * 32 < p.rows;
    ItemIter iter(p, (int)blockIdx.x, (int)gridDim.x);
    Item it, prev;
    uint32_t g = 0, gs = 0, items = 0;
    float m_ref = -INFINITY, l_sum = 0.f, l_rnd = 0.f;
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
        const bool row_valid = c.tid < p.rows;
        const int qi = row_valid ? c.tid / p.h_q : 0;
        const int n_vis = row_valid ? visible_tokens(it.L, p.s_q, qi, p.causal) : 0;
        m_ref = -INFINITY;
        l_sum = 0.f;
        l_rnd = 0.f;
        const uint32_t n = (uint32_t)it.pages();
        for (uint32_t j = 0; j < n; ++j) {
            if (!row_step(p, sh, c, it, n_vis, j, gs + j, (g + j) % C::kStages, m_ref, l_sum, l_rnd))
                return;
        }
        g += n;
        gs += n;
        prev = it;
        prev_m = m_ref;
        prev_l = l_sum;
        prev_r = l_rnd;
        have_prev = true;
        ++items;
    }
    if (have_prev) epilogue(p, sh, c, prev, prev_m, prev_l, prev_r, gs - 1, items - 1);
}

template <int kN>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_page,
              const __grid_constant__ CUtensorMap tm_q) {
    using C = Cfg<kN>;
    extern __shared__ uint8_t smem_raw[];
    Smem<kN> sh;
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
        ptx::mbar_init(sh.bar(kBarQReady), 4);
        ptx::mbar_init(sh.bar(kBarOFree), 4);
        ptx::mbar_init(sh.bar(kBarDecide), 4);
        ptx::mbar_init(sh.bar(kBarEpi), 4);
        ptx::mbar_init(sh.bar(kBarDrain), 1);
        ptx::mbar_init(sh.bar(kBarStall), 1);
        *sh.abort_flag() = 0;
        *sh.resc_tag(0) = 0;
        *sh.resc_tag(1) = 0;
        ptx::fence_mbarrier_init_cluster();
        ptx::prefetch_tensormap(&tm_page);
        ptx::prefetch_tensormap(&tm_q);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(ptx::smem_u32(sh.tmem_slot()), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *sh.tmem_slot();

    if (warp < 4) {
        run_rows<kN>(p, sh, tmem);
    } else if (warp == kWarpProducer) {
        if (lane == 0) run_producer<kN>(p, sh, &tm_page, &tm_q);
    } else if (warp == kWarpMma) {
        if (lane == 0) run_mma<kN>(p, sh, tmem);
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

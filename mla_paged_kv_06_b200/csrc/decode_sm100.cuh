// sm_100a split kernel for paged MLA decode.
//
// One 2-CTA cluster owns one work unit (a contiguous run of pages, see sched.cuh) and
// processes 128 query rows against one 64-token page at a time. Per SM the 128 x 512
// fp32 output accumulator alone would fill all of TMEM (128 lanes x 512 columns), and
// the 128 x 576 bf16 query tile plus a 64 x 576 page would crowd shared memory. So
// the pair splits the 576 dims: CTA c holds latent dims [256c, 256c+256) and rope dims
// [512+32c, 512+32c+32) of q and of every page, computes the partial scores over its
// 288 dims, and owns output columns [256c, 256c+256). The two partial score tiles are
// exchanged over distributed shared memory and summed identically in both CTAs, so
// both run the same online softmax and no FLOP or HBM byte is duplicated.
//
// Per CTA (192 threads):
//   warp 0   TMA producer: page ids from the block table, 4 SW128 latent boxes + 1 SW64
//            rope box per page into a 4-stage ring.
//   warp 1   TMEM owner and MMA issuer (one thread): S = Q K^T (M=128, N=64, K=288;
//            the latent part reads Q from TMEM, the rope part from shared memory) and
//            O += P V (M=128, N=256, K=64; P from TMEM, V = the page's latent boxes
//            read MN-major), completion tracked with tcgen05.commit.
//   warps 2-5 softmax / correction / epilogue, one thread per query row.
// TMEM columns: O [0,256) fp32, Q latent [256,384) bf16x2, S0 [384,448), S1 [448,512);
// P (bf16x2) overwrites the first 32 columns of the S buffer it came from.
// Scores stay in the log2 domain (scale * log2 e folded in). The running max is only
// raised when a new score exceeds it by more than kRescaleLog2, so O is rescaled rarely.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace sm100 {

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kLatentHalf = 256;                     // latent dims per CTA
constexpr int kRopeHalf = 32;                        // rope dims per CTA
constexpr uint32_t kBoxBytes = 64 * 64 * 2;          // one SW128 box: 64 tokens x 64 dims
constexpr uint32_t kRopeBoxBytes = 64 * 32 * 2;      // one SW64 box: 64 tokens x 32 dims
constexpr uint32_t kStageBytes = 4 * kBoxBytes + kRopeBoxBytes;   // 36 KB
constexpr uint32_t kQropeBytes = 128 * kRopeHalf * 2;             // 8 KB
constexpr uint32_t kXRowStride = 272;                // 64 fp32 + 16 B pad: no bank conflicts
constexpr uint32_t kXBytes = 128 * kXRowStride;

constexpr uint32_t kOffStage = 0;
constexpr uint32_t kOffQrope = kStages * kStageBytes;
constexpr uint32_t kOffX = kOffQrope + kQropeBytes;
constexpr uint32_t kOffBar = kOffX + 2 * kXBytes;
// barriers (8 B each)
enum : uint32_t {
    kBarFull = 0,                     // [kStages] TMA -> MMA
    kBarEmpty = kBarFull + kStages,   // [kStages] MMA (PV done) -> TMA
    kBarSFull = kBarEmpty + kStages,  // [2] QK done -> softmax
    kBarPReady = kBarSFull + 2,       // [2] P written -> MMA
    kBarPvDone = kBarPReady + 2,      // [2] PV done -> MMA / softmax
    kBarXFull = kBarPvDone + 2,       // [2] peer scores arrived
    kBarXFree = kBarXFull + 2,        // [2] peer finished reading what we sent
    kBarQReady = kBarXFree + 2,       // query tile in TMEM / smem
    kNumBars = kBarQReady + 1
};
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort flag
constexpr uint32_t kSmemBytes = kOffMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;      // room to align the base to 1 KB

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColQ = 256;
constexpr uint32_t kColS = 384;                          // + 64 * buffer

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

// Warp-uniform bounded wait for the softmax warps: every lane waits, and the warp
// proceeds only if all lanes saw the phase complete, so no lane can leave a loop whose
// body holds .sync.aligned tcgen05 instructions while its neighbours stay in it.
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

// ------------------------------------------------------------------ producer (warp 0)
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
            for (int i = 0; i < 4; ++i) ptx::tma_load_2d(dst + i * kBoxBytes, tm_lat, full, x_lat + 64 * i, y);
            ptx::tma_load_2d(dst + 4 * kBoxBytes, tm_rope, full, x_rope, y);
        }
    }
    // drain: wait until the loads still in flight have landed
    for (uint32_t i = 0; i < (uint32_t)kStages && i < g; ++i) {
        const uint32_t gg = g - 1 - i;
        wait_bar<false>(sh, sh.bar(kBarFull + gg % kStages), (gg / kStages) & 1u, 0x11u);
    }
}

// ------------------------------------------------------------------ MMA issuer (warp 1)
__device__ __forceinline__ void run_mma(const DecodeParams& p, const Shared& sh, uint32_t tmem) {
    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t g = 0;        // pages consumed (stage ring position)
    uint32_t G = 0;        // blocks processed (S/P buffer position), same as g here
    uint32_t items = 0;
    const uint32_t qrope = sh.base_u32 + kOffQrope;
    while (iter.next(it)) {
        if (!wait_bar<false>(sh, sh.bar(kBarQReady), items & 1u, 0x20u)) return;
        ptx::tc_fence_after();
        const int n = it.k_hi - it.k_lo;
        for (int j = 0; j <= n; ++j) {
            if (j < n) {
                // S[G % 2] = Q K^T over this CTA's 288 dims
                const uint32_t s = g % kStages;
                const uint32_t sb = G & 1u;
                if (!wait_bar<false>(sh, sh.bar(kBarFull + s), (g / kStages) & 1u, 0x21u)) return;
                if (G >= 2 && !wait_bar<false>(sh, sh.bar(kBarPvDone + sb), ((G - 2) >> 1) & 1u, 0x22u))
                    return;
                ptx::tc_fence_after();
                const uint32_t d = tmem + kColS + 64 * sb;
                const uint32_t st = sh.stage(s);
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    const uint64_t bdesc = ptx::smem_desc(st + (kk >> 2) * kBoxBytes + (kk & 3) * 32,
                                                          16, 1024, 2);
                    ptx::mma_ts(d, tmem + kColQ + 8 * kk, bdesc, kIdescQK, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint64_t adesc = ptx::smem_desc(qrope + 32 * kk, 16, 512, 4);
                    const uint64_t bdesc = ptx::smem_desc(st + 4 * kBoxBytes + 32 * kk, 16, 512, 4);
                    ptx::mma_ss(d, adesc, bdesc, kIdescQK, 1);
                }
                ptx::mma_commit(sh.bar(kBarSFull + sb));
            }
            if (j >= 1) {
                // O += P V for the previous page
                const uint32_t Gp = G - 1;
                const uint32_t gp = g - 1;
                const uint32_t sbp = Gp & 1u;
                if (!wait_bar<false>(sh, sh.bar(kBarPReady + sbp), (Gp >> 1) & 1u, 0x23u)) return;
                ptx::tc_fence_after();
                const uint32_t st = sh.stage(gp % kStages);
                const uint32_t a = tmem + kColS + 64 * sbp;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bdesc = ptx::smem_desc(st + kk * 2048, kBoxBytes, 1024, 2);
                    ptx::mma_ts(tmem + kColO, a + 8 * kk, bdesc, kIdescPV, (j > 1 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(sh.bar(kBarPvDone + sbp));
                ptx::mma_commit(sh.bar(kBarEmpty + gp % kStages));
            }
            if (j < n) { ++g; ++G; }
        }
        ++items;
    }
}

// ------------------------------------------------------------------ softmax (warps 2-5)
__device__ __forceinline__ float f32(uint32_t x) { return __uint_as_float(x); }

__device__ __forceinline__ void run_softmax(const DecodeParams& p, const Shared& sh, uint32_t tmem,
                                            uint32_t crank, int quarter, int lane) {
    const int row = quarter * 32 + lane;                   // TMEM lane == query row in tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t peer = crank ^ 1u;
    const uint32_t xrow_own = sh.base_u32 + kOffX + (uint32_t)row * kXRowStride;
    const uint32_t xrow_peer = ptx::mapa(xrow_own, peer);
    const uint32_t xfull_peer = ptx::mapa(sh.bar(kBarXFull), peer);
    const uint32_t xfree_peer = ptx::mapa(sh.bar(kBarXFree), peer);
    const int tid = quarter * 32 + lane;                   // 0..127 within the group

    ItemIter iter(p, (int)ptx::cluster_id_x(), (int)ptx::nclusters_x());
    Item it;
    uint32_t G = 0;
    uint32_t g = 0;
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
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 x = row_valid ? __ldg(src + crank * 32 + c * 8 + j) : make_uint4(0, 0, 0, 0);
                    v[4 * j + 0] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                }
                ptx::tmem_st32(qaddr + 32 * c, v);
            }
            // rope half: 32 dims = 4 chunks of 16 B; K-major SW64 layout, 8-row atoms
            const uint32_t qr = sh.base_u32 + kOffQrope + (uint32_t)(row >> 3) * 512 +
                                (uint32_t)(row & 7) * 64;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 x = row_valid ? __ldg(src + 64 + crank * 4 + c) : make_uint4(0, 0, 0, 0);
                const uint32_t phys = (uint32_t)(c ^ ((row & 7) >> 1));
                ptx::st_shared_v4(qr + phys * 16, x.x, x.y, x.z, x.w);
            }
            ptx::fence_proxy_async_smem();
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(sh.bar(kBarQReady));
        }

        float m_ref = -INFINITY;      // running reference max (log2 domain)
        float l_sum = 0.f;
        const int n = it.k_hi - it.k_lo;
        bool ok = true;
        for (int j = 0; j < n && ok; ++j, ++G, ++g) {
            const uint32_t sb = G & 1u;
            const int k = it.k_lo + j;
            if (!warp_wait_bar<false>(sh, sh.bar(kBarSFull + sb), (G >> 1) & 1u, 0x30u)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t sv[64];
            const uint32_t saddr = tmem + lane_base + kColS + 64 * sb;
            ptx::tmem_ld64(saddr, sv);

            // exchange partial scores with the peer CTA
            if (G >= 2 && !warp_wait_bar<true>(sh, sh.bar(kBarXFree + sb), ((G - 2) >> 1) & 1u, 0x31u)) {
                ok = false;
                break;
            }
            const uint32_t dst = xrow_peer + sb * kXBytes;
#pragma unroll
            for (int c = 0; c < 16; ++c)
                ptx::st_cluster_v4(dst + 16 * c, sv[4 * c], sv[4 * c + 1], sv[4 * c + 2], sv[4 * c + 3]);
            ptx::mbar_arrive_remote(xfull_peer + 8 * sb);
            if (!warp_wait_bar<true>(sh, sh.bar(kBarXFull + sb), (G >> 1) & 1u, 0x32u)) { ok = false; break; }
            float s[64];
            const uint32_t src = xrow_own + sb * kXBytes;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                uint32_t a, b2, c2, d;
                ptx::ld_shared_v4(src + 16 * c, a, b2, c2, d);
                s[4 * c + 0] = f32(sv[4 * c + 0]) + f32(a);
                s[4 * c + 1] = f32(sv[4 * c + 1]) + f32(b2);
                s[4 * c + 2] = f32(sv[4 * c + 2]) + f32(c2);
                s[4 * c + 3] = f32(sv[4 * c + 3]) + f32(d);
            }
            ptx::mbar_arrive_remote(xfree_peer + 8 * sb);

            // scale into the log2 domain and mask tokens past this row's visible end
            const int t0 = k * kBlock;
            const int lim = n_vis - t0;                      // valid columns: [0, lim)
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                s[c] = c < lim ? s[c] * p.scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[c]);
            }
            // raise the reference max only when it grows past the threshold
            const bool raise = mx > m_ref + kRescaleLog2 || (m_ref == -INFINITY && mx > -INFINITY);
            float factor = 1.f;
            if (raise) {
                factor = m_ref == -INFINITY ? 0.f : exp2f(m_ref - mx);
                m_ref = mx;
                l_sum *= factor;
            }
            const bool need_o = raise && j > 0 && factor != 1.f;
            if (__any_sync(0xffffffffu, need_o)) {
                // O must hold the previous page's PV before it is rescaled
                if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (sb ^ 1u)), ((G - 1) >> 1) & 1u, 0x33u)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const float f = need_o ? factor : 1.f;
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t ov[32];
                    const uint32_t oaddr = tmem + lane_base + kColO + 32 * c;
                    ptx::tmem_ld32(oaddr, ov);
#pragma unroll
                    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(f32(ov[e]) * f);
                    ptx::tmem_st32(oaddr, ov);
                }
            }
            const float mb = m_ref == -INFINITY ? 0.f : m_ref;
            uint32_t pk[32];
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float p0 = exp2f(s[2 * c] - mb);
                const float p1 = exp2f(s[2 * c + 1] - mb);
                rs += p0 + p1;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                pk[c] = *reinterpret_cast<uint32_t*>(&h2);
            }
            l_sum += rs;
            ptx::tmem_st32(saddr, pk);

            // zero V rows past the sequence end on its last, partial page (they may
            // hold stale or NaN data and P = 0 would not cancel NaN in the MMA)
            const int tail = it.L - t0;
            if (tail < kBlock) {
                const uint32_t st = sh.stage(g % kStages);
                const int nbad = kBlock - tail;
                for (int c = tid; c < nbad * 32; c += 128) {
                    const int rr = tail + (c >> 5);
                    const int box = (c >> 3) & 3;
                    const int ch = c & 7;
                    ptx::st_shared_v4(st + box * kBoxBytes + rr * 128 + ch * 16, 0, 0, 0, 0);
                }
                ptx::fence_proxy_async_smem();
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(sh.bar(kBarPReady + sb));
        }
        if (!ok) return;

        // ---- epilogue: O / l for this row's 256 output columns
        const uint32_t Gl = G - 1;
        if (!warp_wait_bar<false>(sh, sh.bar(kBarPvDone + (Gl & 1u)), (Gl >> 1) & 1u, 0x34u)) return;
        ptx::tc_fence_after();
        const bool empty = !(l_sum > 0.f);
        const float inv = empty ? 0.f : 1.f / l_sum;
        const float lse2 = empty ? -INFINITY : m_ref + __log2f(l_sum);
        const bool final_out = it.n_chunks == 1;
        const bool have_ws = it.part < p.max_chunks;
        if (!final_out && !have_ws && tid == 0) record_error(kErrWorkspace, (uint32_t)it.v & 0xffffffu);
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            uint32_t ov[32];
            ptx::tmem_ld32(tmem + lane_base + kColO + 32 * c, ov);
            if (!row_valid) continue;
            const int col = (int)crank * kLatentHalf + 32 * c;
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
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(sh.bar(kBarSFull + i), 1);
            ptx::mbar_init(sh.bar(kBarPReady + i), 128);
            ptx::mbar_init(sh.bar(kBarPvDone + i), 1);
            ptx::mbar_init(sh.bar(kBarXFull + i), 128);
            ptx::mbar_init(sh.bar(kBarXFree + i), 128);
        }
        ptx::mbar_init(sh.bar(kBarQReady), 128);
        *sh.abort_flag() = 0;
        ptx::fence_mbarrier_init_cluster();
        ptx::prefetch_tensormap(&tm_lat);
        ptx::prefetch_tensormap(&tm_rope);
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(sh.tmem_slot()), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();            // peer barriers initialised before any remote arrive
    ptx::tc_fence_after();
    const uint32_t tmem = *sh.tmem_slot();

    if (warp == 0) {
        if (lane == 0) run_producer(p, sh, &tm_lat, &tm_rope, crank);
    } else if (warp == 1) {
        if (lane == 0) run_mma(p, sh, tmem);
    } else {
        run_softmax(p, sh, tmem, crank, warp & 3, lane);
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();            // no remote store or arrive may target an exited CTA
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace sm100
}  // namespace mla

// LSE-weighted merge of split-KV partials. Chunk c of a work sequence holds the
// normalised output O_c and the log2-domain lse_c of its token subset; the softmax over
// the union weighs chunk c by 2^(lse_c - lse) with lse = log2 sum_c 2^lse_c. Work
// sequences that were not split are skipped (the split kernel already wrote them);
// work sequences that own no page at all (L = 0) get out = 0, lse = -inf here. With
// p.out_f32 set the merged rows are written there in fp32 instead of to p.out.
//
// Layout: one warp per row; lane i owns dims [4 i + 128 j, +4), j < 4: four float4 per
// chunk. The merge is latency-bound, so a warp keeps kChunkBatch chunks' loads in flight
// per round trip, and merges them online (lse and output rows arrive together, so a row
// of two chunks takes one round trip after reading its chunk count). Two chunks per round
// trip keep the kernel at 80 registers, three CTAs per SM; four per round trip needed
// 122 and were slower on the big grids (v3, spec). Where
// the grid is small, a row split over more than kSliceChunks chunks (a long sequence
// spread over many units) is cut into up to kCombineSlices slices, one CTA each (grid z):
// each merges its slice into one partial, written over the slot of the slice's first
// chunk, and the last of them to finish (a per-row-group counter in the workspace)
// merges the slices. Grid z CTAs of rows that need no slicing exit at once.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kCombineThreads = 256;
constexpr int kCombineRowsPerCta = kCombineThreads / 32;   // one warp per row
constexpr int kChunkBatch = 2;
constexpr int kCombineSlices = 4;     // most slices of a row (grid z, small grids only)
constexpr int kSliceChunks = 8;       // a row of more chunks than this is sliced
constexpr int kSliceGridMax = 1024;   // (work sequences x row groups) up to which to slice
static_assert(kCombineCounters == kTileRows / kCombineRowsPerCta, "one counter per row group");

__device__ __forceinline__ int combine_slices(int n_chunks, int max_slices) {
    if (n_chunks <= kSliceChunks) return 1;
    const int s = (n_chunks + kSliceChunks - 1) / kSliceChunks;
    return s < max_slices ? s : max_slices;
}

// This lane's 16 dims of the row (4 lane + 128 j), normalised: bf16 `out` or fp32 `out_f32`.
__device__ __forceinline__ void store_row(const DecodeParams& p, size_t row_index, int lane,
                                          const float4 (&v)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int dim = 4 * lane + 128 * j;
        if (p.out_f32) {
            *reinterpret_cast<float4*>(p.out_f32 + row_index * kHeadDimV + dim) = v[j];
            continue;
        }
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v[j].x, v[j].y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(v[j].z, v[j].w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(p.out + row_index * kHeadDimV + dim) = pk;
    }
}

// Merges `count` partials of row r_local, slot(i) giving the i-th one's slot, online:
// each round trip loads kChunkBatch partials' lse and output rows together, raises the
// running maximum, rescales the running sum and accumulator, and adds the batch. Returns
// the merged lse (log2; -inf when every partial is empty) and leaves the normalised row
// in acc (zeros when empty). kL2: read through L2 only (partials other CTAs of this
// kernel wrote).
template <bool kL2, class SlotFn>
__device__ __forceinline__ float merge_partials(const DecodeParams& p, int count, SlotFn slot,
                                                int lane, float4 (&acc)[4]) {
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = zero4;
    float m = -INFINITY, l = 0.f;
    for (int c0 = 0; c0 < count; c0 += kChunkBatch) {
        float4 x[kChunkBatch][4];
        float w[kChunkBatch];
#pragma unroll
        for (int k = 0; k < kChunkBatch; ++k) {
            const int c = c0 + k;
            const bool in = c < count;
            const size_t sl = in ? slot(c) : 0;
            const float4* src = reinterpret_cast<const float4*>(p.ws_o + sl * kHeadDimV);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                x[k][j] = in ? (kL2 ? __ldcg(src + lane + 32 * j) : src[lane + 32 * j]) : zero4;
            w[k] = in ? (kL2 ? __ldcg(p.ws_lse + sl) : p.ws_lse[sl]) : -INFINITY;
        }
        float bm = w[0];
#pragma unroll
        for (int k = 1; k < kChunkBatch; ++k) bm = fmaxf(bm, w[k]);
        const float mn = fmaxf(m, bm);
        if (mn == -INFINITY) continue;                 // nothing but empty partials so far
        const float sc = exp2f(m - mn);                // 0 on the first non-empty batch
        l *= sc;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[j].x *= sc; acc[j].y *= sc; acc[j].z *= sc; acc[j].w *= sc;
        }
#pragma unroll
        for (int k = 0; k < kChunkBatch; ++k) {
            const float wk = exp2f(w[k] - mn);          // 0 for empty partials and padding
            l += wk;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[j].x = fmaf(wk, x[k][j].x, acc[j].x);
                acc[j].y = fmaf(wk, x[k][j].y, acc[j].y);
                acc[j].z = fmaf(wk, x[k][j].z, acc[j].z);
                acc[j].w = fmaf(wk, x[k][j].w, acc[j].w);
            }
        }
        m = mn;
    }
    if (m == -INFINITY) return -INFINITY;
    const float inv = 1.f / l;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        acc[j].x *= inv; acc[j].y *= inv; acc[j].z *= inv; acc[j].w *= inv;
    }
    return m + __log2f(l);
}

// Grid (work sequences, row groups of kCombineRowsPerCta, slices): gridDim.z is the
// largest number of slices a row may be cut into (1 keeps every merge in one CTA).
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const DecodeParams p) {
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int v = blockIdx.x;
    const int base = p.num_splits[v];
    const int n_chunks = p.num_splits[v + 1] - base;
    if (n_chunks == 1) return;
    const bool ws_ok = n_chunks > 0 && base + n_chunks <= p.max_chunks;
    const int slices = ws_ok && v < p.max_chunks ? combine_slices(n_chunks, (int)gridDim.z) : 1;
    const int slice = (int)blockIdx.z;
    if (slice >= slices) return;
    const int b = v % p.batch, t = v / p.batch;
    const int r_local = blockIdx.y * kCombineRowsPerCta + warp;
    const int r = t * kTileRows + r_local;
    const bool valid = r < p.rows;
    const size_t row_index = (size_t)b * p.rows + r;
    float* lse_dst = p.lse + ((size_t)b * p.h_q + (valid ? r % p.h_q : 0)) * p.s_q +
                     (valid ? r / p.h_q : 0);
    float4 acc[4];
    auto chunk_slot = [&](int c) { return (size_t)(base + c) * kTileRows + r_local; };
    if (slices == 1) {
        if (!valid) return;
        if (!ws_ok) {
            if (n_chunks > 0 && lane == 0) record_error(kErrWorkspace, (uint32_t)v & 0xffffffu);
            const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 zero[4] = {zero4, zero4, zero4, zero4};
            store_row(p, row_index, lane, zero);
            if (lane == 0) *lse_dst = -INFINITY;
            return;
        }
        const float lse2 = merge_partials<false>(p, n_chunks, chunk_slot, lane, acc);
        store_row(p, row_index, lane, acc);
        if (lane == 0) *lse_dst = lse2 == -INFINITY ? -INFINITY : lse2 * kLn2;
        return;
    }
    // Slice `slice` of the chunks: [lo, hi). Its merged partial replaces the partial of
    // its first chunk (this warp read that slot for its row before overwriting it).
    const int lo = slice * n_chunks / slices, hi = (slice + 1) * n_chunks / slices;
    if (valid) {
        const float lse2 = merge_partials<false>(
            p, hi - lo, [&](int c) { return chunk_slot(lo + c); }, lane, acc);
        const size_t sl = chunk_slot(lo);
        float4* dst = reinterpret_cast<float4*>(p.ws_o + sl * kHeadDimV);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[lane + 32 * j] = acc[j];
        if (lane == 0) p.ws_lse[sl] = lse2;
    }
    __threadfence();
    __syncthreads();
    int* cnt = combine_counters(p) + (size_t)v * kCombineCounters + blockIdx.y;
    if (threadIdx.x == 0) s_last = atomicAdd(cnt, 1) == slices - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) *cnt = 0;                  // ready for the next call
    if (!valid) return;
    // the slices' partials, in the slots of their first chunks
    const float lse2 = merge_partials<true>(
        p, slices, [&](int s) { return chunk_slot(s * n_chunks / slices); }, lane, acc);
    store_row(p, row_index, lane, acc);
    if (lane == 0) *lse_dst = lse2 == -INFINITY ? -INFINITY : lse2 * kLn2;
}

}  // namespace mla

// LSE-weighted merge of split-KV partials. Chunk c of a work sequence holds the
// normalised output O_c and the log2-domain lse_c of its token subset; the softmax over
// the union weighs chunk c by 2^(lse_c - lse) with lse = log2 sum_c 2^lse_c. Work
// sequences that were not split are skipped (the split kernel already wrote them);
// work sequences that own no page at all (L = 0) get out = 0, lse = -inf here. With
// p.out_f32 set the merged rows are written there in fp32 instead of to p.out.
//
// Layout: one warp per row; lane i owns dims [4 i + 128 j, +4), j < 4: four float4 per
// chunk. The merge is latency-bound, so a warp keeps kChunkBatch chunks' loads in flight
// per round trip: a row split over 30 units needs eight round trips, a row of two
// chunks one. (A warp per 128-dim quarter of a row cut the round trips further but
// multiplied the CTAs fourfold, and the many rows of two chunks lost more to the extra
// waves than the few long rows gained.)
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kCombineThreads = 256;
constexpr int kCombineRowsPerCta = kCombineThreads / 32;   // one warp per row
constexpr int kChunkBatch = 4;

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

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const DecodeParams p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int v = blockIdx.x;
    const int base = p.num_splits[v];
    const int n_chunks = p.num_splits[v + 1] - base;
    if (n_chunks == 1) return;
    const int b = v % p.batch, t = v / p.batch;
    const int r_local = blockIdx.y * kCombineRowsPerCta + warp;
    const int r = t * kTileRows + r_local;
    if (r >= p.rows) return;
    const int i = r / p.h_q, h = r % p.h_q;
    const size_t row_index = (size_t)b * p.rows + r;
    float* lse_dst = p.lse + ((size_t)b * p.h_q + h) * p.s_q + i;
    const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 zero[4] = {zero4, zero4, zero4, zero4};
    if (n_chunks <= 0 || base + n_chunks > p.max_chunks) {
        if (n_chunks > 0 && lane == 0) record_error(kErrWorkspace, (uint32_t)v & 0xffffffu);
        store_row(p, row_index, lane, zero);
        if (lane == 0) *lse_dst = -INFINITY;
        return;
    }
    // max and sum of 2^lse_c over the chunks, lanes striding over chunks
    float mx = -INFINITY;
    for (int c = lane; c < n_chunks; c += 32)
        mx = fmaxf(mx, p.ws_lse[(size_t)(base + c) * kTileRows + r_local]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (mx == -INFINITY) {   // every chunk empty for this row
        store_row(p, row_index, lane, zero);
        if (lane == 0) *lse_dst = -INFINITY;
        return;
    }
    float sum = 0.f;
    for (int c = lane; c < n_chunks; c += 32)
        sum += exp2f(p.ws_lse[(size_t)(base + c) * kTileRows + r_local] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float lse2 = mx + __log2f(sum);
    // out = sum_c 2^(lse_c - lse) O_c: kChunkBatch chunks' loads in flight, then their FMAs
    float4 acc[4] = {zero4, zero4, zero4, zero4};
    for (int c0 = 0; c0 < n_chunks; c0 += kChunkBatch) {
        float4 x[kChunkBatch][4];
        float w[kChunkBatch];
#pragma unroll
        for (int k = 0; k < kChunkBatch; ++k) {
            const int c = c0 + k;
            const bool in = c < n_chunks;
            const size_t slot = (size_t)(base + (in ? c : 0)) * kTileRows + r_local;
            const float4* src = reinterpret_cast<const float4*>(p.ws_o + slot * kHeadDimV);
#pragma unroll
            for (int j = 0; j < 4; ++j) x[k][j] = in ? src[lane + 32 * j] : zero4;
            w[k] = in ? p.ws_lse[slot] : -INFINITY;
        }
#pragma unroll
        for (int k = 0; k < kChunkBatch; ++k) {
            const float wk = exp2f(w[k] - lse2);          // 0 for padding past the last chunk
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[j].x = fmaf(wk, x[k][j].x, acc[j].x);
                acc[j].y = fmaf(wk, x[k][j].y, acc[j].y);
                acc[j].z = fmaf(wk, x[k][j].z, acc[j].z);
                acc[j].w = fmaf(wk, x[k][j].w, acc[j].w);
            }
        }
    }
    store_row(p, row_index, lane, acc);
    if (lane == 0) *lse_dst = lse2 * kLn2;
}

}  // namespace mla

// LSE-weighted merge of split-KV partials. Chunk c of a work sequence holds the
// normalised output O_c and the log2-domain lse_c of its token subset; the softmax over
// the union weighs chunk c by 2^(lse_c - lse) with lse = log2 sum_c 2^lse_c. Work
// sequences that were not split are skipped (the split kernel already wrote them);
// work sequences that own no page at all (L = 0) get out = 0, lse = -inf here. With
// p.out_f32 set the merged rows are written there in fp32 instead of to p.out.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kCombineThreads = 256;
constexpr int kCombineRowsPerCta = kCombineThreads / 32;   // one warp per row

// Row of 512 outputs held as 16 floats per lane: lane owns dims [4 lane + 128 j, +4).
__device__ __forceinline__ void store_out_row(const DecodeParams& p, size_t row_index,
                                              const float (&acc)[16], int lane) {
    if (p.out_f32) {
        float4* dst = reinterpret_cast<float4*>(p.out_f32 + row_index * kHeadDimV);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            dst[lane + 32 * j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
        return;
    }
    uint2* dst = reinterpret_cast<uint2*>(p.out + row_index * kHeadDimV);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[4 * j + 0], acc[4 * j + 1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[4 * j + 2], acc[4 * j + 3]);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        dst[lane + 32 * j] = pk;
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
    const float zero[16] = {};
    float* lse_dst = p.lse + ((size_t)b * p.h_q + h) * p.s_q + i;
    if (n_chunks <= 0 || base + n_chunks > p.max_chunks) {
        if (n_chunks > 0 && lane == 0) record_error(kErrWorkspace, (uint32_t)v & 0xffffffu);
        store_out_row(p, row_index, zero, lane);
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
        store_out_row(p, row_index, zero, lane);
        if (lane == 0) *lse_dst = -INFINITY;
        return;
    }
    float sum = 0.f;
    for (int c = lane; c < n_chunks; c += 32)
        sum += exp2f(p.ws_lse[(size_t)(base + c) * kTileRows + r_local] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float lse2 = mx + __log2f(sum);
    // out = sum_c 2^(lse_c - lse) O_c; lane owns dims [4 lane, 4 lane + 4) and +128 j.
    // Chunks go two at a time so both chunks' loads are in flight together (most split
    // rows have exactly two chunks).
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    auto add = [&](const float4 (&x)[4], float w) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc[4 * j + 0] = fmaf(w, x[j].x, acc[4 * j + 0]);
            acc[4 * j + 1] = fmaf(w, x[j].y, acc[4 * j + 1]);
            acc[4 * j + 2] = fmaf(w, x[j].z, acc[4 * j + 2]);
            acc[4 * j + 3] = fmaf(w, x[j].w, acc[4 * j + 3]);
        }
    };
    int c = 0;
    for (; c + 2 <= n_chunks; c += 2) {
        const size_t s0 = (size_t)(base + c) * kTileRows + r_local;
        const size_t s1 = s0 + kTileRows;
        const float4* src0 = reinterpret_cast<const float4*>(p.ws_o + s0 * kHeadDimV);
        const float4* src1 = reinterpret_cast<const float4*>(p.ws_o + s1 * kHeadDimV);
        float4 x0[4], x1[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x0[j] = src0[lane + 32 * j];
            x1[j] = src1[lane + 32 * j];
        }
        const float w0 = exp2f(p.ws_lse[s0] - lse2);
        const float w1 = exp2f(p.ws_lse[s1] - lse2);
        add(x0, w0);
        add(x1, w1);
    }
    if (c < n_chunks) {
        const size_t s0 = (size_t)(base + c) * kTileRows + r_local;
        const float4* src0 = reinterpret_cast<const float4*>(p.ws_o + s0 * kHeadDimV);
        float4 x0[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) x0[j] = src0[lane + 32 * j];
        add(x0, exp2f(p.ws_lse[s0] - lse2));
    }
    store_out_row(p, row_index, acc, lane);
    if (lane == 0) *lse_dst = lse2 * kLn2;
}

}  // namespace mla

// Merge of partial decode results that several devices computed for the same query rows
// over disjoint token ranges of each sequence (split-KV across devices). Part g holds,
// for every row, the output O_g normalised over its own tokens (fp32) and
// lse_g = ln sum_{t in part g} exp(s_t). The softmax over the union of the parts weighs
// part g by exp(lse_g - lse) with lse = ln sum_g exp(lse_g): the same identity the
// in-device combine applies to split chunks, here in the natural-log domain the public
// lse uses. A part with lse_g = -inf (no visible token) weighs nothing; a row no part
// sees gets out = 0, lse = -inf.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kRankCombineThreads = 256;
constexpr int kRankCombineRowsPerCta = kRankCombineThreads / 32;   // one warp per row

struct RankCombineParams {
    const float* o_parts;      // [parts][batch][s_q][h_q][512]
    const float* lse_parts;    // [parts][batch][h_q][s_q]
    __nv_bfloat16* out;        // [batch][s_q][h_q][512]
    float* lse;                // [batch][h_q][s_q]
    int parts, batch, s_q, h_q;
};

__global__ void __launch_bounds__(kRankCombineThreads)
rank_combine_kernel(const RankCombineParams p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long rows = (long long)p.batch * p.s_q * p.h_q;
    const long long row = (long long)blockIdx.x * kRankCombineRowsPerCta + warp;
    if (row >= rows) return;
    // row = (b * s_q + i) * h_q + h, the order of `out`
    const int h = (int)(row % p.h_q);
    const long long bi = row / p.h_q;
    const int i = (int)(bi % p.s_q);
    const long long b = bi / p.s_q;
    const size_t lse_index = ((size_t)b * p.h_q + h) * p.s_q + i;
    const size_t lse_stride = (size_t)rows;
    const size_t o_stride = (size_t)rows * kHeadDimV;

    float mx = -INFINITY;
    for (int g = lane; g < p.parts; g += 32) mx = fmaxf(mx, p.lse_parts[g * lse_stride + lse_index]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    float lse_row = -INFINITY;
    if (mx != -INFINITY) {
        float sum = 0.f;
        for (int g = lane; g < p.parts; g += 32) sum += expf(p.lse_parts[g * lse_stride + lse_index] - mx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        lse_row = mx + logf(sum);
        // parts four at a time, every load of a group in flight before its arithmetic
        for (int g0 = 0; g0 < p.parts; g0 += 4) {
            float w[4];
            float4 x[4][4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int g = g0 + k;
                w[k] = g < p.parts ? expf(p.lse_parts[g * lse_stride + lse_index] - lse_row) : 0.f;
                // an empty part weighs 0 and its O (possibly NaN) is not read
                if (w[k] != 0.f) {
                    const float4* src = reinterpret_cast<const float4*>(
                        p.o_parts + g * o_stride + (size_t)row * kHeadDimV);
#pragma unroll
                    for (int j = 0; j < 4; ++j) x[k][j] = src[lane + 32 * j];
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (w[k] == 0.f) continue;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc[4 * j + 0] = fmaf(w[k], x[k][j].x, acc[4 * j + 0]);
                    acc[4 * j + 1] = fmaf(w[k], x[k][j].y, acc[4 * j + 1]);
                    acc[4 * j + 2] = fmaf(w[k], x[k][j].z, acc[4 * j + 2]);
                    acc[4 * j + 3] = fmaf(w[k], x[k][j].w, acc[4 * j + 3]);
                }
            }
        }
    }
    uint2* dst = reinterpret_cast<uint2*>(p.out + (size_t)row * kHeadDimV);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc[4 * j + 0], acc[4 * j + 1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc[4 * j + 2], acc[4 * j + 3]);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        dst[lane + 32 * j] = pk;
    }
    if (lane == 0) p.lse[lse_index] = lse_row;
}

}  // namespace mla

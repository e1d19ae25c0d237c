// Cache append: writes each sequence's new latent rows into their pages through the
// block table (the block-based paging of the FlashMLA articles; the operation is a
// byte copy). One warp per new row moves its 1152 bytes as 72 coalesced 16-byte words.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kAppendThreads = 256;
constexpr int kRowWords = kHeadDim * 2 / 16;   // 72 x 16 B per cache row

// Row w = b * s_new + j of kv_new goes to position seqlens[b] + j of sequence b. A
// position past the block table or a block id outside the pool is recorded as a bad
// input and its row is skipped (nothing is written for it).
__global__ void __launch_bounds__(kAppendThreads)
kv_append_kernel(const uint4* __restrict__ kv_new, int s_new,
                 const int32_t* __restrict__ block_table, int max_blocks,
                 const int32_t* __restrict__ seqlens, int batch, uint4* __restrict__ kcache,
                 int num_blocks) {
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (long long)batch * s_new) return;
    const int b = (int)(w / s_new), j = (int)(w % s_new);
    const long long L = seqlens[b];
    const long long t = L + j;
    if (L < 0 || t >= (long long)max_blocks * kBlock) {
        if (lane == 0) record_error(kErrBadInput, 0x400000u | ((uint32_t)b & 0x3fffffu));
        return;
    }
    const int blk = block_table[(size_t)b * max_blocks + (size_t)(t / kBlock)];
    if (blk < 0 || blk >= num_blocks) {
        if (lane == 0) record_error(kErrBadInput, 0x800000u | ((uint32_t)b & 0x7fffffu));
        return;
    }
    const uint4* src = kv_new + (size_t)w * kRowWords;
    uint4* dst = kcache + ((size_t)blk * kBlock + (size_t)(t % kBlock)) * kRowWords;
    for (int i = lane; i < kRowWords; i += 32) dst[i] = src[i];
}

}  // namespace mla

// FP8 cache append: quantizes each new bf16 latent row into the FP8 row format and writes
// it into its page through the block table. The format (this library's own; the pages
// fix none for the cache) is, per token, 656 bytes:
//   [0, 512)    the 512 latent dims as E4M3 codes
//   [512, 528)  four fp32 scales, one per 128-dim group: s = fp32(amax / 448)
//   [528, 656)  the 64 rope dims, unchanged bf16
// code = E4M3(fp32(x / s)) with round-to-nearest-even and saturation at +-448 (0 when
// s = 0). One warp per row: lane l quantizes dims [16 l, 16 l + 16) (group l / 8, so a
// group's amax is a max over 8 lanes) and lanes 0-7 copy the rope dims.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kFp8RowBytes = 656;
constexpr int kFp8ScaleOff = 512;
constexpr int kFp8RopeOff = 528;
constexpr float kE4m3Max = 448.0f;

// Two fp32 values to E4M3 codes, nearest-even, saturating: `lo` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// max(|a|, |b|) that returns NaN if either is NaN (a NaN in a group makes its scale NaN).
__device__ __forceinline__ float abs_max_nan(float a, float b) {
    const float x = fabsf(a), y = fabsf(b);
    return (x != x || y != y) ? __int_as_float(0x7fc00000) : fmaxf(x, y);
}

// Row w = b * s_new + j of kv_new goes to position seqlens[b] + j of sequence b. A
// position past the block table or a block id outside the pool is recorded as a bad
// input and its row is skipped (nothing is written for it).
__global__ void __launch_bounds__(kAppendThreads)
kv_append_fp8_kernel(const __nv_bfloat16* __restrict__ kv_new, int s_new,
                     const int32_t* __restrict__ block_table, int max_blocks,
                     const int32_t* __restrict__ seqlens, int batch,
                     uint8_t* __restrict__ kcache, int num_blocks) {
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
    const __nv_bfloat16* src = kv_new + (size_t)w * kHeadDim;
    uint8_t* dst = kcache + ((size_t)blk * kBlock + (size_t)(t % kBlock)) * kFp8RowBytes;

    const uint4 r0 = reinterpret_cast<const uint4*>(src)[2 * lane];
    const uint4 r1 = reinterpret_cast<const uint4*>(src)[2 * lane + 1];
    const uint32_t words[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
    float x[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        x[2 * k] = __uint_as_float(words[k] << 16);
        x[2 * k + 1] = __uint_as_float(words[k] & 0xffff0000u);
    }
    float amax = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) amax = abs_max_nan(amax, x[k]);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = abs_max_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, kE4m3Max);
    uint32_t codes[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t c = 0;
        if (s != 0.f) {
            c = e4m3x2(__fdiv_rn(x[4 * k], s), __fdiv_rn(x[4 * k + 1], s)) |
                (e4m3x2(__fdiv_rn(x[4 * k + 2], s), __fdiv_rn(x[4 * k + 3], s)) << 16);
        }
        codes[k] = c;
    }
    reinterpret_cast<uint4*>(dst)[lane] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    if ((lane & 7) == 0) reinterpret_cast<float*>(dst + kFp8ScaleOff)[lane >> 3] = s;
    if (lane < 8)
        reinterpret_cast<uint4*>(dst + kFp8RopeOff)[lane] =
            reinterpret_cast<const uint4*>(src + 512)[lane];
}

}  // namespace mla

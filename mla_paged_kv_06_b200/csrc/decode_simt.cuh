// Correctness-first decode on CUDA cores: one warp per query row, lanes split the
// 576 dims of each dot product and the 512 output dims, fp32 online softmax in the
// log2 domain. It walks the same schedule and writes the same partials as the
// tensor-core kernel, so it doubles as an independent check of that kernel.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kSimtThreads = 256;
constexpr int kSimtWarps = kSimtThreads / 32;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Writes one row's result: final output when the work sequence is unsplit, a
// normalised fp32 partial otherwise. `o` holds 16 dims per lane (d = lane + 32 j).
__device__ __forceinline__ void simt_store_row(const DecodeParams& p, int b, int r, int r_local,
                                               int n_chunks, int part, const float* o,
                                               float m2, float l) {
    const int lane = threadIdx.x & 31;
    const bool empty = !(l > 0.f);
    const float inv = empty ? 0.f : 1.f / l;
    const float lse2 = empty ? -INFINITY : m2 + __log2f(l);
    if (n_chunks == 1) {
        const int i = r / p.h_q, h = r % p.h_q;
        if (p.out_f32) {
            float* dst = p.out_f32 + ((size_t)b * p.rows + r) * kHeadDimV;
#pragma unroll
            for (int j = 0; j < 16; ++j) dst[lane + 32 * j] = o[j] * inv;
        } else {
            __nv_bfloat16* dst = p.out + ((size_t)b * p.rows + r) * kHeadDimV;
#pragma unroll
            for (int j = 0; j < 16; ++j) dst[lane + 32 * j] = __float2bfloat16_rn(o[j] * inv);
        }
        if (lane == 0)
            p.lse[((size_t)b * p.h_q + h) * p.s_q + i] = empty ? -INFINITY : lse2 * kLn2;
    } else {
        float* dst = p.ws_o + ((size_t)part * kTileRows + r_local) * kHeadDimV;
#pragma unroll
        for (int j = 0; j < 16; ++j) dst[lane + 32 * j] = o[j] * inv;
        if (lane == 0) p.ws_lse[(size_t)part * kTileRows + r_local] = lse2;
    }
}

__global__ void __launch_bounds__(kSimtThreads)
decode_simt_kernel(const DecodeParams p) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int num_units = p.metadata[0];
    const int V = p.batch * p.tiles;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
        const int32_t* m = p.metadata + kMetaInts * (u + 1);
        const int v_begin = m[0], k_begin = m[1], v_end = m[2], k_end = m[3];
        for (int v = v_begin; v <= v_end && v < V; ++v) {
            const int b = v % p.batch, t = v / p.batch;
            const int L = checked_seqlen(p, b);
            const int nblk = pages_of(L);
            const int k_lo = v == v_begin ? k_begin : 0;
            int k_hi = v == v_end ? k_end : nblk;
            if (k_hi > nblk) k_hi = nblk;
            if (k_lo >= k_hi) continue;
            const int chunk = v == v_begin ? m[4] : 0;
            const int n_chunks = p.num_splits[v + 1] - p.num_splits[v];
            const int part = p.num_splits[v] + chunk;
            if (n_chunks > 1 && part >= p.max_chunks) {
                record_error(kErrWorkspace, (uint32_t)v & 0xffffffu);
                continue;
            }
            for (int r_local = warp; r_local < kTileRows; r_local += kSimtWarps) {
                const int r = t * kTileRows + r_local;
                if (r >= p.rows) break;
                const int i = r / p.h_q;
                const int n = visible_tokens(L, p.s_q, i, p.causal);
                const int t_lo = k_lo * kBlock;
                int t_hi = k_hi * kBlock;
                if (t_hi > n) t_hi = n;
                // q row, pre-scaled into the log2 domain: lane holds d = lane + 32 j
                const __nv_bfloat16* qr = p.q + ((size_t)b * p.rows + r) * kHeadDim;
                float qv[18];
#pragma unroll
                for (int j = 0; j < 18; ++j)
                    qv[j] = __bfloat162float(qr[lane + 32 * j]) * p.scale_log2;
                float o[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) o[j] = 0.f;
                float m2 = -INFINITY, l = 0.f;
                for (int tok = t_lo; tok < t_hi; ++tok) {
                    const int pid = p.block_table[(size_t)b * p.max_blocks + tok / kBlock];
                    if (pid < 0 || pid >= p.num_blocks) {
                        record_error(kErrBadInput, (uint32_t)(0x800000u | (b & 0x7fffff)));
                        continue;
                    }
                    const __nv_bfloat16* kr =
                        p.kcache + ((size_t)pid * kBlock + (tok % kBlock)) * kHeadDim;
                    float kv[18];
#pragma unroll
                    for (int j = 0; j < 18; ++j) kv[j] = __bfloat162float(kr[lane + 32 * j]);
                    float dot = 0.f;
#pragma unroll
                    for (int j = 0; j < 18; ++j) dot = fmaf(qv[j], kv[j], dot);
                    const float s = warp_sum(dot);
                    const float m_new = fmaxf(m2, s);
                    const float corr = exp2f(m2 - m_new);
                    const float pr = exp2f(s - m_new);
                    l = l * corr + pr;
#pragma unroll
                    for (int j = 0; j < 16; ++j) o[j] = fmaf(o[j], corr, pr * kv[j]);
                    m2 = m_new;
                }
                simt_store_row(p, b, r, r_local, n_chunks, part, o, m2, l);
            }
        }
    }
}

}  // namespace mla

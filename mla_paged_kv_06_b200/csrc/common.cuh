// Shared device-side definitions for the paged MLA decode kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sched.cuh"

namespace mla {

constexpr int kHeadDim = 576;    // latent (512) + rope (64) dims of a cache row
constexpr int kHeadDimV = 512;   // V = first 512 dims of the row
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device-side error word: bits 0-7 the kind, bits 8-31 where it arose. The first
// error recorded since the last read sticks.
enum ErrorKind : uint32_t { kErrNone = 0, kErrTimeout = 1, kErrBadInput = 2, kErrWorkspace = 3 };

// Programmatic dependent launch. The split kernels are launched with programmatic stream
// serialization, so they may be scheduled while the metadata kernel before them in the
// stream still runs (it signals launch_dependents() as it starts): their set-up (barrier
// initialisation, TMEM allocation, tensor-map prefetch) overlaps it, and each thread then
// waits in grid_dependency_wait(), before its first global memory access, until the
// previous kernel has completed and its writes are visible. (The same link from the split
// kernel to the combine measured slower and is not used.)
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Combine counters per work sequence in the workspace: one per 8-row group of a tile.
constexpr int kCombineCounters = 16;

// Everything one decode launch needs. Plain pointers; layouts as in include/mla.h.
struct DecodeParams {
    const __nv_bfloat16* q;        // [batch][s_q][h_q][576]
    const __nv_bfloat16* kcache;   // [num_blocks][64][576]
    const int32_t* block_table;    // [batch][max_blocks]
    const int32_t* seqlens;        // [batch]
    const int32_t* metadata;       // header + per-unit ranges
    const int32_t* num_splits;     // [V + 1] chunk prefix
    float* ws_lse;                 // [max_chunks][128]   log2-domain partial lse
    float* ws_o;                   // [max_chunks][128][512] normalised partial outputs
    __nv_bfloat16* out;            // [batch][s_q][h_q][512]
    float* lse;                    // [batch][h_q][s_q]
    float* out_f32;                // when set, fp32 [batch][s_q][h_q][512] replaces `out`
    int num_blocks, max_blocks;
    int batch, s_q, h_q, rows, tiles;
    int max_chunks;                // partial slots the workspace holds
    float scale_log2;              // scale * log2(e): scores kept in the log2 domain
    int causal;
};

// The combine's counters, [max_chunks][kCombineCounters] int32, follow the output
// partials in the workspace (their end is 256-byte aligned: 256 KB per slot).
__device__ __forceinline__ int* combine_counters(const DecodeParams& p) {
    return reinterpret_cast<int*>(p.ws_o + (size_t)p.max_chunks * kTileRows * kHeadDimV);
}

// Visible tokens of query i (causal decode appends the s_q queries at the end).
__device__ __forceinline__ int visible_tokens(int L, int s_q, int i, int causal) {
    return causal ? L - s_q + i + 1 : L;
}

}  // namespace mla

// Device error word of the library (one translation unit includes this header).
__device__ uint32_t g_mla_error = 0;
// Limit of every pipeline wait, in ns, and the stall test hook (mla_test_set_stall sets
// both on the current device; kept out of DecodeParams, whose size the 2-CTA kernel's
// register budget feels).
__device__ unsigned long long g_mla_wait_limit_ns = 2000000000ull;
__device__ int g_mla_debug_stall = 0;

namespace mla {

__device__ __forceinline__ void record_error(uint32_t kind, uint32_t where) {
    atomicCAS(&g_mla_error, 0u, (kind & 0xffu) | (where << 8));
}

// Sequence length with the block-table bound enforced: a length the table cannot
// hold is an input error; the kernel records it and uses the largest valid length.
__device__ __forceinline__ int checked_seqlen(const DecodeParams& p, int b) {
    int L = p.seqlens[b];
    int cap = p.max_blocks * kBlock;
    if (L < 0 || L > cap) {
        record_error(kErrBadInput, (uint32_t)b & 0xffffffu);
        L = L < 0 ? 0 : cap;
    }
    return L;
}

}  // namespace mla

// Device split-KV scheduler: one CTA computes the whole schedule so the call needs no
// host round trip and can sit inside a captured CUDA graph.
#pragma once

#include "common.cuh"

namespace mla {

constexpr int kMetaThreads = 1024;
// Largest table (cumulative costs C[V+1] and page counts per sequence, int32) the
// scheduler keeps in shared memory; larger batches use the num_splits buffer itself.
constexpr size_t kMetaSmemMax = 160 * 1024;

// Block-wide exclusive scan of one int64 per thread; returns the block total.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t x, int64_t* smem_warp,
                                                        int64_t* out_prefix) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) smem_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int64_t w = lane < (int)(blockDim.x >> 5) ? smem_warp[lane] : 0;
        int64_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int64_t y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        smem_warp[lane] = wi - w;          // exclusive prefix of warp totals
        if (lane == 31) smem_warp[32] = wi;
    }
    __syncthreads();
    *out_prefix = smem_warp[warp] + incl - x;
    int64_t total = smem_warp[32];
    __syncthreads();
    return total;
}

// metadata: header {num_units, tiles, batch, h_q, s_q, unit_cost, overhead, tile_aligned}
// then one
// {v_begin, page_begin, v_end, page_end, chunk_begin, 0, 0, 0} per unit.
// `in_smem`: the cost table C[0..V] and page counts live in dynamic shared memory (the
// launch provides (V + 1 + batch) int32), so the per-unit searches never wait on L2, and
// one pass locates the units and counts the chunks; otherwise num_splits holds the costs
// while the units are located, is then overwritten with the chunk prefix, and the lengths
// are re-read from seqlens.
__global__ void __launch_bounds__(kMetaThreads)
metadata_kernel(const int32_t* __restrict__ seqlens, int batch, int h_q, int s_q, int tiles,
                int num_units, int in_smem,
                int32_t* __restrict__ metadata, int32_t* __restrict__ num_splits) {
    __shared__ int64_t warp_sums[33];
    extern __shared__ int32_t dyn[];
    launch_dependents();         // the decode kernel may set up meanwhile; it waits for us
    const int V = batch * tiles;
    const int overhead = overhead_pages(h_q, s_q);
    int32_t* Cs = in_smem ? dyn : num_splits;               // cumulative costs C[0..V]
    int32_t* Ps = in_smem ? dyn + V + 1 : nullptr;          // pages per sequence
    if (in_smem) {
        for (int b = threadIdx.x; b < batch; b += blockDim.x) {
            const int L = seqlens[b];
            Ps[b] = pages_of(L < 0 ? 0 : L);
        }
        __syncthreads();
    }
    auto pages = [&](int v) {
        if (Ps) return (int)Ps[v % batch];
        const int L = seqlens[v % batch];
        return pages_of(L < 0 ? 0 : L);
    };

    // Phase 1: cumulative costs.
    int64_t carry = 0;
    for (int base = 0; base < V; base += blockDim.x) {
        int v = base + threadIdx.x;
        int64_t cost = v < V ? (int64_t)overhead + pages(v) : 0;
        int64_t pre;
        int64_t tot = block_exclusive_scan(cost, warp_sums, &pre);
        int64_t c = carry + pre;
        if (v < V) {
            if (c > 0x7fffffffLL) record_error(kErrBadInput, 0xfffffeu);
            Cs[v] = (int32_t)(c > 0x7fffffffLL ? 0x7fffffff : c);
        }
        carry += tot;
    }
    if (threadIdx.x == 0) {
        if (carry > 0x7fffffffLL) { record_error(kErrBadInput, 0xfffffeu); carry = 0x7fffffff; }
        Cs[V] = (int32_t)carry;
    }
    __syncthreads();
    auto C = [&](int v) { return (int64_t)Cs[v]; };
    // the header, from a thread that has no unit or sequence of its own when there is one
    if (threadIdx.x == blockDim.x - 1) {
        const int64_t W = header_unit_cost(num_units, tiles, batch, V, C);
        metadata[0] = num_units; metadata[1] = tiles; metadata[2] = batch;
        metadata[3] = h_q; metadata[4] = s_q;
        metadata[5] = (int32_t)(W > 0x7fffffffLL ? 0x7fffffff : W);
        metadata[6] = overhead; metadata[7] = tile_aligned(tiles, num_units) ? 1 : 0;
    }
    // Phase 2: unit u locates its first and one-past-last page.
    auto write_unit = [&](int u) {
        int vb, kb, ve, ke, chunk;
        unit_range(u, num_units, tiles, batch, V, overhead, C, pages, &vb, &kb, &ve, &ke, &chunk);
        int32_t* m = metadata + kMetaInts * (u + 1);
        m[0] = vb; m[1] = kb; m[2] = ve; m[3] = ke; m[4] = chunk;
        m[5] = 0; m[6] = 0; m[7] = 0;
    };
    // Phase 3: chunk counts -> exclusive prefix into num_splits. With the costs in shared
    // memory the two phases share one pass, a thread taking unit i and sequence i (their
    // chains overlap, and no barrier separates them); with the costs kept in num_splits,
    // which phase 3 overwrites, phase 2 runs first and phase 3 goes tile by tile.
    // A sequence's chunk count reads its own cost C[v] (overwritten only after it is read,
    // in the same pass), and the costs at multiples of batch: the start C[t batch] of its
    // tile's line and C[batch] or C[V] for the line's unit cost. The tiles' lines repeat the
    // same costs, so C[t batch] = t C[batch]: phase 3 takes those from C[batch], read
    // before the first overwrite.
    int64_t c_batch = 0;
    if (!in_smem) {
        for (int u = threadIdx.x; u < num_units; u += blockDim.x) write_unit(u);
        c_batch = C(batch);
        __syncthreads();
    }
    auto C3 = [&](int v) {
        if (in_smem || v % batch != 0) return (int64_t)Cs[v];
        return (int64_t)(v / batch) * c_batch;
    };
    const int span = in_smem && num_units > V ? num_units : V;
    carry = 0;
    for (int base = 0; base < span; base += blockDim.x) {
        const int i = base + threadIdx.x;
        if (in_smem && i < num_units) write_unit(i);
        int n = i < V ? chunks_of_v(i, num_units, tiles, batch, V, overhead, C3, pages) : 0;
        int64_t pre;
        int64_t tot = block_exclusive_scan(n, warp_sums, &pre);   // also a barrier
        if (i < V) num_splits[i] = (int32_t)(carry + pre);
        carry += tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) num_splits[V] = (int32_t)carry;
}

}  // namespace mla

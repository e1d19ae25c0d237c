// Work items of the split kernels: what one CTA (or CTA pair) decodes between loading
// a query tile and writing its result, walked in the same order by every role.
#pragma once

#include "common.cuh"

namespace mla {

// One piece of work: pages [k_lo, k_hi) of work sequence v.
struct Item {
    int v, b, t, L, k_lo, k_hi, chunk, n_chunks, part;
    __device__ int pages() const { return k_hi - k_lo; }
    __device__ int steps() const { return (k_hi - k_lo + 1) >> 1; }   // pair steps: 2 pages
};

// Iterates the items of every unit a CTA (or cluster) owns, units first_unit,
// first_unit + unit_step, ..., in the same order for all roles.
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

// First pool row of logical page k of sequence b, or the row just past the pool (a box
// there is read as zeros) when the page is outside [k_lo, k_hi) or its id is invalid.
__device__ __forceinline__ int page_row(const DecodeParams& p, int b, int k, int k_hi) {
    if (k >= k_hi) return p.num_blocks * kBlock;
    const int pid = p.block_table[(size_t)b * p.max_blocks + k];
    if (pid < 0 || pid >= p.num_blocks) {
        record_error(kErrBadInput, 0x800000u | ((uint32_t)b & 0x7fffffu));
        return p.num_blocks * kBlock;
    }
    return pid * kBlock;
}

}  // namespace mla

// Split-KV tile scheduler arithmetic, shared by the device metadata kernel and the
// host planner (mla_plan_host), so both produce the same schedule bit for bit.
//
// Cost model. Work sequence v = tile * batch + b owns nblk(v) = ceil(L_b / 64) pages
// and pays a fixed `overhead` (in page units) for loading its query tile and writing
// its result. Laying the work sequences end to end gives a cost line:
//   C[v]            = sum_{v' < v} (overhead + nblk(v'))
//   page k of v     occupies position P(v, k) = C[v] + overhead + k
// With W = max(ceil(C[V] / units), kMinUnitCost), unit u owns every page whose position lies in
// [u*W, (u+1)*W). So each unit owns one contiguous run of pages, every page has
// exactly one owner, and a work sequence whose pages straddle a multiple of W is
// split there. Tile-major numbering puts tile t of sequence b about units/tiles units
// after tile t-1 of b, so both tiles stream the same pages at about the same time and
// the second read hits L2.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define MLA_HD __host__ __device__ __forceinline__
#else
#define MLA_HD inline
#endif

namespace mla {

constexpr int kBlock = 64;
constexpr int kTileRows = 128;
// Fixed cost of one work sequence in page units: loading its query tile, refilling the
// pipeline and its epilogue. Measured on B200: an item boundary of the 2-CTA kernel costs
// about as much as three and a half pages; one of the 1-CTA kernel (sequences of at most
// kSoloMaxRows query rows), whose q rows ride in a slot of the page ring and whose
// epilogue overlaps the next item's first QK, about half a page.
constexpr int kOverheadPages = 3;
constexpr int kOverheadPagesSolo = 1;
constexpr int kSoloMaxRows = 64;

MLA_HD int overhead_pages(int h_q, int s_q) {
    return h_q * s_q <= kSoloMaxRows ? kOverheadPagesSolo : kOverheadPages;
}
constexpr int kMetaInts = 8;
// Smallest per-unit cost: a split costs a partial tile write and a combine read, so
// cutting work finer than a few pages loses more than it balances.
constexpr int kMinUnitCost = 4;

// Per-unit cost budget W for a total cost over `units` units.
MLA_HD int64_t unit_cost(int64_t total, int units) {
    int64_t w = (total + units - 1) / units;
    return w < kMinUnitCost ? kMinUnitCost : w;
}

MLA_HD int ceil_div(int a, int b) { return (a + b - 1) / b; }
MLA_HD int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

MLA_HD int num_tiles(int h_q, int s_q) { return ceil_div(h_q * s_q, kTileRows); }

MLA_HD int pages_of(int seqlen) { return seqlen <= 0 ? 0 : ceil_div(seqlen, kBlock); }

// Unit owning cost position p.
MLA_HD int unit_of(int64_t p, int64_t W) { return (int)(p / W); }

// Chunks work sequence v is split into, from its cost start C[v] and page count.
MLA_HD int chunks_of(int64_t Cv, int nblk, int64_t W, int overhead) {
    if (nblk <= 0) return 0;
    int64_t p0 = Cv + overhead;
    int64_t p1 = p0 + nblk - 1;
    return unit_of(p1, W) - unit_of(p0, W) + 1;
}

// Unit range record written into metadata[8 + 8u ..].
struct UnitRange {
    int v_begin, page_begin, v_end, page_end, chunk_begin;
};

// First page position >= target, as (v, page). C(v) returns the cumulative cost
// C[v] (v in [0, V]) and nblk(v) the page count of v. Returns (V, 0) when no page lies
// at or after target.
template <class CostFn, class PagesFn>
MLA_HD void locate(const int64_t target, CostFn C, PagesFn nblk, int V, int overhead,
                   int* v_out, int* k_out) {
    // smallest v with C[v+1] > target: its page range [C[v]+overhead, C[v+1]) ends
    // after target
    int lo = 0, hi = V;
    while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)C(mid + 1) > target) hi = mid; else lo = mid + 1;
    }
    int v = lo;
    while (v < V && nblk(v) == 0) ++v;     // empty sequences own no page
    if (v >= V) { *v_out = V; *k_out = 0; return; }
    int64_t k = target - ((int64_t)C(v) + overhead);
    *v_out = v;
    *k_out = k < 0 ? 0 : (int)k;
}

}  // namespace mla

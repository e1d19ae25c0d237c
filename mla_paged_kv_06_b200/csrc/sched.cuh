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
// split there.
//
// Tile-aligned cut. With T > 1 row tiles per sequence and at least T units, every tile
// has the same cost line (the pages are the sequence's), so the line is cut per tile:
// tile t owns units [floor(t U / T), floor((t+1) U / T)) and cuts its own line of the
// batch's costs C[0..batch] with W_t = max(ceil(C[batch] / U_t), kMinUnitCost). Where
// the tiles get equal unit counts, unit u of tile 0 and unit u + U/T of tile 1 own the
// same pages in the same order and stream them at the same time, so each page comes
// from DRAM once for all tiles. (On one line the tiles' runs drift apart by up to W
// pages, and the second read of a page missed L2.)
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
// pipeline and its epilogue. Measured on B200 (per-CTA timelines, a least-squares fit of
// unit time over pages and items): an item boundary of the 2-CTA kernel costs about as
// much as three and a half pages; one of the 1-CTA kernel (sequences of at most
// kSoloMaxRows query rows), whose q rows ride in a slot of the page ring and whose
// epilogue overlaps the next item's first QK, about 0.6 of a page with 16 rows (three
// stages) but 2.5 pages with 64 rows (two stages, a 72 KB q slot and a 48 KB copy of the
// q rows into shared memory). For 33-64 rows, 2 measured best once QK and PV got issuers
// of their own (2, 3 and 4 timed).
constexpr int kOverheadPages = 3;
constexpr int kOverheadPagesSolo = 1;
constexpr int kOverheadPagesSoloWide = 2;   // 1-CTA kernel, 33-64 query rows
constexpr int kSoloMaxRows = 64;

MLA_HD int overhead_pages(int h_q, int s_q) {
    const int rows = h_q * s_q;
    if (rows > kSoloMaxRows) return kOverheadPages;
    return rows <= 32 ? kOverheadPagesSolo : kOverheadPagesSoloWide;
}
constexpr int kMetaInts = 8;
// Smallest per-unit cost: a split costs a partial tile write and a combine read, so
// cutting work finer than a few pages loses more than it balances.
constexpr int kMinUnitCost = 4;

// a / b for a >= 0, b > 0. The values divided here are positions on a cost line of int32
// costs, so on the device they nearly always fit the 32-bit divide, which is several
// times shorter than the 64-bit one; the quotient is the same either way.
MLA_HD int64_t div_nonneg(int64_t a, int64_t b) {
#ifdef __CUDA_ARCH__
    if ((((uint64_t)a | (uint64_t)b) >> 32) == 0) return (int64_t)((uint32_t)a / (uint32_t)b);
#endif
    return a / b;
}

// Per-unit cost budget W for a total cost over `units` units.
MLA_HD int64_t unit_cost(int64_t total, int units) {
    int64_t w = div_nonneg(total + units - 1, units);
    return w < kMinUnitCost ? kMinUnitCost : w;
}

MLA_HD int ceil_div(int a, int b) { return (a + b - 1) / b; }
MLA_HD int64_t ceil_div64(int64_t a, int64_t b) { return div_nonneg(a + b - 1, b); }

MLA_HD int num_tiles(int h_q, int s_q) { return ceil_div(h_q * s_q, kTileRows); }

MLA_HD int pages_of(int seqlen) { return seqlen <= 0 ? 0 : ceil_div(seqlen, kBlock); }

// Unit owning cost position p.
MLA_HD int unit_of(int64_t p, int64_t W) { return (int)div_nonneg(p, W); }

// Chunks work sequence v is split into, from its cost start C[v] and page count.
MLA_HD int chunks_of(int64_t Cv, int nblk, int64_t W, int overhead) {
    if (nblk <= 0) return 0;
    int64_t p0 = Cv + overhead;
    int64_t p1 = p0 + nblk - 1;
    return unit_of(p1, W) - unit_of(p0, W) + 1;
}

MLA_HD bool tile_aligned(int tiles, int units) { return tiles > 1 && units >= tiles; }
MLA_HD int tile_first_unit(int t, int tiles, int units) {
    return (int)div_nonneg((int64_t)t * units, tiles);
}

// Where unit u cuts: the line it cuts (its first work sequence v0 and sequence count n,
// the costs of that line being C[v0 + i] - C[v0]), its index within the line's units and
// the line's per-unit cost. C(v) is the cumulative cost over all V work sequences.
struct UnitCut {
    int v0, n, local;
    int64_t W;
};

template <class CostFn>
MLA_HD UnitCut cut_of_unit(int u, int units, int tiles, int batch, int V, CostFn C) {
    UnitCut c;
    if (!tile_aligned(tiles, units)) {
        c.v0 = 0; c.n = V; c.local = u;
        c.W = unit_cost(C(V), units);
        return c;
    }
    const int t = (int)div_nonneg(((int64_t)u + 1) * tiles - 1, units);
    const int first = tile_first_unit(t, tiles, units);
    c.v0 = t * batch; c.n = batch; c.local = u - first;
    c.W = unit_cost(C(batch), tile_first_unit(t + 1, tiles, units) - first);
    return c;
}

// Per-unit cost of the line work sequence v lies on.
template <class CostFn>
MLA_HD int64_t line_cost_of(int v, int units, int tiles, int batch, int V, CostFn C) {
    if (!tile_aligned(tiles, units)) return unit_cost(C(V), units);
    const int t = v / batch;
    return unit_cost(C(batch), tile_first_unit(t + 1, tiles, units) - tile_first_unit(t, tiles, units));
}

// Unit range record written into metadata[8 + 8u ..].
struct UnitRange {
    int v_begin, page_begin, v_end, page_end, chunk_begin;
};

// Count of i in [1, n] with C(i) <= target, for the two targets t0 <= t1 at once (two
// independent load chains per step). C is non-decreasing with C(0) = 0 <= t0, so this is
// the smallest v with C(v + 1) > target, or n when there is none.
template <class CostFn>
MLA_HD void count_le_pair(int64_t t0, int64_t t1, CostFn C, int n, int* c0, int* c1) {
    int step = 1;
    while (step * 2 <= n) step *= 2;
    int a = 0, b = 0;
    for (; n > 0 && step > 0; step >>= 1) {
        const bool ina = a + step <= n, inb = b + step <= n;
        const int64_t ca = ina ? (int64_t)C(a + step) : 0;
        const int64_t cb = inb ? (int64_t)C(b + step) : 0;
        if (ina && ca <= t0) a += step;
        if (inb && cb <= t1) b += step;
    }
    *c0 = a;
    *c1 = b;
}

// First page position >= target, as (v, page), given v = the smallest work sequence
// whose range [C[v] + overhead, C[v + 1]) ends after target (count_le_pair). Returns
// (V, 0) when no page lies at or after target.
template <class CostFn, class PagesFn>
MLA_HD void locate_from(int v, const int64_t target, CostFn C, PagesFn nblk, int V,
                        int overhead, int* v_out, int* k_out) {
    while (v < V && nblk(v) == 0) ++v;     // empty sequences own no page
    if (v >= V) { *v_out = V; *k_out = 0; return; }
    int64_t k = target - ((int64_t)C(v) + overhead);
    *v_out = v;
    *k_out = k < 0 ? 0 : (int)k;
}

// Unit u's run [(vb, kb), (ve, ke)) in (work sequence, page) order, and the chunk index
// of its first work sequence. C(v) over [0, V] and nblk(v) are the cost line's inputs.
template <class CostFn, class PagesFn>
MLA_HD void unit_range(int u, int units, int tiles, int batch, int V, int overhead, CostFn C,
                       PagesFn nblk, int* vb, int* kb, int* ve, int* ke, int* chunk) {
    const UnitCut c = cut_of_unit(u, units, tiles, batch, V, C);
    const int64_t base = C(c.v0);
    auto Cl = [&](int i) { return (int64_t)C(c.v0 + i) - base; };
    auto Pl = [&](int i) { return nblk(c.v0 + i); };
    const int64_t t0 = (int64_t)c.local * c.W, t1 = t0 + c.W;
    int b0, k0, b1, k1;
    count_le_pair(t0, t1, Cl, c.n, &b0, &b1);
    locate_from(b0, t0, Cl, Pl, c.n, overhead, &b0, &k0);
    locate_from(b1, t1, Cl, Pl, c.n, overhead, &b1, &k1);
    int ch = 0;
    if (b0 < c.n && (b0 != b1 || k0 != k1)) ch = c.local - unit_of(Cl(b0) + overhead, c.W);
    *vb = c.v0 + b0; *kb = k0; *ve = c.v0 + b1; *ke = k1; *chunk = ch;
}

// Chunks work sequence v is split into under the cut above.
template <class CostFn, class PagesFn>
MLA_HD int chunks_of_v(int v, int units, int tiles, int batch, int V, int overhead, CostFn C,
                       PagesFn nblk) {
    const int v0 = tile_aligned(tiles, units) ? (v / batch) * batch : 0;
    const int64_t W = line_cost_of(v, units, tiles, batch, V, C);
    return chunks_of((int64_t)C(v) - (int64_t)C(v0), nblk(v), W, overhead);
}

// The metadata header's unit cost: the largest per-unit cost of any line.
template <class CostFn>
MLA_HD int64_t header_unit_cost(int units, int tiles, int batch, int V, CostFn C) {
    if (!tile_aligned(tiles, units)) return unit_cost(C(V), units);
    int64_t w = 0;
    for (int t = 0; t < tiles; ++t) {
        const int64_t wt = line_cost_of(t * batch, units, tiles, batch, V, C);
        w = wt > w ? wt : w;
    }
    return w;
}

}  // namespace mla

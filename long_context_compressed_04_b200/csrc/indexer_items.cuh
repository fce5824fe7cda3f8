// Work items of the tensor-core lightning indexers (FP8 and MXFP4 keys): tiles of 128
// entries aligned to each query's sequence; query q owns the tiles [q * T, q * T + T) of a
// virtual tile space (T = tiles of the longest query); one persistent CTA per SM takes an
// equal contiguous range of that space and walks it as items, the pieces of the range cut
// at query boundaries and every 8 tiles.  The argument structs of both kernels carry the
// fields read here (seq_len, er, q_seq, q_pos, ent_rows, st, Q, B, m, max_n, qtiles,
// chunks_per_q).  With a block table (er.bt) the key rows of a tile come block by block
// (kPageRows entries each) and are checked there; row0 is then unused.
#pragma once

#include "common.cuh"

namespace csa {
namespace {

constexpr int kTileRows = 128;           // entries per tile (MMA M)
constexpr int kChunkTiles = 8;           // tiles per item at most
constexpr int kMaxItems = 64;            // work items per CTA resolved up front
constexpr int kPageRows = 32;            // entries per classical-cache block (128 tokens, m = 4)
constexpr int kTilePages = kTileRows / kPageRows;

struct Item {
    int q;
    int b;
    int n_vis;
    int tile0;
    int ntiles;
    int64_t row0;
};

// Virtual tile range [v0, v1) of CTA `cta` of `grid`; equal shares of Q * qtiles.
template <class A>
__device__ __forceinline__ void cta_range(const A& a, int cta, int grid, int64_t& v0,
                                          int64_t& v1) {
    const int64_t V = (int64_t)a.Q * a.qtiles;
    v0 = V * cta / grid;
    v1 = V * (cta + 1) / grid;
}

template <class A>
__device__ __forceinline__ int64_t chunk_of(const A& a, int64_t v) {
    const int64_t q = v / a.qtiles;
    return q * a.chunks_per_q + (v - q * a.qtiles) / kChunkTiles;
}

// Decodes item `ii` of the range [v0, v1) (the piece of the range inside its ii-th chunk);
// false when it has no tiles.  Every role calls this with the same arguments and so walks
// the same item sequence.
template <class A>
__device__ __forceinline__ bool get_item(const A& a, int64_t v0, int64_t v1, int ii,
                                         Item& x, bool report) {
    const int64_t g = chunk_of(a, v0) + ii;
    x.q = (int)(g / a.chunks_per_q);
    const int cq = (int)(g - (int64_t)x.q * a.chunks_per_q);
    const int64_t cbeg = (int64_t)x.q * a.qtiles + (int64_t)cq * kChunkTiles;
    const int64_t cend = min(cbeg + kChunkTiles, (int64_t)(x.q + 1) * a.qtiles);
    const int lo = (int)(max(v0, cbeg) - cbeg);
    const int hi = (int)(min(v1, cend) - cbeg);
    report = report && cq == 0 && lo == 0;   // one piece per query reports its errors
    const int b = a.q_seq[x.q];
    const int t = a.q_pos[x.q];
    if (b < 0 || b >= a.B || t < 0 || (int64_t)t >= a.seq_len[b]) {
        if (report) flag(a.st, CSA_DEV_OOB);
        return false;
    }
    int n = (t + 1) / a.m;
    if (n > a.max_n) {
        if (report) flag(a.st, CSA_DEV_CAPACITY);
        n = a.max_n;
    }
    x.b = b;
    if (a.er.bt) {
        x.row0 = 0;
    } else {
        x.row0 = a.er.ent_off[b];
        const int64_t avail = a.ent_rows - x.row0;
        if ((int64_t)n > avail) {
            if (report) flag(a.st, CSA_DEV_OOB);
            n = avail > 0 ? (int)avail : 0;
        }
    }
    x.n_vis = n;
    x.tile0 = cq * kChunkTiles + lo;
    const int tiles = (n + kTileRows - 1) / kTileRows;
    x.ntiles = min(cq * kChunkTiles + hi, tiles) - x.tile0;
    return x.ntiles > 0;
}

// Item ii of this CTA: from the table built at kernel start, or decoded directly past it.
template <class A>
__device__ __forceinline__ bool fetch_item(const A& a, const Item* items, int64_t v0,
                                           int64_t v1, int ii, Item& x, bool report) {
    if (ii < kMaxItems) {
        x = items[ii];
        return x.ntiles > 0;
    }
    return get_item(a, v0, v1, ii, x, report);
}

// Rows of the kTilePages blocks of virtual tile `tile` of item x (-1: not loaded, because it
// holds no visible entry or, flagged, its block lies outside the key store); returns the
// number of blocks to load.
template <class A>
__device__ __forceinline__ int tile_pages(const A& a, const Item& x, int tile,
                                          int32_t (&rows)[kTilePages]) {
    int n = 0;
#pragma unroll
    for (int p = 0; p < kTilePages; p++) {
        const int e = tile * kTileRows + p * kPageRows;
        rows[p] = -1;
        if (e >= x.n_vis) continue;
        const int64_t blk = a.er.bt[(int64_t)x.b * a.er.bt_stride + e / kPageRows];
        const int64_t r = blk * kPageRows;
        if (blk < 0 || r + kPageRows > a.ent_rows) {
            flag(a.st, CSA_DEV_OOB);
            continue;
        }
        rows[p] = (int32_t)r;
        n++;
    }
    return n;
}

}  // namespace
}  // namespace csa

// grouped_common.cuh -- tile scheduling shared by the grouped expert GEMMs.
//
// The permuted activation rows form G = E (+1 shared) groups: group g < E
// owns rows offsets[g] .. offsets[g+1]-1 (the contiguous per-expert interval
// of the routing stage), the shared expert owns rows T*k .. T*k+T-1.  A group
// of n rows has ceil(n / 128) m-tiles; every group has the same number of
// n-tiles.  Tiles are numbered group by group, and inside a group n-tile by
// n-tile with the m-tiles innermost, so CTAs that run at the same time share
// weight tiles through L2.  The host never learns the counts: each CTA
// rebuilds the m-tile prefix from `offsets` in its prologue.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kMaxGroups = 257;  // 256 routed + 1 shared

struct TileTable {
    int32_t goff[kMaxGroups + 1];     // first row of each group, goff[G] = end
    int32_t mstart[kMaxGroups + 1];   // prefix of m-tiles, mstart[G] = total
};

// Warp 0 fills the table (G = E + has_shared groups); the caller syncs.
__device__ __forceinline__ void build_tile_table(TileTable* tt, const int32_t* __restrict__ offsets,
                                                 int E, int T, int k, int has_shared, int BM) {
    const int lane = threadIdx.x & 31;
    const int G = E + has_shared;
    for (int g = lane; g <= E; g += 32) tt->goff[g] = offsets[g];
    if (has_shared && lane == 0) tt->goff[E + 1] = T * k + T;
    __syncwarp();
    // each lane scans a contiguous chunk of groups, then a warp scan of the sums
    const int per = (G + 31) / 32;
    const int g0 = lane * per, g1 = min(G, g0 + per);
    int sum = 0;
    for (int g = g0; g < g1; ++g) sum += (tt->goff[g + 1] - tt->goff[g] + BM - 1) / BM;
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int g = g0; g < g1; ++g) {
        tt->mstart[g] = run;
        run += (tt->goff[g + 1] - tt->goff[g] + BM - 1) / BM;
    }
    if (lane == 31) tt->mstart[G] = incl;
}

struct Tile {
    int g;       // group (E = shared expert)
    int row0;    // first permuted row of the tile
    int nrows;   // valid rows (<= BM)
    int n;       // n-tile index
};

__device__ __forceinline__ Tile decode_tile(const TileTable* tt, int G, int n_tiles, int tile,
                                            int BM) {
    int lo = 0, hi = G;  // largest g with mstart[g] * n_tiles <= tile
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tt->mstart[mid] * n_tiles <= tile) lo = mid; else hi = mid;
    }
    Tile t;
    t.g = lo;
    const int mt = tt->mstart[lo + 1] - tt->mstart[lo];
    const int local = tile - tt->mstart[lo] * n_tiles;
    t.n = local / mt;
    const int m = local - t.n * mt;
    t.row0 = tt->goff[lo] + m * BM;
    const int rows = tt->goff[lo + 1] - tt->goff[lo];
    t.nrows = min(BM, rows - m * BM);
    return t;
}

}  // namespace moe

// grouped_common.cuh -- tile scheduling shared by the grouped expert GEMMs.
//
// The permuted activation rows form G = E (+1 shared) groups: group g < E
// owns rows offsets[g] .. offsets[g+1]-1 (the contiguous per-expert interval
// of the routing stage), the shared expert owns rows T*k .. T*k+T-1.  A group
// of n rows has ceil(n / 128) m-tiles; every group has the same number of
// n-tiles.  Tiles are numbered group by group; inside a group, the m-tiles
// are taken in blocks of kMBlock, and each block runs n-tile by n-tile with
// its m-tiles innermost.  Tiles with neighbouring numbers therefore share a
// weight tile, and the rows of one block (a few MB) stay in L2 while they are
// read once per n-tile; a group of at most kMBlock m-tiles is one block.
// The host never learns the counts: each CTA rebuilds the m-tile prefix from
// `offsets` in its prologue.
//
// Tiles are handed out dynamically: the producer of each CTA takes the next
// number from a global counter when it is ready for a new tile and publishes
// it to the CTA's other roles through a small ring in shared memory.  Tiles
// that share a weight tile are therefore started at about the same time by
// whichever CTAs are free, and the second reader of a weight tile finds it
// in L2; a static round-robin order lets the CTAs drift apart over the waves
// until those second reads miss L2 and go to DRAM again.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kMaxGroups = 257;  // 256 routed + 1 shared
constexpr int kMBlock = 8;       // m-tiles per block of a large group

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
    const int blk = local / (kMBlock * n_tiles);      // block of m-tiles
    const int mb = min(kMBlock, mt - blk * kMBlock);  // m-tiles in this block
    const int r = local - blk * kMBlock * n_tiles;
    t.n = r / mb;
    const int m = blk * kMBlock + (r - t.n * mb);
    t.row0 = tt->goff[lo] + m * BM;
    const int rows = tt->goff[lo + 1] - tt->goff[lo];
    t.nrows = min(BM, rows - m * BM);
    return t;
}

// ---------------------------------------------------------------- tile ring
constexpr int kTileRing = 8;

struct TileRing {
    uint64_t full[kTileRing];   // producer published the slot (one arrival)
    uint64_t empty[kTileRing];  // every consumer read it
    int32_t tile[kTileRing];    // tile number, or -1 past the end
};

__device__ __forceinline__ void tile_ring_init(TileRing* r, uint32_t consumers) {
    for (int i = 0; i < kTileRing; ++i) {
        mbar_init(&r->full[i], 1);
        mbar_init(&r->empty[i], consumers);
    }
}

// Producer thread: takes the next tile number (its i-th) from the global
// counter and publishes it; returns it, or -1 past the last tile.  Sets
// `ok` false when the wait for a free slot runs out.
__device__ __forceinline__ int tile_ring_push(TileRing* r, uint32_t i, int32_t* counter, int total,
                                              uint64_t timeout_ns, const volatile int* abort,
                                              bool& ok) {
    const int slot = i % kTileRing;
    if (!mbar_wait(&r->empty[slot], ((i / kTileRing) & 1) ^ 1, timeout_ns, abort)) {
        ok = false;
        return -1;
    }
    int t = atomicAdd(counter, 1);
    if (t >= total) t = -1;
    *reinterpret_cast<volatile int32_t*>(&r->tile[slot]) = t;
    mbar_arrive(&r->full[slot]);  // release: the number is visible to the waiters
    return t;
}

// Consumer, one thread: the i-th tile number; the slot is released at once.
__device__ __forceinline__ int tile_ring_pop(TileRing* r, uint32_t i, uint64_t timeout_ns,
                                             const volatile int* abort, bool& ok) {
    const int slot = i % kTileRing;
    if (!mbar_wait(&r->full[slot], (i / kTileRing) & 1, timeout_ns, abort)) {
        ok = false;
        return -1;
    }
    const int t = *reinterpret_cast<volatile int32_t*>(&r->tile[slot]);
    mbar_arrive(&r->empty[slot]);
    return t;
}

// Consumer, a whole warp (one arrival for the warp): the i-th tile number.
__device__ __forceinline__ int tile_ring_pop_warp(TileRing* r, uint32_t i, uint64_t timeout_ns,
                                                  const volatile int* abort, bool& ok) {
    const int slot = i % kTileRing;
    if (!warp_wait(&r->full[slot], (i / kTileRing) & 1, timeout_ns, abort)) {
        ok = false;
        return -1;
    }
    const int t = *reinterpret_cast<volatile int32_t*>(&r->tile[slot]);
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&r->empty[slot]);
    return t;
}

}  // namespace moe

// Tile geometry of the copy engine, shared by host and device code so the CPU tests can check it.
//
// A segment of `len` bytes starting at address `src` is cut into tiles of at most `tile` bytes
// (a multiple of 16).
// When every destination agrees with the source modulo 16 ("congruent"), tile boundaries after
// the first lie on 16-byte boundaries of the source, and each tile splits into
//   head [lo, blo)   bytes before the first 16-byte boundary      (element-wise copy)
//   body [blo, bhi)  16-byte aligned, a multiple of 16 bytes       (one bulk copy)
//   tail [bhi, hi)   bytes after the last 16-byte boundary         (element-wise copy)
// Otherwise tiles are plain kTile slices copied element-wise. The three parts always tile
// [lo, hi) exactly, and the tiles tile [0, len) exactly.
#pragma once

#include <stddef.h>
#include <stdint.h>

#ifdef __CUDACC__
#define SIMCOMM_HD __host__ __device__ __forceinline__
#else
#define SIMCOMM_HD inline
#endif

namespace simcomm {

struct TileGeom {
    size_t lo, hi;    // byte range of the tile within the segment
    size_t blo, bhi;  // bulk part; blo == bhi when the tile has none
};

SIMCOMM_HD uint32_t tile_count(uint64_t src, size_t len, bool congruent, uint32_t tile) {
    if (len == 0) return 0;
    const size_t delta = congruent ? size_t(src & 15u) : 0;
    return uint32_t((len + delta + tile - 1) / tile);
}

SIMCOMM_HD TileGeom tile_geom(uint64_t src, size_t len, bool congruent, uint32_t k, uint32_t tile) {
    TileGeom g;
    if (!congruent) {
        g.lo = size_t(k) * tile;
        g.hi = (g.lo + tile < len) ? g.lo + tile : len;
        g.blo = g.bhi = g.hi;  // no bulk part: the head covers the tile
        return g;
    }
    const size_t delta = size_t(src & 15u);
    g.lo = (k == 0) ? 0 : size_t(k) * tile - delta;
    const size_t end = size_t(k + 1) * tile - delta;
    g.hi = end < len ? end : len;
    // first 16-byte boundary at or after lo, last one at or before hi (as offsets, no wrap-around)
    const size_t first = g.lo + ((16u - ((src + g.lo) & 15u)) & 15u);
    const size_t below = size_t((src + g.hi) & 15u);
    const size_t last = (g.hi >= below) ? g.hi - below : 0;
    if (first < last) {
        g.blo = first;
        g.bhi = last;
    } else {
        g.blo = g.bhi = g.hi;  // the tile sits inside one 16-byte window: all head
    }
    return g;
}

}  // namespace simcomm

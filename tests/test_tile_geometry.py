"""The copy engine's tile geometry (csrc/tile_geom.h), compiled for the host and brute-forced:
for every source offset modulo 16 and many lengths, the tiles cover the segment exactly, each
tile's head/body/tail cover the tile exactly, bodies are 16-byte aligned multiples of 16 bytes no
larger than a tile, and nothing wraps around (the p = 2, n = 2 All-to-All block at offset 4 that
once produced a wrapped-around bulk size is among the cases)."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "collective_communication_primitives_b200", "csrc")

PROGRAM = r'''
#include <cstdio>
#include <initializer_list>
#include "tile_geom.h"
using namespace simcomm;
static uint32_t kTile = 32768;
static int check(uint64_t src, size_t len, bool cong) {
    uint32_t n = tile_count(src, len, cong, kTile);
    if (len == 0) return n == 0 ? 0 : 1;
    size_t covered = 0;
    for (uint32_t k = 0; k < n; ++k) {
        TileGeom g = tile_geom(src, len, cong, k, kTile);
        if (g.lo != covered) return 2;
        if (!(g.lo < g.hi && g.hi <= len)) return 3;
        if (!(g.lo <= g.blo && g.blo <= g.bhi && g.bhi <= g.hi)) return 4;
        if (g.hi - g.lo > kTile) return 5;
        if (g.bhi > g.blo) {
            if (!cong) return 6;
            if (((src + g.blo) & 15) || ((g.bhi - g.blo) & 15)) return 7;
            if (g.bhi - g.blo > kTile) return 8;
        }
        if (cong && k > 0 && ((src + g.lo) & 15)) return 9;
        covered = g.hi;
    }
    return covered == len ? 0 : 10;
}
int main() {
  int bad = 0;
  for (uint32_t tsz : {16384u, 32768u, 65536u}) {
    kTile = tsz;
    const size_t lens[] = {1, 2, 3, 4, 6, 8, 12, 14, 15, 16, 17, 18, 30, 31, 32, 33, 46, 100,
                           kTile - 17, kTile - 16, kTile - 2, kTile - 1, kTile, kTile + 1, kTile + 2,
                           kTile + 14, kTile + 15, kTile + 16, 2 * kTile - 4, 2 * kTile, 3 * kTile + 6,
                           1000003, 4194304};
    for (uint64_t base : {0x7f0000000000ull, 0x7f0000000100ull})
        for (int off = 0; off < 16; off += 2)
            for (size_t len : lens)
                for (int c = 0; c < 2; ++c) {
                    int r = check(base + off, len, c == 1);
                    if (r) { std::printf("FAIL off=%d len=%zu cong=%d code=%d\n", off, len, c, r); ++bad; }
                }
    for (size_t len = 0; len < 200; len += 2)
        for (int off = 0; off < 16; off += 2)
            if (int r = check(0x1000 + off, len, true)) { std::printf("FAIL small off=%d len=%zu code=%d\n", off, len, r); ++bad; }
  }
    std::printf(bad ? "BAD\n" : "OK\n");
    return bad ? 1 : 0;
}
'''


def test_tile_geometry_brute_force(tmp_path):
    src = tmp_path / "geom.cpp"
    src.write_text(PROGRAM)
    exe = tmp_path / "geom"
    subprocess.run(["g++", "-std=c++17", "-O1", "-I", CSRC, "-o", str(exe), str(src)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True)
    assert res.returncode == 0, res.stdout[-3000:]
    assert res.stdout.strip().endswith("OK")

// The neighbour map's lookup structures (map_build.cu builds them): a
// direct-address table of int32 rows over batch * (grid + 2)^3 cells (each
// batch element's grid with a one-cell border that no voxel occupies, so all
// 27 neighbour cells of a voxel exist and lookups need no bounds test); a
// brick table over the same bordered cells (a directory of 8 x 4 x 2-cell
// bricks, x fastest, pointing at 64-cell row blocks for the occupied bricks
// only, -1 elsewhere: two dependent loads per lookup, no bounds test either);
// or an open-addressing hash table with linear probing -- compact 8-byte slots
// (key32 << 32 | row) when batch <= 4 and grid_dim <= 1024, else 64-bit keys
// with a separate int32 row array.  The home slot is 4 * h(key >> 2) + (key & 3)
// with a 32-bit avalanche mix h, so the x-neighbours of a voxel usually share a
// 32-byte sector.  Probe loops are bounded by the capacity.  Lookups read the
// tables with ld_dep(): the query kernel may start while the insert kernel
// still writes them.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "internal.h"

namespace subm3d {
namespace {

constexpr unsigned long long kEmpty = ~0ull;

__device__ __forceinline__ uint32_t mix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85ebca6bu;
  h ^= h >> 13;
  h *= 0xc2b2ae35u;
  h ^= h >> 16;
  return h;
}

__device__ __forceinline__ uint32_t mix64to32(unsigned long long k) {
  k ^= k >> 33;
  k *= 0xff51afd7ed558ccdull;
  k ^= k >> 33;
  k *= 0xc4ceb9fe1a85ec53ull;
  k ^= k >> 33;
  return static_cast<uint32_t>(k);
}

__device__ __forceinline__ uint32_t pack32(int b, int z, int y, int x) {
  return (static_cast<uint32_t>(b) << 30) | (static_cast<uint32_t>(z) << 20) |
         (static_cast<uint32_t>(y) << 10) | static_cast<uint32_t>(x);
}
__device__ __forceinline__ unsigned long long pack64(int b, int z, int y, int x) {
  return (static_cast<unsigned long long>(b) << 48) | (static_cast<unsigned long long>(z) << 32) |
         (static_cast<unsigned long long>(y) << 16) | static_cast<unsigned long long>(x);
}
__device__ __forceinline__ uint32_t home32(uint32_t key, uint32_t capmask) {
  return ((mix32(key >> 2) << 2) | (key & 3u)) & capmask;
}
__device__ __forceinline__ uint32_t home64(unsigned long long key, uint32_t capmask) {
  return ((mix64to32(key >> 2) << 2) | static_cast<uint32_t>(key & 3u)) & capmask;
}

__device__ __forceinline__ bool in_volume(int4 c, int grid, int batch) {
  return static_cast<unsigned>(c.x) < static_cast<unsigned>(batch) &&
         static_cast<unsigned>(c.y) < static_cast<unsigned>(grid) &&
         static_cast<unsigned>(c.z) < static_cast<unsigned>(grid) &&
         static_cast<unsigned>(c.w) < static_cast<unsigned>(grid);
}

// Cell of (b, z, y, x) in the bordered direct table: batch element b owns a
// block of (grid + 2)^3 cells and the voxel sits one cell in from its faces.
__device__ __forceinline__ int64_t cell_of(int b, int z, int y, int x, int grid) {
  const int64_t g = grid + 2;
  return ((static_cast<int64_t>(b) * g + (z + 1)) * g + (y + 1)) * g + (x + 1);
}

enum class Kind { kDirect, kCompact, kWide, kBrick };

struct Tables {
  const int32_t* cells;             // direct cells; brick: the pool of 64-cell blocks
  const unsigned long long* table;  // compact slots or wide keys
  const int32_t* rows;              // wide rows; brick: the directory
  uint32_t capmask;
  int32_t bgx, bgy, bgz;            // brick: bricks per bordered grid along x, y, z
};

// Brick of bordered cell (b, Z, Y, X) (Z = z + 1 ...) in the directory, and the
// cell's index inside its 64-cell block.
__device__ __forceinline__ int64_t brick_of(const Tables& t, int b, int Z, int Y, int X) {
  return ((static_cast<int64_t>(b) * t.bgz + (Z >> 1)) * t.bgy + (Y >> 2)) * t.bgx + (X >> 3);
}
__device__ __forceinline__ int brick_cell(int Z, int Y, int X) {
  return ((Z & 1) * 4 + (Y & 3)) * 8 + (X & 7);
}

template <Kind K>
__device__ __forceinline__ int32_t lookup(const Tables& t, int b, int z, int y, int x, int grid) {
  if constexpr (K == Kind::kDirect) {
    return ld_dep(t.cells + cell_of(b, z, y, x, grid));
  } else if constexpr (K == Kind::kBrick) {
    (void)grid;  // -1 <= z, y, x <= grid: every bordered cell has a directory entry
    const int32_t s = ld_dep(t.rows + brick_of(t, b, z + 1, y + 1, x + 1));
    return s < 0 ? -1
                 : ld_dep(t.cells + static_cast<int64_t>(s) * 64 + brick_cell(z + 1, y + 1, x + 1));
  } else if constexpr (K == Kind::kCompact) {
    const uint32_t key = pack32(b, z, y, x);
    uint32_t slot = home32(key, t.capmask);
    for (uint64_t step = 0; step <= t.capmask; ++step) {
      const unsigned long long e = ld_dep(t.table + slot);
      if (e == kEmpty) return -1;
      if (static_cast<uint32_t>(e >> 32) == key)
        return static_cast<int32_t>(static_cast<uint32_t>(e));
      slot = (slot + 1) & t.capmask;
    }
    return -1;
  } else {
    const unsigned long long key = pack64(b, z, y, x);
    uint32_t slot = home64(key, t.capmask);
    for (uint64_t step = 0; step <= t.capmask; ++step) {
      const unsigned long long e = ld_dep(t.table + slot);
      if (e == kEmpty) return -1;
      if (e == key) return ld_dep(t.rows + slot);
      slot = (slot + 1) & t.capmask;
    }
    return -1;
  }
}

}  // namespace
}  // namespace subm3d

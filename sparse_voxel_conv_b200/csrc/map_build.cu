// Neighbour-map build for the submanifold 3x3x3 convolution: a GPU hash table
// over packed (b, z, y, x) keys, then 27 probes per voxel.
//
// The pages build a "sorted-key indice map (27 lookups/voxel vectorised)"
// (lato.2_mrp_mlx, commit 97dcdfb54a message).  On the B200 the table is an
// open-addressing hash table with linear probing that stays resident in L2
// (8 MB at 330k voxels, 32 MB at 2.1M), built with 64-bit atomicCAS:
//
//   map_init    fills the table with EMPTY, zeroes the status word and the
//               per-tile offset masks (one grid-stride pass);
//   map_insert  one thread per voxel: 16-byte coordinate load, range check,
//               key pack, CAS into the first free slot of its probe sequence;
//               an equal key already present flags a duplicate;
//   map_query   one thread per (voxel, offset) pair, so the [N,27] int32 map is
//               written with fully coalesced stores; each thread probes one
//               neighbour key.  A block covers 32 voxels and ORs the offsets it
//               found into the mask word of its 128-row tile.
//
// Keys: with batch <= 4 and grid_dim <= 1024 a key is b:2|z:10|y:10|x:10 and a
// slot is the 8-byte word (key << 32 | row), so one CAS publishes key and row
// together and one load returns both.  Otherwise a key is b:16|z:16|y:16|x:16
// in a uint64 array with a separate int32 row array (rows are read only after
// the insert kernel has finished).
//
// Locality: the home slot of a key is 4 * h(key >> 2) + (key & 3), h a 32-bit
// avalanche mix, so the x-neighbours (dx = -1, 0, +1) of a voxel usually sit in
// the same 32-byte sector and the 27 probes of one voxel touch ~10 sectors.
//
// Every probe loop is bounded by the capacity; a full table sets kErrTableFull
// instead of spinning.
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

struct CompactKeys {
  using key_t = uint32_t;
  __device__ static key_t pack(int b, int z, int y, int x) {
    return (static_cast<uint32_t>(b) << 30) | (static_cast<uint32_t>(z) << 20) |
           (static_cast<uint32_t>(y) << 10) | static_cast<uint32_t>(x);
  }
  __device__ static uint32_t home(key_t key, uint32_t capmask) {
    return ((mix32(key >> 2) << 2) | (key & 3u)) & capmask;
  }
};

struct WideKeys {
  using key_t = unsigned long long;
  __device__ static key_t pack(int b, int z, int y, int x) {
    return (static_cast<unsigned long long>(b) << 48) |
           (static_cast<unsigned long long>(z) << 32) |
           (static_cast<unsigned long long>(y) << 16) | static_cast<unsigned long long>(x);
  }
  __device__ static uint32_t home(key_t key, uint32_t capmask) {
    return ((mix64to32(key >> 2) << 2) | static_cast<uint32_t>(key & 3u)) & capmask;
  }
};

__global__ void map_init(uint4* table, size_t table_words16, uint32_t* head, size_t head_words) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t t0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint4 ones = make_uint4(~0u, ~0u, ~0u, ~0u);
  for (size_t t = t0; t < table_words16; t += stride) table[t] = ones;
  for (size_t t = t0; t < head_words; t += stride) head[t] = 0u;
}

__device__ __forceinline__ bool in_volume(int4 c, int grid, int batch) {
  return static_cast<unsigned>(c.x) < static_cast<unsigned>(batch) &&
         static_cast<unsigned>(c.y) < static_cast<unsigned>(grid) &&
         static_cast<unsigned>(c.z) < static_cast<unsigned>(grid) &&
         static_cast<unsigned>(c.w) < static_cast<unsigned>(grid);
}

__global__ void map_insert_compact(const int4* __restrict__ coords, int64_t n, int grid, int batch,
                                   unsigned long long* __restrict__ table, uint32_t capmask,
                                   uint32_t* status) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int4 c = __ldg(coords + i);
  if (!in_volume(c, grid, batch)) {
    atomicOr(status, kErrRange);
    return;
  }
  const uint32_t key = CompactKeys::pack(c.x, c.y, c.z, c.w);
  const unsigned long long entry =
      (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(i);
  uint32_t slot = CompactKeys::home(key, capmask);
  for (uint64_t step = 0; step <= capmask; ++step) {
    const unsigned long long prev = atomicCAS(table + slot, kEmpty, entry);
    if (prev == kEmpty) return;
    if (static_cast<uint32_t>(prev >> 32) == key) {
      atomicOr(status, kErrDuplicate);
      return;
    }
    slot = (slot + 1) & capmask;
  }
  atomicOr(status, kErrTableFull);
}

__global__ void map_insert_wide(const int4* __restrict__ coords, int64_t n, int grid, int batch,
                                unsigned long long* __restrict__ keys, int32_t* __restrict__ rows,
                                uint32_t capmask, uint32_t* status) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int4 c = __ldg(coords + i);
  if (!in_volume(c, grid, batch)) {
    atomicOr(status, kErrRange);
    return;
  }
  const unsigned long long key = WideKeys::pack(c.x, c.y, c.z, c.w);
  uint32_t slot = WideKeys::home(key, capmask);
  for (uint64_t step = 0; step <= capmask; ++step) {
    const unsigned long long prev = atomicCAS(keys + slot, kEmpty, key);
    if (prev == kEmpty) {
      rows[slot] = static_cast<int32_t>(i);
      return;
    }
    if (prev == key) {
      atomicOr(status, kErrDuplicate);
      return;
    }
    slot = (slot + 1) & capmask;
  }
  atomicOr(status, kErrTableFull);
}

constexpr int kQueryVoxels = 32;                     // voxels per query block
constexpr int kQueryThreads = kQueryVoxels * kKvol;  // 864

template <bool kCompact>
__global__ void __launch_bounds__(kQueryThreads)
    map_query(const int4* __restrict__ coords, int64_t n, int grid,
              const unsigned long long* __restrict__ table, const int32_t* __restrict__ rows,
              uint32_t capmask, int32_t* __restrict__ nbr, uint32_t* __restrict__ tile_mask) {
  __shared__ uint32_t s_mask;
  if (threadIdx.x == 0) s_mask = 0u;
  __syncthreads();
  const int local = threadIdx.x / kKvol;
  const int k = threadIdx.x - local * kKvol;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kQueryVoxels + local;
  uint32_t bits = 0u;
  if (i < n) {
    int32_t found = -1;
    if (k == 13) {
      found = static_cast<int32_t>(i);  // the centre offset is the voxel itself
    } else {
      const int4 c = __ldg(coords + i);
      const int z = c.y + (k / 9) - 1;
      const int y = c.z + (k / 3) % 3 - 1;
      const int x = c.w + k % 3 - 1;
      if (static_cast<unsigned>(z) < static_cast<unsigned>(grid) &&
          static_cast<unsigned>(y) < static_cast<unsigned>(grid) &&
          static_cast<unsigned>(x) < static_cast<unsigned>(grid)) {
        if constexpr (kCompact) {
          const uint32_t key = CompactKeys::pack(c.x, z, y, x);
          uint32_t slot = CompactKeys::home(key, capmask);
          for (uint64_t step = 0; step <= capmask; ++step) {
            const unsigned long long e = table[slot];
            if (e == kEmpty) break;
            if (static_cast<uint32_t>(e >> 32) == key) {
              found = static_cast<int32_t>(static_cast<uint32_t>(e));
              break;
            }
            slot = (slot + 1) & capmask;
          }
        } else {
          const unsigned long long key = WideKeys::pack(c.x, z, y, x);
          uint32_t slot = WideKeys::home(key, capmask);
          for (uint64_t step = 0; step <= capmask; ++step) {
            const unsigned long long e = table[slot];
            if (e == kEmpty) break;
            if (e == key) {
              found = rows[slot];
              break;
            }
            slot = (slot + 1) & capmask;
          }
        }
      }
    }
    nbr[static_cast<int64_t>(blockIdx.x) * kQueryThreads + threadIdx.x] = found;
    bits = found >= 0 ? (1u << k) : 0u;
  }
  // one shared atomic per warp instead of one per thread
  bits = __reduce_or_sync(0xFFFFFFFFu, bits);
  if ((threadIdx.x & 31) == 0 && bits != 0u) atomicOr(&s_mask, bits);
  __syncthreads();
  if (threadIdx.x == 0 && s_mask != 0u) {
    atomicOr(tile_mask + (static_cast<int64_t>(blockIdx.x) * kQueryVoxels) / kTileRows, s_mask);
  }
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

bool map_layout(int64_t n, int32_t grid_dim, int32_t batch, uint64_t forced_capacity,
                MapLayout* out) {
  if (n < 0 || n >= 0x7FFFFFFFll || grid_dim < 1 || grid_dim > 65535 || batch < 1 ||
      batch > 65535)
    return false;
  MapLayout lay;
  lay.compact = (batch <= 4 && grid_dim <= 1024);
  uint64_t cap = 1024;
  while (cap < 2ull * static_cast<uint64_t>(n)) cap <<= 1;
  if (forced_capacity != 0 && forced_capacity < cap) {
    cap = 4;
    while (cap < forced_capacity) cap <<= 1;
  }
  lay.capacity = cap;
  lay.n_tiles = (n + kTileRows - 1) / kTileRows;
  lay.status_off = 0;
  lay.mask_off = 256;
  lay.table_off = align_up(lay.mask_off + static_cast<size_t>(lay.n_tiles) * 4, 256);
  lay.rows_off = align_up(lay.table_off + cap * 8, 256);
  lay.total = lay.compact ? lay.rows_off : align_up(lay.rows_off + cap * 4, 256);
  *out = lay;
  return true;
}

cudaError_t launch_map_build(const int32_t* coords, int64_t n, int32_t grid_dim, int32_t batch,
                             int32_t* nbr, void* workspace, const MapLayout& lay,
                             cudaStream_t stream) {
  auto* ws = static_cast<uint8_t*>(workspace);
  auto* status = reinterpret_cast<uint32_t*>(ws + lay.status_off);
  auto* mask = reinterpret_cast<uint32_t*>(ws + lay.mask_off);
  auto* table = reinterpret_cast<unsigned long long*>(ws + lay.table_off);
  auto* rows = reinterpret_cast<int32_t*>(ws + lay.rows_off);
  const uint32_t capmask = static_cast<uint32_t>(lay.capacity - 1);
  // head = status word (+ padding) and the mask words, all cleared to zero
  const size_t head_words = (lay.table_off - lay.status_off) / 4;
  const size_t table_words16 = lay.capacity * 8 / 16;
  {
    const size_t work = table_words16 > head_words ? table_words16 : head_words;
    size_t blocks = (work + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    map_init<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(reinterpret_cast<uint4*>(table),
                                                               table_words16, status, head_words);
  }
  if (n == 0) return cudaGetLastError();
  const auto* c4 = reinterpret_cast<const int4*>(coords);
  const unsigned ins_blocks = static_cast<unsigned>((n + 255) / 256);
  const unsigned q_blocks = static_cast<unsigned>((n + kQueryVoxels - 1) / kQueryVoxels);
  if (lay.compact) {
    map_insert_compact<<<ins_blocks, 256, 0, stream>>>(c4, n, grid_dim, batch, table, capmask,
                                                       status);
    map_query<true><<<q_blocks, kQueryThreads, 0, stream>>>(c4, n, grid_dim, table, nullptr,
                                                            capmask, nbr, mask);
  } else {
    map_insert_wide<<<ins_blocks, 256, 0, stream>>>(c4, n, grid_dim, batch, table, rows, capmask,
                                                    status);
    map_query<false><<<q_blocks, kQueryThreads, 0, stream>>>(c4, n, grid_dim, table, rows,
                                                             capmask, nbr, mask);
  }
  return cudaGetLastError();
}

}  // namespace subm3d

// Neighbour-map build for the submanifold 3x3x3 convolution.
//
// The pages build a "sorted-key indice map (27 lookups/voxel vectorised)"
// (lato.2_mrp_mlx, commit 97dcdfb54a message).  Here the lookup structure is
// one of two GPU tables over packed (b, z, y, x) keys, chosen per call:
//
//   direct  when batch * grid_dim^3 int32 cells fit in 64 MB (every 128^3
//           volume): cell -> row, -1 when empty.  A collision-free perfect
//           hash: insert is one plain store per voxel, a lookup is one load,
//           and voxels adjacent in raster order look up adjacent cells, so the
//           27 lookups of a warp coalesce.  A duplicate coordinate leaves one
//           of its rows in the cell; the other row sees a foreign row at its
//           own centre offset and raises the duplicate flag.
//   hash    otherwise: open addressing with linear probing, capacity a power
//           of two >= 2N.  With batch <= 4 and grid_dim <= 1024 a key is
//           b:2|z:10|y:10|x:10 and a slot the 8-byte word (key << 32 | row),
//           published by one 64-bit CAS; else a key is b:16|z:16|y:16|x:16 in
//           a uint64 array with a separate int32 row array.  The home slot is
//           4 * h(key >> 2) + (key & 3), h a 32-bit avalanche mix, so the
//           x-neighbours of a voxel usually share a 32-byte sector.  Probe
//           loops are bounded by the capacity; a full table raises a flag.
//
// Kernels: map_init (table <- empty, status <- 0), map_insert (one thread per
// voxel: 16-byte coordinate load, range check, insert), map_query (one block
// per 128-row tile, one thread per voxel: 27 lookups into shared memory, then
// the [128, 27] block and the tile's offset mask are written with coalesced
// stores; no atomics on the output).
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

__device__ __forceinline__ int64_t cell_of(int b, int z, int y, int x, int grid) {
  return ((static_cast<int64_t>(b) * grid + z) * grid + y) * grid + x;
}

// Fills two regions (`words16a`, `words16b` 16-byte words) with all-ones --
// the lookup table and the position table -- and zeroes the status word.
__global__ void map_init(uint4* a, size_t words16a, uint4* b, size_t words16b, uint32_t* status) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t t0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint4 ones = make_uint4(~0u, ~0u, ~0u, ~0u);
  for (size_t t = t0; t < words16a; t += stride) a[t] = ones;
  for (size_t t = t0; t < words16b; t += stride) b[t] = ones;
  if (t0 == 0) *status = 0u;
}

__global__ void map_insert_direct(const int4* __restrict__ coords, int64_t n, int grid, int batch,
                                  int32_t* __restrict__ cells, uint32_t* status) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int4 c = __ldg(coords + i);
  if (!in_volume(c, grid, batch)) {
    atomicOr(status, kErrRange);
    return;
  }
  cells[cell_of(c.x, c.y, c.z, c.w, grid)] = static_cast<int32_t>(i);
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
  const uint32_t key = pack32(c.x, c.y, c.z, c.w);
  const unsigned long long entry =
      (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(i);
  uint32_t slot = home32(key, capmask);
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
  const unsigned long long key = pack64(c.x, c.y, c.z, c.w);
  uint32_t slot = home64(key, capmask);
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

enum class Kind { kDirect, kCompact, kWide };

struct Tables {
  const int32_t* cells;             // direct
  const unsigned long long* table;  // compact slots or wide keys
  const int32_t* rows;              // wide rows
  uint32_t capmask;
};

template <Kind K>
__device__ __forceinline__ int32_t lookup(const Tables& t, int b, int z, int y, int x, int grid) {
  if constexpr (K == Kind::kDirect) {
    return __ldg(t.cells + cell_of(b, z, y, x, grid));
  } else if constexpr (K == Kind::kCompact) {
    const uint32_t key = pack32(b, z, y, x);
    uint32_t slot = home32(key, t.capmask);
    for (uint64_t step = 0; step <= t.capmask; ++step) {
      const unsigned long long e = __ldg(t.table + slot);
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
      const unsigned long long e = __ldg(t.table + slot);
      if (e == kEmpty) return -1;
      if (e == key) return __ldg(t.rows + slot);
      slot = (slot + 1) & t.capmask;
    }
    return -1;
  }
}

template <Kind K>
__global__ void __launch_bounds__(kTileRows)
    map_query(const int4* __restrict__ coords, int64_t n, int grid, int batch, Tables t,
              int32_t* __restrict__ nbr, uint32_t* __restrict__ tile_mask, uint32_t* status) {
  __shared__ __align__(16) int32_t s_nbr[kTileRows * kKvol];
  __shared__ uint32_t s_bits[kTileRows / 32];
  const int r = threadIdx.x;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kTileRows;
  const int64_t i = row0 + r;
  uint32_t bits = 0u;
  if (i < n) {
    const int4 c = __ldg(coords + i);
    if (in_volume(c, grid, batch)) {
#pragma unroll
      for (int k = 0; k < kKvol; ++k) {
        const int z = c.y + k / 9 - 1;
        const int y = c.z + (k / 3) % 3 - 1;
        const int x = c.w + k % 3 - 1;
        int32_t found = -1;
        if (static_cast<unsigned>(z) < static_cast<unsigned>(grid) &&
            static_cast<unsigned>(y) < static_cast<unsigned>(grid) &&
            static_cast<unsigned>(x) < static_cast<unsigned>(grid))
          found = lookup<K>(t, c.x, z, y, x, grid);
        s_nbr[r * kKvol + k] = found;
        bits |= (found >= 0 ? 1u : 0u) << k;
      }
      if (K == Kind::kDirect && s_nbr[r * kKvol + 13] != static_cast<int32_t>(i))
        atomicOr(status, kErrDuplicate);  // another row owns this voxel's cell
    } else {
#pragma unroll
      for (int k = 0; k < kKvol; ++k) s_nbr[r * kKvol + k] = -1;
    }
  }
  bits = __reduce_or_sync(0xFFFFFFFFu, bits);
  if ((r & 31) == 0) s_bits[r >> 5] = bits;
  __syncthreads();
  if (r == 0) tile_mask[blockIdx.x] = s_bits[0] | s_bits[1] | s_bits[2] | s_bits[3];
  const int rows = static_cast<int>(n - row0 < kTileRows ? n - row0 : kTileRows);
  int32_t* dst = nbr + row0 * kKvol;
  if (rows == kTileRows) {
    // 13824 bytes = 864 16-byte words; each tile's nbr block starts 16-byte aligned
    const int4* src4 = reinterpret_cast<const int4*>(s_nbr);
    int4* dst4 = reinterpret_cast<int4*>(dst);
    for (int e = r; e < kTileRows * kKvol / 4; e += kTileRows) dst4[e] = src4[e];
  } else {
    for (int e = r; e < rows * kKvol; e += kTileRows) dst[e] = s_nbr[e];
  }
}

// ----------------------------------------------------------- run layout ----
// A voxel starts a run unless the previous row is its x-1 neighbour (same b, z,
// y and x one less).

__device__ __forceinline__ bool run_start(const int4* coords, int64_t v) {
  if (v == 0) return true;
  const int4 p = __ldg(coords + v - 1);
  const int4 c = __ldg(coords + v);
  return !(p.x == c.x && p.y == c.y && p.z == c.z && p.w + 1 == c.w);
}

// Run starts per block of kRunBlock rows.
__global__ void __launch_bounds__(256) map_run_count(const int4* __restrict__ coords, int64_t n,
                                                     int32_t* __restrict__ cnt) {
  __shared__ int32_t s_sum[8];
  int32_t c = 0;
  for (int i = 0; i < kRunBlock / 256; ++i) {
    const int64_t v = static_cast<int64_t>(blockIdx.x) * kRunBlock + i * 256 + threadIdx.x;
    if (v < n && run_start(coords, v)) ++c;
  }
  c = __reduce_add_sync(0xFFFFFFFFu, c);
  if ((threadIdx.x & 31) == 0) s_sum[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t t = 0;
    for (int w = 0; w < 8; ++w) t += s_sum[w];
    cnt[blockIdx.x] = t;
  }
}

// Exclusive scan of the per-block run counts (one block), and the header:
// hdr[0] = runs, hdr[1] = position tiles, hdr[2] = positions.
__global__ void __launch_bounds__(1024) map_run_scan(int32_t* __restrict__ cnt, int64_t n_blocks,
                                                     int64_t n, int32_t* __restrict__ hdr) {
  __shared__ int32_t s_warp[32];
  __shared__ int64_t s_carry;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t base = 0; base < n_blocks; base += 1024) {
    const int64_t i = base + threadIdx.x;
    const int32_t x = i < n_blocks ? cnt[i] : 0;
    int32_t incl = x;
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int32_t w = s_warp[lane];
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t y = __shfl_up_sync(0xFFFFFFFFu, w, d);
        if (lane >= d) w += y;
      }
      s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int32_t before = (warp > 0 ? s_warp[warp - 1] : 0) + incl - x;
    const int64_t carry = s_carry;
    if (i < n_blocks) cnt[i] = static_cast<int32_t>(carry + before);
    __syncthreads();
    if (threadIdx.x == 0) s_carry = carry + s_warp[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int64_t runs = s_carry;
    const int64_t positions = n + 2 * runs;
    hdr[0] = static_cast<int32_t>(runs);
    hdr[1] = static_cast<int32_t>((positions + kPosTile - 1) / kPosTile);
    hdr[2] = static_cast<int32_t>(positions);
    hdr[3] = 0;
  }
}

// Places every voxel v at position v + 2 R(v), R(v) = run starts among rows
// 0..v, with the left-pad slot before a run's first voxel and the right-pad
// slot after its last.  Each thread handles 4 consecutive rows.
__global__ void __launch_bounds__(256) map_run_place(const int4* __restrict__ coords, int64_t n,
                                                     const int32_t* __restrict__ blk_off,
                                                     int32_t* __restrict__ pos) {
  __shared__ int32_t s_warp[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * kRunBlock + 4 * threadIdx.x;
  bool rs[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) rs[i] = (v0 + i < n) ? run_start(coords, v0 + i) : true;
  int32_t local = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) local += (v0 + i < n && rs[i]) ? 1 : 0;
  int32_t incl = local;
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int32_t warp_before = 0;
  for (int w = 0; w < warp; ++w) warp_before += s_warp[w];
  int64_t r = blk_off[blockIdx.x] + warp_before + incl - local;  // run starts before v0
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t v = v0 + i;
    if (v >= n) break;
    if (rs[i]) ++r;
    const int64_t p = v + 2 * r;
    pos[p] = static_cast<int32_t>(v * 4 + kPosVoxel);
    if (rs[i]) pos[p - 1] = static_cast<int32_t>(v * 4 + kPosLeftPad);
    if (v + 1 == n || rs[i + 1]) pos[p + 1] = static_cast<int32_t>(v * 4 + kPosRightPad);
  }
}

// E index table: for position tile t and offset pair (dz, dy), entry i is the
// feature row of E row i-1: a voxel position takes its (dz, dy, 0) neighbour,
// a left pad its voxel's (dz, dy, -1) neighbour, a right pad the (dz, dy, +1)
// one; entry 0 (row -1) and entry 257 (row 256) are the (dz, dy, -1) and
// (dz, dy, +1) neighbours of the voxels at positions 0 and 255.  So for the
// voxel at position p, E rows p-1, p, p+1 hold its dx = -1, 0, +1 neighbours.
__global__ void __launch_bounds__(kEtStride) map_etable(const int32_t* __restrict__ pos,
                                                         const int32_t* __restrict__ nbr,
                                                         const int32_t* __restrict__ hdr,
                                                         int32_t* __restrict__ et) {
  const int64_t t = blockIdx.x;
  if (t >= hdr[1]) return;
  const int i = threadIdx.x;  // 0 .. kEtStride-1
  int64_t v = -1;
  int dx = 0;
  if (i == 0 || i == 257) {
    const int32_t e = pos[t * kPosTile + (i == 0 ? 0 : kPosTile - 1)];
    if (e >= 0 && (e & 3) == kPosVoxel) {
      v = e >> 2;
      dx = i == 0 ? -1 : 1;
    }
  } else if (i < 257) {
    const int32_t e = pos[t * kPosTile + i - 1];
    if (e >= 0) {
      v = e >> 2;
      dx = (e & 3) == kPosLeftPad ? -1 : ((e & 3) == kPosRightPad ? 1 : 0);
    }
  }
#pragma unroll
  for (int dzdy = 0; dzdy < 9; ++dzdy)
    et[(t * 9 + dzdy) * kEtStride + i] = v >= 0 ? __ldg(nbr + v * kKvol + 3 * dzdy + dx + 1) : -1;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

bool map_layout(int64_t n, int32_t grid_dim, int32_t batch, const MapOptions& opt,
                MapLayout* out) {
  if (n < 0 || n >= 0x7FFFFFFFll || grid_dim < 1 || grid_dim > 65535 || batch < 1 ||
      batch > 65535)
    return false;
  MapLayout lay;
  const double cells = static_cast<double>(batch) * grid_dim * grid_dim * grid_dim;
  const bool direct_fits = cells * 4.0 <= static_cast<double>(kDirectTableMaxBytes);
  lay.kind = (direct_fits && !opt.force_hash && opt.forced_capacity == 0) ? MapKind::kDirect
                                                                         : MapKind::kHash;
  lay.compact = (batch <= 4 && grid_dim <= 1024);
  uint64_t cap = 1024;
  while (cap < 2ull * static_cast<uint64_t>(n)) cap <<= 1;
  if (opt.forced_capacity != 0 && opt.forced_capacity < cap) {
    cap = 4;
    while (cap < opt.forced_capacity) cap <<= 1;
  }
  lay.capacity = cap;
  lay.cells = direct_fits ? static_cast<uint64_t>(cells) : 0;
  lay.n_tiles = (n + kTileRows - 1) / kTileRows;
  lay.status_off = 0;
  lay.mask_off = 256;
  lay.table_off = align_up(lay.mask_off + static_cast<size_t>(lay.n_tiles) * 4, 256);
  size_t end = 0;
  if (lay.kind == MapKind::kDirect) {
    lay.table_bytes = align_up(lay.cells * 4, 256);
    lay.rows_off = lay.table_off + lay.table_bytes;
    end = lay.rows_off;
  } else {
    lay.table_bytes = cap * 8;
    lay.rows_off = align_up(lay.table_off + lay.table_bytes, 256);
    end = lay.compact ? lay.rows_off : align_up(lay.rows_off + cap * 4, 256);
  }
  if (!opt.run_layout) {  // nbr and tile masks only
    lay.runcnt_off = lay.hdr_off = lay.pos_off = lay.et_off = end;
    lay.total = end;
    *out = lay;
    return true;
  }
  lay.n_run_blocks = (n + kRunBlock - 1) / kRunBlock;
  lay.pos_max = static_cast<int64_t>(align_up(static_cast<size_t>(3 * n), kPosTile)) + kPosTile;
  lay.ptile_max = lay.pos_max / kPosTile;
  lay.runcnt_off = end;
  lay.hdr_off = align_up(lay.runcnt_off + static_cast<size_t>(lay.n_run_blocks) * 4, 256);
  lay.pos_off = lay.hdr_off + 256;
  lay.pos_bytes = static_cast<size_t>(lay.pos_max) * 4;
  lay.et_off = align_up(lay.pos_off + lay.pos_bytes, 256);
  lay.total = align_up(lay.et_off + static_cast<size_t>(lay.ptile_max) * 9 * kEtStride * 4, 256);
  *out = lay;
  return true;
}

cudaError_t launch_map_build(const int32_t* coords, int64_t n, int32_t grid_dim, int32_t batch,
                             int32_t* nbr, void* workspace, const MapLayout& lay,
                             cudaStream_t stream) {
  auto* ws = static_cast<uint8_t*>(workspace);
  auto* status = reinterpret_cast<uint32_t*>(ws + lay.status_off);
  auto* mask = reinterpret_cast<uint32_t*>(ws + lay.mask_off);
  auto* table = ws + lay.table_off;
  const size_t words16 = lay.table_bytes / 16;
  const size_t pos_words16 = lay.pos_bytes / 16;
  auto* pos = reinterpret_cast<int32_t*>(ws + lay.pos_off);
  {
    const size_t work = words16 > pos_words16 ? words16 : pos_words16;
    size_t blocks = (work + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks == 0) blocks = 1;
    map_init<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        reinterpret_cast<uint4*>(table), words16, reinterpret_cast<uint4*>(pos), pos_words16,
        status);
  }
  if (n == 0) return cudaGetLastError();
  const auto* c4 = reinterpret_cast<const int4*>(coords);
  const unsigned ins_blocks = static_cast<unsigned>((n + 255) / 256);
  const unsigned q_blocks = static_cast<unsigned>(lay.n_tiles);
  Tables t{};
  t.capmask = static_cast<uint32_t>(lay.capacity - 1);
  if (lay.kind == MapKind::kDirect) {
    t.cells = reinterpret_cast<const int32_t*>(table);
    map_insert_direct<<<ins_blocks, 256, 0, stream>>>(c4, n, grid_dim, batch,
                                                      reinterpret_cast<int32_t*>(table), status);
    map_query<Kind::kDirect><<<q_blocks, kTileRows, 0, stream>>>(c4, n, grid_dim, batch, t, nbr,
                                                                 mask, status);
  } else if (lay.compact) {
    t.table = reinterpret_cast<const unsigned long long*>(table);
    map_insert_compact<<<ins_blocks, 256, 0, stream>>>(
        c4, n, grid_dim, batch, reinterpret_cast<unsigned long long*>(table), t.capmask, status);
    map_query<Kind::kCompact><<<q_blocks, kTileRows, 0, stream>>>(c4, n, grid_dim, batch, t, nbr,
                                                                  mask, status);
  } else {
    auto* rows = reinterpret_cast<int32_t*>(ws + lay.rows_off);
    t.table = reinterpret_cast<const unsigned long long*>(table);
    t.rows = rows;
    map_insert_wide<<<ins_blocks, 256, 0, stream>>>(c4, n, grid_dim, batch,
                                                    reinterpret_cast<unsigned long long*>(table),
                                                    rows, t.capmask, status);
    map_query<Kind::kWide><<<q_blocks, kTileRows, 0, stream>>>(c4, n, grid_dim, batch, t, nbr,
                                                               mask, status);
  }
  if (lay.ptile_max == 0) return cudaGetLastError();
  // x-run position layout and E index table for the run-padded forward
  auto* runcnt = reinterpret_cast<int32_t*>(ws + lay.runcnt_off);
  auto* hdr = reinterpret_cast<int32_t*>(ws + lay.hdr_off);
  auto* et = reinterpret_cast<int32_t*>(ws + lay.et_off);
  const unsigned rblocks = static_cast<unsigned>(lay.n_run_blocks);
  map_run_count<<<rblocks, 256, 0, stream>>>(c4, n, runcnt);
  map_run_scan<<<1, 1024, 0, stream>>>(runcnt, lay.n_run_blocks, n, hdr);
  map_run_place<<<rblocks, 256, 0, stream>>>(c4, n, runcnt, pos);
  map_etable<<<static_cast<unsigned>(lay.ptile_max), kEtStride, 0, stream>>>(pos, nbr, hdr, et);
  return cudaGetLastError();
}

}  // namespace subm3d

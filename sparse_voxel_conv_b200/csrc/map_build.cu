// Neighbour-map build for the submanifold 3x3x3 convolution.
//
// The pages build a "sorted-key indice map (27 lookups/voxel vectorised)"
// (lato.2_mrp_mlx, commit 97dcdfb54a message).  Here the lookup structure is
// one of two GPU tables over packed (b, z, y, x) keys, chosen per call:
//
//   direct  when batch * grid_dim^3 int32 cells take at most max(64 MB,
//           256 B x N) and 2^28 cells (every 128^3 volume; 4 x 256^3 from
//           about a million voxels): cell -> row, -1 when empty.  A collision-free perfect
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
// stores; no atomics on the output; and the tile's share of the x-run layout).
#include <cuda_runtime.h>

#include <algorithm>

#include "internal.h"
#include "map_table.cuh"

namespace subm3d {
namespace {

// Fills the lookup table (`words16a` 16-byte words) with all-ones, zeroes the
// run layout's superblock sums (`words16z` words), the status word and the
// run layout's header (when there is one).
__global__ void map_init(uint4* a, size_t words16a, uint4* z, size_t words16z, uint32_t* status,
                         int32_t* hdr) {
  pdl_wait();
  pdl_trigger();
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t t0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint4 ones = make_uint4(~0u, ~0u, ~0u, ~0u);
  for (size_t t = t0; t < words16a; t += stride) a[t] = ones;
  for (size_t t = t0; t < words16z; t += stride) z[t] = make_uint4(0u, 0u, 0u, 0u);
  if (t0 == 0) {
    *status = 0u;
    if (hdr)
      for (int k = 0; k < 4; ++k) hdr[k] = 0;
  }
}

// ----------------------------------------------------- run-start counts ----
// A voxel starts a run unless the previous row is its x-1 neighbour (same b, z,
// y and x one less).  The insert kernels (256 rows per block = two 128-row
// tiles) count run starts per tile and add the block's total to its superblock
// (128 tiles) sum; the query tile then finds the run starts before it by
// summing the superblock sums before its superblock and the tile counts before
// it within its superblock -- at most N / 16384 + 127 loads, no waits.

constexpr int kInsertThreads = 2 * kTileRows;
constexpr int kSuperTiles = 128;

struct RunCount {
  int32_t* cnt;  // [n_tiles] run starts per 128-row tile (nullptr: no run layout)
  int32_t* sb;   // [ceil(n_tiles / 128)] run starts per superblock, zeroed by map_init
};

__device__ __forceinline__ bool x_next(int4 a, int4 b) {  // b is a's x+1 neighbour
  return a.x == b.x && a.y == b.y && a.z == b.z && a.w + 1 == b.w;
}

// Called by all kInsertThreads threads of an insert block; c = coords[i] for i < n.
__device__ __forceinline__ void count_run_starts(const int4* __restrict__ coords, int64_t n,
                                                 int64_t i, int4 c, const RunCount& rc) {
  __shared__ int32_t s_cnt[kInsertThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int4 prev;
  prev.x = __shfl_up_sync(0xFFFFFFFFu, c.x, 1);
  prev.y = __shfl_up_sync(0xFFFFFFFFu, c.y, 1);
  prev.z = __shfl_up_sync(0xFFFFFFFFu, c.z, 1);
  prev.w = __shfl_up_sync(0xFFFFFFFFu, c.w, 1);
  if (lane == 0 && i > 0 && i < n) prev = __ldg(coords + i - 1);
  const bool starts = i < n && (i == 0 || !x_next(prev, c));
  const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, starts);
  if (lane == 0) s_cnt[warp] = __popc(ballot);
  __syncthreads();
  if (threadIdx.x < 2) {
    const int h = threadIdx.x * 4;
    const int64_t tile = static_cast<int64_t>(blockIdx.x) * 2 + threadIdx.x;
    if (tile * kTileRows < n) rc.cnt[tile] = s_cnt[h] + s_cnt[h + 1] + s_cnt[h + 2] + s_cnt[h + 3];
  }
  if (threadIdx.x == 0) {
    int32_t total = 0;
#pragma unroll
    for (int w = 0; w < kInsertThreads / 32; ++w) total += s_cnt[w];
    if (total) atomicAdd(rc.sb + (static_cast<int64_t>(blockIdx.x) * 2) / kSuperTiles, total);
  }
}

__global__ void map_insert_direct(const int4* __restrict__ coords, int64_t n, int grid, int batch,
                                  int32_t* __restrict__ cells, uint32_t* status,
                                  RunCount rc) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int4 c = i < n ? __ldg(coords + i) : make_int4(-1, -1, -1, -1);
  if (rc.cnt) count_run_starts(coords, n, i, c, rc);
  if (i >= n) return;
  if (!in_volume(c, grid, batch)) {
    atomicOr(status, kErrRange);
    return;
  }
  cells[cell_of(c.x, c.y, c.z, c.w, grid)] = static_cast<int32_t>(i);
}

__global__ void map_insert_compact(const int4* __restrict__ coords, int64_t n, int grid, int batch,
                                   unsigned long long* __restrict__ table, uint32_t capmask,
                                   uint32_t* status, RunCount rc) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int4 c = i < n ? __ldg(coords + i) : make_int4(-1, -1, -1, -1);
  if (rc.cnt) count_run_starts(coords, n, i, c, rc);
  if (i >= n) return;
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
                                uint32_t capmask, uint32_t* status, RunCount rc) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int4 c = i < n ? __ldg(coords + i) : make_int4(-1, -1, -1, -1);
  if (rc.cnt) count_run_starts(coords, n, i, c, rc);
  if (i >= n) return;
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

// ----------------------------------------------------------- run layout ----
// The query kernel also lays out the x-run positions: with R(v) the run starts
// among rows 0..v, voxel v sits at position v + 2 R(v), its run's left pad (when
// v starts the run) at the position before, the right pad (when v ends it) at
// the one after.

static_assert(kPosTile == 256, "et_store_row splits positions with shifts by 8");
static_assert(kInsertThreads == 256 && kSuperTiles % 2 == 0, "insert block = two query tiles");

struct RunOut {
  const int32_t* cnt;  // run starts per 128-row tile (insert kernel)
  const int32_t* sb;   // run starts per superblock of 128 tiles (insert kernel)
  int32_t* hdr;        // [4]: runs, position tiles, positions, 0
  int32_t* pos;        // position table
  int32_t* et;         // E index table
};

// E row q of offset pair dzdy is entry (q mod 256) + 1 of tile q / 256; a tile
// also keeps copies of its edge rows' outer neighbours (entry 0 of the next
// tile is row 255 of this one; entry 257 of the previous tile is row 0).
// Writes E row q for all 9 pairs, the value of pair dzdy being v[3 * dzdy].
__device__ __forceinline__ void et_store_row(int32_t* et, int64_t q, const int32_t* v) {
  const int64_t t = q >> 8;
  const int i = static_cast<int>(q & 255);
  int32_t* b = et + t * (9 * kEtStride) + i + 1;
#pragma unroll
  for (int dzdy = 0; dzdy < 9; ++dzdy) b[dzdy * kEtStride] = v[3 * dzdy];
  if (i == kPosTile - 1 || (i == 0 && t > 0)) {  // one row in 128
    int32_t* h = i == 0 ? et + (t - 1) * (9 * kEtStride) + kPosTile + 1
                        : et + (t + 1) * (9 * kEtStride);
#pragma unroll
    for (int dzdy = 0; dzdy < 9; ++dzdy) h[dzdy * kEtStride] = v[3 * dzdy];
  }
}

// One block per 128-row tile, one thread per voxel: 27 lookups into shared
// memory, then the [128, 27] nbr block and the tile's offset mask with
// coalesced stores.  With RUNS, also the tile's positions and E index entries.
template <Kind K, bool RUNS>
__global__ void __launch_bounds__(kTileRows)
    map_query(const int4* __restrict__ coords, int64_t n, int grid, int batch, Tables t,
              int32_t* __restrict__ nbr, uint32_t* __restrict__ tile_mask, uint32_t* status,
              RunOut ro) {
  __shared__ __align__(16) int32_t s_nbr[kTileRows * kKvol];
  __shared__ uint32_t s_bits[kTileRows / 32];
  __shared__ uint32_t s_starts[kTileRows / 32];  // run-start ballot of each warp
  __shared__ int32_t s_before[kTileRows / 32];   // partial sums of the run starts before the tile
  __shared__ int64_t s_end;
  const int r = threadIdx.x;
  const int lane = r & 31, warp = r >> 5;
  pdl_wait();
  pdl_trigger();
  const int64_t tile = blockIdx.x;
  const int64_t row0 = tile * kTileRows;
  const int64_t i = row0 + r;
  int4 c = make_int4(-1, -1, -1, -1);
  if (i < n) c = __ldg(coords + i);
  bool starts = false, ends = false;
  if constexpr (RUNS) {
    if (i < n) {
      starts = i == 0 || !x_next(__ldg(coords + i - 1), c);
      ends = i == n - 1 || !x_next(c, __ldg(coords + i + 1));
    }
    const int64_t sb = tile / kSuperTiles;
    int32_t part = 0;
    for (int64_t j = r; j < sb; j += kTileRows) part += __ldg(ro.sb + j);
    for (int64_t j = sb * kSuperTiles + r; j < tile; j += kTileRows) part += __ldg(ro.cnt + j);
    part = __reduce_add_sync(0xFFFFFFFFu, part);
    const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, starts);
    if (lane == 0) {
      s_starts[warp] = ballot;
      s_before[warp] = part;
    }
  }
  uint32_t bits = 0u;
  if (i < n) {
    if (in_volume(c, grid, batch)) {
      if constexpr (K == Kind::kDirect) {
        // the direct table has <= 2^28 cells: int32 cell indices.  The 9 (dz, dy)
        // rows are base pointers; dx = -1, 0, +1 are the cells before and after.
        const int32_t g = grid, g2 = grid * grid;
        const int32_t* centre = t.cells + (((c.x * g + c.y) * g + c.z) * g + c.w);
        const bool vz[3] = {c.y > 0, true, c.y < g - 1};
        const bool vy[3] = {c.z > 0, true, c.z < g - 1};
        const bool vx[3] = {c.w > 0, true, c.w < g - 1};
#pragma unroll
        for (int dz = 0; dz < 3; ++dz) {
#pragma unroll
          for (int dy = 0; dy < 3; ++dy) {
            const int32_t* row = centre + (dz - 1) * g2 + (dy - 1) * g;
#pragma unroll
            for (int dx = 0; dx < 3; ++dx) {
              const int k = dz * 9 + dy * 3 + dx;
              const int32_t found = (vz[dz] && vy[dy] && vx[dx]) ? __ldg(row + dx - 1) : -1;
              s_nbr[r * kKvol + k] = found;
              bits |= (found >= 0 ? 1u : 0u) << k;
            }
          }
        }
        if (s_nbr[r * kKvol + 13] != static_cast<int32_t>(i))
          atomicOr(status, kErrDuplicate);  // another row owns this voxel's cell
      } else {
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
      }
    } else {
#pragma unroll
      for (int k = 0; k < kKvol; ++k) s_nbr[r * kKvol + k] = -1;
    }
  }
  bits = __reduce_or_sync(0xFFFFFFFFu, bits);
  if (lane == 0) s_bits[warp] = bits;
  __syncthreads();
  if (r == 0) tile_mask[tile] = s_bits[0] | s_bits[1] | s_bits[2] | s_bits[3];
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
  if constexpr (!RUNS) return;
  // (the __syncthreads above also published s_starts and s_before)
  const int64_t excl = static_cast<int64_t>(s_before[0]) + s_before[1] + s_before[2] + s_before[3];
  const uint32_t agg = __popc(s_starts[0]) + __popc(s_starts[1]) + __popc(s_starts[2]) +
                       __popc(s_starts[3]);
  int64_t runs = excl;  // run starts among rows 0..i
  for (int w = 0; w < warp; ++w) runs += __popc(s_starts[w]);
  runs += __popc(s_starts[warp] & (0xFFFFFFFFu >> (31 - lane)));
  if (i < n) {
    const int64_t p = i + 2 * runs;
    const int32_t tag = static_cast<int32_t>(i * 4);
    ro.pos[p] = tag + kPosVoxel;
    if (starts) ro.pos[p - 1] = tag + kPosLeftPad;
    if (ends) ro.pos[p + 1] = tag + kPosRightPad;
    const int32_t* nb = s_nbr + r * kKvol;  // nb[3 * dzdy + dx + 1]
    et_store_row(ro.et, p, nb + 1);
    if (starts) et_store_row(ro.et, p - 1, nb);
    if (ends) et_store_row(ro.et, p + 1, nb + 2);
    if (i == 0) {  // position 0 (the absent right pad before the first run) and row -1
      ro.pos[0] = -1;
#pragma unroll
      for (int dzdy = 0; dzdy < 9; ++dzdy) {
        ro.et[dzdy * kEtStride] = -1;
        ro.et[dzdy * kEtStride + 1] = -1;
      }
    }
    if (i == n - 1) s_end = p + 2;  // one past the last run's right pad
  }
  if (row0 + kTileRows >= n) {  // the tile of row n-1: header, and the line's tail
    __syncthreads();
    // positions up to the last voxel: N + 2 runs; the last right pad is not counted,
    // as its only reader, row 256 of its voxel's tile, holds a copy of it
    const int64_t end = s_end;
    const int64_t positions = end - 1;
    const int64_t ptiles = (positions + kPosTile - 1) / kPosTile;
    if (r == 0) {
      ro.hdr[0] = static_cast<int32_t>(excl + agg);
      ro.hdr[1] = static_cast<int32_t>(ptiles);
      ro.hdr[2] = static_cast<int32_t>(positions);
      ro.hdr[3] = 0;
    }
    int32_t none[kKvol];
#pragma unroll
    for (int k = 0; k < kKvol; ++k) none[k] = -1;
    for (int64_t q = end + r; q <= ptiles * kPosTile; q += kTileRows) {
      if (q < ptiles * kPosTile) ro.pos[q] = -1;
      et_store_row(ro.et, q, none);
    }
  }
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
  const double direct_budget = std::max(static_cast<double>(kDirectTableMinBytes),
                                        kDirectTableBytesPerVoxel * static_cast<double>(n));
  const bool direct_fits = cells * 4.0 <= direct_budget && cells <= kDirectTableMaxCells;
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
  if (!opt.run_layout || n >= kRunLayoutMaxRows) {  // nbr and tile masks only
    lay.cnt_off = lay.sb_off = lay.hdr_off = lay.pos_off = lay.et_off = end;
    lay.total = end;
    *out = lay;
    return true;
  }
  lay.pos_max = static_cast<int64_t>(align_up(static_cast<size_t>(3 * n), kPosTile)) + kPosTile;
  lay.ptile_max = lay.pos_max / kPosTile;
  lay.cnt_off = end;
  lay.sb_off = align_up(lay.cnt_off + static_cast<size_t>(lay.n_tiles) * 4, 256);
  const int64_t n_super = (lay.n_tiles + kSuperTiles - 1) / kSuperTiles;
  lay.hdr_off = align_up(lay.sb_off + static_cast<size_t>(n_super) * 4, 256);
  lay.pos_off = lay.hdr_off + 256;
  lay.pos_bytes = static_cast<size_t>(lay.pos_max) * 4;
  lay.et_off = align_up(lay.pos_off + lay.pos_bytes, 256);
  lay.total = align_up(lay.et_off + static_cast<size_t>(lay.ptile_max) * 9 * kEtStride * 4, 256);
  *out = lay;
  return true;
}

namespace {

template <Kind K>
void launch_query(unsigned blocks, bool runs, const int4* c4, int64_t n, int grid, int batch,
                  const Tables& t, int32_t* nbr, uint32_t* mask, uint32_t* status,
                  const RunOut& ro, cudaStream_t stream) {
  if (runs)
    launch_pdl(map_query<K, true>, blocks, kTileRows, 0, stream, c4, n, grid, batch, t, nbr, mask,
               status, ro);
  else
    launch_pdl(map_query<K, false>, blocks, kTileRows, 0, stream, c4, n, grid, batch, t, nbr,
               mask, status, ro);
}

}  // namespace

cudaError_t launch_map_build(const int32_t* coords, int64_t n, int32_t grid_dim, int32_t batch,
                             int32_t* nbr, void* workspace, const MapLayout& lay,
                             cudaStream_t stream) {
  auto* ws = static_cast<uint8_t*>(workspace);
  auto* status = reinterpret_cast<uint32_t*>(ws + lay.status_off);
  auto* mask = reinterpret_cast<uint32_t*>(ws + lay.mask_off);
  auto* table = ws + lay.table_off;
  const bool runs = lay.ptile_max > 0;
  RunOut ro{};
  RunCount rc{};
  size_t sb_words16 = 0;
  if (runs) {
    rc.cnt = reinterpret_cast<int32_t*>(ws + lay.cnt_off);
    rc.sb = reinterpret_cast<int32_t*>(ws + lay.sb_off);
    ro.cnt = rc.cnt;
    ro.sb = rc.sb;
    ro.hdr = reinterpret_cast<int32_t*>(ws + lay.hdr_off);
    ro.pos = reinterpret_cast<int32_t*>(ws + lay.pos_off);
    ro.et = reinterpret_cast<int32_t*>(ws + lay.et_off);
    sb_words16 = (lay.hdr_off - lay.sb_off) / 16;  // the 256-byte aligned superblock region
  }
  const size_t words16 = lay.table_bytes / 16;
  {
    const size_t work = words16 > sb_words16 ? words16 : sb_words16;
    size_t blocks = (work + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks == 0) blocks = 1;
    launch_pdl(map_init, static_cast<unsigned>(blocks), 256, 0, stream,
               reinterpret_cast<uint4*>(table), words16, reinterpret_cast<uint4*>(rc.sb),
               sb_words16, status, ro.hdr);
  }
  if (n == 0) return cudaGetLastError();
  const auto* c4 = reinterpret_cast<const int4*>(coords);
  const unsigned ins_blocks = static_cast<unsigned>((n + kInsertThreads - 1) / kInsertThreads);
  const unsigned q_blocks = static_cast<unsigned>(lay.n_tiles);
  Tables t{};
  t.capmask = static_cast<uint32_t>(lay.capacity - 1);
  if (lay.kind == MapKind::kDirect) {
    t.cells = reinterpret_cast<const int32_t*>(table);
    launch_pdl(map_insert_direct, ins_blocks, kInsertThreads, 0, stream, c4, n, grid_dim, batch,
               reinterpret_cast<int32_t*>(table), status, rc);
    launch_query<Kind::kDirect>(q_blocks, runs, c4, n, grid_dim, batch, t, nbr, mask, status, ro,
                                stream);
  } else if (lay.compact) {
    t.table = reinterpret_cast<const unsigned long long*>(table);
    launch_pdl(map_insert_compact, ins_blocks, kInsertThreads, 0, stream, c4, n, grid_dim, batch,
               reinterpret_cast<unsigned long long*>(table), t.capmask, status, rc);
    launch_query<Kind::kCompact>(q_blocks, runs, c4, n, grid_dim, batch, t, nbr, mask, status,
                                 ro, stream);
  } else {
    auto* rows = reinterpret_cast<int32_t*>(ws + lay.rows_off);
    t.table = reinterpret_cast<const unsigned long long*>(table);
    t.rows = rows;
    launch_pdl(map_insert_wide, ins_blocks, kInsertThreads, 0, stream, c4, n, grid_dim, batch,
               reinterpret_cast<unsigned long long*>(table), rows, t.capmask, status, rc);
    launch_query<Kind::kWide>(q_blocks, runs, c4, n, grid_dim, batch, t, nbr, mask, status, ro,
                              stream);
  }
  return cudaGetLastError();
}

}  // namespace subm3d

// Neighbour-map build for the submanifold 3x3x3 convolution.
//
// The pages build a "sorted-key indice map (27 lookups/voxel vectorised)"
// (lato.2_mrp_mlx, commit 97dcdfb54a message).  Here the lookup structure is
// one of three GPU tables over packed (b, z, y, x) keys, chosen per call:
//
//   direct  when batch * (grid_dim + 2)^3 int32 cells take at most max(64 MB,
//           256 B x N) and 2^28 cells, and the table is small (<= 64 MB) or
//           dense (<= 16 cells per voxel): cell -> row, -1 when empty; each
//           grid has a one-cell border no voxel occupies, so a voxel's 27
//           neighbour cells all exist and its lookups need no bounds test.  A
//           collision-free perfect hash: insert is one plain store per voxel,
//           a lookup is one load, and voxels adjacent in raster order look up
//           adjacent cells, so the 27 lookups of a warp coalesce.  A duplicate
//           coordinate leaves one of its rows in the cell; the other row sees
//           a foreign row at its own centre offset and raises the duplicate
//           flag (likewise in the brick table).
//   brick   for sparser volumes whose brick directory fits the same budget: the
//           bordered cells in bricks of 8 (x) x 4 (y) x 2 (z); the directory
//           (one int32 per brick) is cleared, the occupied bricks get 64-cell
//           blocks from a counter, and lookups go directory -> block.  Only the
//           directory and the blocks in use are written, not the whole volume.
//   hash    otherwise: open addressing with linear probing, capacity a power
//           of two >= 2N.  With batch <= 4 and grid_dim <= 1024 a key is
//           b:2|z:10|y:10|x:10 and a slot the 8-byte word (key << 32 | row),
//           published by one 64-bit CAS; else a key is b:16|z:16|y:16|x:16 in
//           a uint64 array with a separate int32 row array.  The home slot is
//           4 * h(key >> 2) + (key & 3), h a 32-bit avalanche mix, so the
//           x-neighbours of a voxel usually share a 32-byte sector.  Probe
//           loops are bounded by the capacity; a full table raises a flag.
//
// Kernels (each launched with programmatic dependent launch, so that its
// blocks start while the previous kernel drains and do whatever touches only
// the build's inputs before griddepcontrol.wait):
//   map_init    table (brick: directory) <- empty, run-count sums, status
//               word, brick counter and header <- 0;
//   map_brick_alloc (brick table only) a pool block for every occupied brick;
//   map_insert  one thread per voxel: 16-byte coordinate load, range check and
//               the run starts of its 128-row tile (before the wait), then the
//               insert;
//   map_query   one block per 128-row tile, one thread per voxel: the 27
//               lookups go to shared memory, then one bulk asynchronous copy
//               writes the tile's [128, 27] nbr block and one store its offset
//               mask (no atomics on the output), and the tile's share of the
//               x-run layout.
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
    status[0] = 0u;  // error bits
    status[1] = 0u;  // brick table: pool blocks handed out
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

// The row before and the row after row i (lanes take them from their
// neighbours; the warp's first and last lanes load them).
__device__ __forceinline__ int4 shfl_up_int4(int4 c, int lane, const int4* coords, int i) {
  int4 p;
  p.x = __shfl_up_sync(0xFFFFFFFFu, c.x, 1);
  p.y = __shfl_up_sync(0xFFFFFFFFu, c.y, 1);
  p.z = __shfl_up_sync(0xFFFFFFFFu, c.z, 1);
  p.w = __shfl_up_sync(0xFFFFFFFFu, c.w, 1);
  if (lane == 0) p = i > 0 ? __ldg(coords + i - 1) : make_int4(-1, -1, -1, -1);
  return p;
}
__device__ __forceinline__ int4 shfl_down_int4(int4 c, int lane, const int4* coords, int i,
                                               int n) {
  int4 q;
  q.x = __shfl_down_sync(0xFFFFFFFFu, c.x, 1);
  q.y = __shfl_down_sync(0xFFFFFFFFu, c.y, 1);
  q.z = __shfl_down_sync(0xFFFFFFFFu, c.z, 1);
  q.w = __shfl_down_sync(0xFFFFFFFFu, c.w, 1);
  if (lane == 31) q = i + 1 < n ? __ldg(coords + i + 1) : make_int4(-1, -1, -1, -1);
  return q;
}

// The coordinates of row i (i < n) or -1s, with the run-start counts of its
// insert block written (before the kernel's wait: they depend on the
// coordinates only).  Returns the block's run-start total in thread 0.
__device__ __forceinline__ int32_t insert_prologue(const int4* __restrict__ coords, int n, int i,
                                                   int4 c, const RunCount& rc) {
  __shared__ int32_t s_cnt[kInsertThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int4 prev = shfl_up_int4(c, lane, coords, i);
  const bool starts = i < n && !x_next(prev, c);
  const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, starts);
  if (lane == 0) s_cnt[warp] = __popc(ballot);
  __syncthreads();
  if (threadIdx.x < 2) {
    const int h = threadIdx.x * 4;
    const int tile = blockIdx.x * 2 + threadIdx.x;
    if (tile * kTileRows < n) rc.cnt[tile] = s_cnt[h] + s_cnt[h + 1] + s_cnt[h + 2] + s_cnt[h + 3];
  }
  int32_t total = 0;
  if (threadIdx.x == 0)
#pragma unroll
    for (int w = 0; w < kInsertThreads / 32; ++w) total += s_cnt[w];
  return total;
}

// Brick table: each occupied brick gets a pool block.  Among a warp's lanes
// that share a brick the lowest one claims its directory entry (-1 -> -2, after
// a plain read that turns most claims away); the block's winners then take
// consecutive blocks from the counter after the status word with one atomic
// add, fill them with -1 and publish their indices.  The insert kernel,
// launched after this grid completes, writes rows into them.  Voxels outside
// the volume are left to the insert kernel's range check.
constexpr int kAllocThreads = 256;

__global__ void __launch_bounds__(kAllocThreads)
    map_brick_alloc(const int4* __restrict__ coords, int n, int grid, int batch, Tables t,
                    int32_t* __restrict__ dir, int32_t* __restrict__ pool, uint32_t* status) {
  __shared__ uint32_t s_won[kAllocThreads / 32];
  __shared__ uint32_t s_base;
  const int i = blockIdx.x * kAllocThreads + threadIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int4 c = i < n ? __ldg(coords + i) : make_int4(-1, -1, -1, -1);
  const bool valid = i < n && in_volume(c, grid, batch);
  const long long brick = valid ? brick_of(t, c.x, c.y + 1, c.z + 1, c.w + 1) : -1ll;
  const unsigned peers = __match_any_sync(0xFFFFFFFFu, brick);
  pdl_wait();  // the directory and the counter are cleared
  pdl_trigger();
  bool won = false;
  if (valid && __ffs(peers) - 1 == lane) {
    int32_t* d = dir + brick;
    won = *reinterpret_cast<volatile int32_t*>(d) == -1 && atomicCAS(d, -1, -2) == -1;
  }
  const unsigned wins = __ballot_sync(0xFFFFFFFFu, won);
  if (lane == 0) s_won[warp] = __popc(wins);
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t total = 0;
    for (int w = 0; w < kAllocThreads / 32; ++w) {
      const uint32_t k = s_won[w];
      s_won[w] = total;  // exclusive prefix over the warps
      total += k;
    }
    s_base = total ? atomicAdd(status + 1, total) : 0u;  // < min(N, bricks) blocks in all
  }
  __syncthreads();
  if (won) {
    const uint32_t slot = s_base + s_won[warp] + __popc(wins & ((1u << lane) - 1u));
    uint4* blk = reinterpret_cast<uint4*>(pool + static_cast<int64_t>(slot) * kBrickCells);
    const uint4 ones = make_uint4(~0u, ~0u, ~0u, ~0u);
#pragma unroll
    for (int k = 0; k < kBrickCells / 4; ++k) blk[k] = ones;
    dir[brick] = static_cast<int32_t>(slot);
  }
}

template <Kind K>
__global__ void __launch_bounds__(kInsertThreads)
    map_insert(const int4* __restrict__ coords, int n, int grid, int batch, Tables t,
               int32_t* __restrict__ cells, unsigned long long* __restrict__ table,
               int32_t* __restrict__ rows, uint32_t* status, RunCount rc) {
  const int i = blockIdx.x * kInsertThreads + threadIdx.x;
  const int4 c = i < n ? __ldg(coords + i) : make_int4(-1, -1, -1, -1);
  const int32_t total = rc.cnt ? insert_prologue(coords, n, i, c, rc) : 0;
  pdl_wait();  // the table and the superblock sums are cleared
  pdl_trigger();
  if (total) atomicAdd(rc.sb + (blockIdx.x * 2) / kSuperTiles, total);
  if (i >= n) return;
  if (!in_volume(c, grid, batch)) {
    atomicOr(status, kErrRange);
    return;
  }
  if constexpr (K == Kind::kDirect) {
    cells[cell_of(c.x, c.y, c.z, c.w, grid)] = i;
  } else if constexpr (K == Kind::kBrick) {  // `cells` is the pool, t.rows the directory
    const int32_t slot = ld_dep(t.rows + brick_of(t, c.x, c.y + 1, c.z + 1, c.w + 1));
    cells[static_cast<int64_t>(slot) * kBrickCells + brick_cell(c.y + 1, c.z + 1, c.w + 1)] = i;
  } else if constexpr (K == Kind::kCompact) {
    const uint32_t key = pack32(c.x, c.y, c.z, c.w);
    const unsigned long long entry =
        (static_cast<unsigned long long>(key) << 32) | static_cast<uint32_t>(i);
    uint32_t slot = home32(key, t.capmask);
    for (uint64_t step = 0; step <= t.capmask; ++step) {
      const unsigned long long prev = atomicCAS(table + slot, kEmpty, entry);
      if (prev == kEmpty) return;
      if (static_cast<uint32_t>(prev >> 32) == key) {
        atomicOr(status, kErrDuplicate);
        return;
      }
      slot = (slot + 1) & t.capmask;
    }
    atomicOr(status, kErrTableFull);
  } else {
    const unsigned long long key = pack64(c.x, c.y, c.z, c.w);
    uint32_t slot = home64(key, t.capmask);
    for (uint64_t step = 0; step <= t.capmask; ++step) {
      const unsigned long long prev = atomicCAS(table + slot, kEmpty, key);
      if (prev == kEmpty) {
        rows[slot] = i;
        return;
      }
      if (prev == key) {
        atomicOr(status, kErrDuplicate);
        return;
      }
      slot = (slot + 1) & t.capmask;
    }
    atomicOr(status, kErrTableFull);
  }
}

// ----------------------------------------------------------- run layout ----
// The query kernel also lays out the x-run positions: with R(v) the run starts
// among rows 0..v, voxel v sits at position v + 2 R(v), its run's left pad (when
// v starts the run) at the position before, the right pad (when v ends it) at
// the one after.  E row q of pair dz-dy is entry q + 1 of that pair's line.

static_assert(kInsertThreads == 256 && kSuperTiles % 2 == 0, "insert block = two query tiles");
// Positions one warp's 32 rows can occupy: each row its own run, with both pads.
constexpr int kWarpSpan = 3 * 32;

struct RunOut {
  const int32_t* cnt;  // run starts per 128-row tile (insert kernel)
  const int32_t* sb;   // run starts per superblock of 128 tiles (insert kernel)
  int32_t* hdr;        // [4]: runs, position tiles, positions, E line stride
  int32_t* pos;        // position table
  int32_t* et;         // E index table: 9 lines of `es` entries
  int32_t es;          // E line stride (entries)
};

__device__ __forceinline__ void bulk_store_smem(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
               "r"(static_cast<uint32_t>(__cvta_generic_to_shared(ssrc))), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// One block per 128-row tile, one thread per voxel: 27 lookups into shared
// memory, then the [128, 27] nbr block (one bulk copy for a whole tile) and the
// tile's offset mask.  With RUNS, also the tile's positions and E entries.
template <Kind K, bool RUNS>
__global__ void __launch_bounds__(kTileRows)
    map_query(const int4* __restrict__ coords, int n, int grid, int batch, Tables t,
              int32_t* __restrict__ nbr, uint32_t* __restrict__ tile_mask, uint32_t* status,
              RunOut ro) {
  __shared__ __align__(128) int32_t s_nbr[kTileRows * kKvol];
  __shared__ uint32_t s_bits[kTileRows / 32];
  __shared__ uint32_t s_starts[kTileRows / 32];  // run-start ballot of each warp
  __shared__ int32_t s_before[kTileRows / 32];   // partial sums of the run starts before the tile
  __shared__ int32_t s_end;
  __shared__ uint8_t s_src[RUNS ? 4 * kWarpSpan : 4];  // position -> row and kind, per warp
  const int r = threadIdx.x;
  const int lane = r & 31, warp = r >> 5;
  const int tile = blockIdx.x;
  const int row0 = tile * kTileRows;
  const int i = row0 + r;
  const bool live = i < n;
  // the coordinates are the build's input: read before the wait for the table
  const int4 c = live ? __ldg(coords + i) : make_int4(-1, -1, -1, -1);
  bool starts = false, ends = false;
  if constexpr (RUNS) {
    // the same rule as the insert kernel's count, so positions match the counts
    const int4 prev = shfl_up_int4(c, lane, coords, i);
    const int4 next = shfl_down_int4(c, lane, coords, i, n);
    starts = live && !x_next(prev, c);
    ends = live && !x_next(c, next);
  }
  pdl_wait();  // the table, the run counts and the superblock sums are complete
  pdl_trigger();
  if constexpr (RUNS) {
    const int sb = tile / kSuperTiles;
    int32_t part = 0;
    for (int j = r; j < sb; j += kTileRows) part += ld_dep(ro.sb + j);
    for (int j = sb * kSuperTiles + r; j < tile; j += kTileRows) part += ld_dep(ro.cnt + j);
    part = __reduce_add_sync(0xFFFFFFFFu, part);
    const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, starts);
    if (lane == 0) {
      s_starts[warp] = ballot;
      s_before[warp] = part;
    }
  }
  int32_t* nb = s_nbr + r * kKvol;
  uint32_t absent = 0u;  // bit 26 - k set when offset k has no neighbour
  if (live) {
    if (in_volume(c, grid, batch)) {
      if constexpr (K == Kind::kDirect) {
        // the bordered table has <= 2^28 cells: int32 cell indices; every one of
        // the 27 cells exists.  Rows (dz, dy) are base pointers, dx = -1, 0, +1
        // the cells before and after.
        const int32_t g = grid + 2, g2 = g * g;
        const int32_t* centre = t.cells + (((c.x * g + c.y + 1) * g + c.z + 1) * g + c.w + 1);
#pragma unroll
        for (int dz = 0; dz < 3; ++dz) {
#pragma unroll
          for (int dy = 0; dy < 3; ++dy) {
            const int32_t* row = centre + ((dz - 1) * g2 + (dy - 1) * g);
#pragma unroll
            for (int dx = 0; dx < 3; ++dx) {
              const int32_t v = ld_dep(row + dx - 1);
              nb[dz * 9 + dy * 3 + dx] = v;
              absent = __funnelshift_l(static_cast<uint32_t>(v), absent, 1);  // sign bit in
            }
          }
        }
        if (nb[13] != i) atomicOr(status, kErrDuplicate);  // another row owns this cell
      } else if constexpr (K == Kind::kBrick) {
        // bordered cells: the 27 directory loads first (mostly one brick), then
        // the cells of the bricks that exist
        const int Z = c.y + 1, Y = c.z + 1, X = c.w + 1;
        int32_t slot[kKvol];
#pragma unroll
        for (int k = 0; k < kKvol; ++k)
          slot[k] = ld_dep(t.rows + brick_of(t, c.x, Z + k / 9 - 1, Y + (k / 3) % 3 - 1,
                                            X + k % 3 - 1));
#pragma unroll
        for (int k = 0; k < kKvol; ++k) {
          const int32_t v =
              slot[k] < 0 ? -1
                          : ld_dep(t.cells + static_cast<int64_t>(slot[k]) * kBrickCells +
                                  brick_cell(Z + k / 9 - 1, Y + (k / 3) % 3 - 1, X + k % 3 - 1));
          nb[k] = v;
          absent = __funnelshift_l(static_cast<uint32_t>(v), absent, 1);
        }
        if (nb[13] != i) atomicOr(status, kErrDuplicate);  // another row owns this cell
      } else {
#pragma unroll
        for (int k = 0; k < kKvol; ++k) {
          const int z = c.y + k / 9 - 1;
          const int y = c.z + (k / 3) % 3 - 1;
          const int x = c.w + k % 3 - 1;
          int32_t v = -1;
          if (static_cast<unsigned>(z) < static_cast<unsigned>(grid) &&
              static_cast<unsigned>(y) < static_cast<unsigned>(grid) &&
              static_cast<unsigned>(x) < static_cast<unsigned>(grid))
            v = lookup<K>(t, c.x, z, y, x, grid);
          nb[k] = v;
          absent = __funnelshift_l(static_cast<uint32_t>(v), absent, 1);
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < kKvol; ++k) nb[k] = -1;
      absent = (1u << kKvol) - 1u;
    }
  } else {
    absent = (1u << kKvol) - 1u;
  }
  // bit k of the mask: offset k present somewhere in the tile
  const uint32_t present = __brev(~absent << (32 - kKvol)) & ((1u << kKvol) - 1u);
  const uint32_t bits = __reduce_or_sync(0xFFFFFFFFu, present);
  if (lane == 0) s_bits[warp] = bits;
  const int rows = n - row0 < kTileRows ? n - row0 : kTileRows;
  if (rows == kTileRows)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // nb -> the bulk copy
  __syncthreads();
  if (r == 0) {
    tile_mask[tile] = s_bits[0] | s_bits[1] | s_bits[2] | s_bits[3];
    // 13,824 bytes = 864 16-byte words; each tile's block starts 16-byte aligned
    if (rows == kTileRows)
      bulk_store_smem(nbr + static_cast<int64_t>(row0) * kKvol, s_nbr, kTileRows * kKvol * 4);
  }
  if (rows < kTileRows) {
    int32_t* dst = nbr + static_cast<int64_t>(row0) * kKvol;
    for (int e = r; e < rows * kKvol; e += kTileRows) dst[e] = s_nbr[e];
  }
  if constexpr (RUNS) {
    // (the __syncthreads above also published s_starts and s_before)
    const int32_t excl = s_before[0] + s_before[1] + s_before[2] + s_before[3];
    const int32_t agg = __popc(s_starts[0]) + __popc(s_starts[1]) + __popc(s_starts[2]) +
                        __popc(s_starts[3]);
    int32_t runs = excl;  // run starts among rows 0..i
    for (int w = 0; w < warp; ++w) runs += __popc(s_starts[w]);
    runs += __popc(s_starts[warp] & (0xFFFFFFFFu >> (31 - lane)));
    const int es = ro.es;
    const int p = i + 2 * runs;  // this row's position (when live)
    // Position-major stores: the warp's positions form one range [w0, w1] (its
    // first row's left pad, if that row starts a run, to its last row's right
    // pad, if that row ends one; at most 96), every position the voxel, left pad
    // or right pad of one of its rows.  Each lane records which row and which of
    // the three occupies its positions, then the lanes write the range's
    // position entries and E entries in order, 32 consecutive positions per
    // store, instead of scattered single stores for the pads.
    const uint32_t live_lanes = __ballot_sync(0xFFFFFFFFu, live);
    int w0 = 0, w1 = -1;
    if (live_lanes) {
      w0 = __shfl_sync(0xFFFFFFFFu, starts ? p - 1 : p, __ffs(live_lanes) - 1);
      w1 = __shfl_sync(0xFFFFFFFFu, ends ? p + 1 : p, 31 - __clz(live_lanes));
    }
    uint8_t* src_of = s_src + warp * kWarpSpan;  // position - w0 -> lane * 4 + kind
    if (live) {
      src_of[p - w0] = static_cast<uint8_t>(lane * 4 + 1);                 // the voxel
      if (starts) src_of[p - 1 - w0] = static_cast<uint8_t>(lane * 4 + 0);  // its left pad
      if (ends) src_of[p + 1 - w0] = static_cast<uint8_t>(lane * 4 + 2);    // its right pad
    }
    __syncwarp();
    for (int q = w0 + lane; q <= w1; q += 32) {
      const int code = src_of[q - w0];
      const int r_src = warp * 32 + (code >> 2), kind = code & 3;  // kind = dx + 1
      ro.pos[q] = (row0 + r_src) * 4 +
                  (kind == 1 ? kPosVoxel : (kind == 0 ? kPosLeftPad : kPosRightPad));
      // E row q of pair dz-dy: the (dz, dy, dx) neighbour of the row's voxel
      const int32_t* nbs = s_nbr + r_src * kKvol + kind;
      int32_t* e = ro.et + (q + 1);
#pragma unroll
      for (int dzdy = 0; dzdy < 9; ++dzdy) e[dzdy * es] = nbs[3 * dzdy];
    }
    if (live) {
      if (i == 0) {  // position 0 (the absent right pad before the first run) and row -1
        ro.pos[0] = -1;
#pragma unroll
        for (int dzdy = 0; dzdy < 9; ++dzdy) {
          ro.et[dzdy * es] = -1;
          ro.et[dzdy * es + 1] = -1;
        }
      }
      if (i == n - 1) s_end = p + 2;  // one past the last run's right pad
    }
    if (row0 + kTileRows >= n) {  // the tile of row n-1: header, and the line's tail
      __syncthreads();
      // positions up to the last voxel: N + 2 runs - 1 (the last right pad, at
      // position `end` - 1, is read only as E row 256 of the last tile when it
      // falls there, and its entry is written above)
      const int end = s_end;
      const int positions = end - 1;
      const int ptiles = (positions + kPosTile - 1) / kPosTile;
      if (r == 0) {
        ro.hdr[0] = excl + agg;
        ro.hdr[1] = ptiles;
        ro.hdr[2] = positions;
        ro.hdr[3] = es;
      }
      for (int q = end + r; q <= ptiles * kPosTile; q += kTileRows) {
        if (q < ptiles * kPosTile) ro.pos[q] = -1;
#pragma unroll
        for (int dzdy = 0; dzdy < 9; ++dzdy) ro.et[dzdy * es + q + 1] = -1;
      }
    }
  }
  if (r == 0 && rows == kTileRows) bulk_wait_read();  // s_nbr stays until the copy has read it
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

bool map_layout(int64_t n, int32_t grid_dim, int32_t batch, const MapOptions& opt,
                MapLayout* out) {
  if (n < 0 || n >= kMaxMapRows || grid_dim < 1 || grid_dim > 65535 || batch < 1 ||
      batch > 65535)
    return false;
  MapLayout lay;
  const double gb = static_cast<double>(grid_dim) + 2.0;  // bordered grid
  const double cells = static_cast<double>(batch) * gb * gb * gb;
  const double direct_budget = std::max(static_cast<double>(kDirectTableMinBytes),
                                        kDirectTableBytesPerVoxel * static_cast<double>(n));
  const bool direct_fits = cells * 4.0 <= direct_budget && cells <= kDirectTableMaxCells;
  // brick directory over the bordered grids: bricks of 8 (x) x 4 (y) x 2 (z) cells
  const int64_t g2 = static_cast<int64_t>(grid_dim) + 2;
  lay.bgx = static_cast<int32_t>((g2 + 7) / 8);
  lay.bgy = static_cast<int32_t>((g2 + 3) / 4);
  lay.bgz = static_cast<int32_t>((g2 + 1) / 2);
  const double dir_cells = static_cast<double>(batch) * lay.bgz * lay.bgy * lay.bgx;
  const bool brick_fits = dir_cells * 4.0 <= direct_budget;
  if (opt.force_hash || opt.forced_capacity != 0)
    lay.kind = MapKind::kHash;
  else if (opt.force_brick && brick_fits)
    lay.kind = MapKind::kBrick;
  else if (opt.force_direct && direct_fits)
    lay.kind = MapKind::kDirect;
  else if (direct_fits && (cells * 4.0 <= static_cast<double>(kDirectTableMinBytes) ||
                           cells <= kDirectCellsPerVoxel * static_cast<double>(n)))
    lay.kind = MapKind::kDirect;  // small or dense: clearing the table is cheap
  else if (brick_fits)
    lay.kind = MapKind::kBrick;
  else
    lay.kind = direct_fits ? MapKind::kDirect : MapKind::kHash;
  lay.compact = (batch <= 4 && grid_dim <= 1024);
  uint64_t cap = 1024;
  while (cap < 2ull * static_cast<uint64_t>(n)) cap <<= 1;
  if (opt.forced_capacity != 0 && opt.forced_capacity < cap) {
    cap = 4;
    while (cap < opt.forced_capacity) cap <<= 1;
  }
  lay.capacity = cap;
  lay.cells = lay.kind == MapKind::kDirect ? static_cast<uint64_t>(cells) : 0;
  lay.n_tiles = (n + kTileRows - 1) / kTileRows;
  lay.status_off = 0;
  lay.mask_off = 256;
  lay.table_off = align_up(lay.mask_off + static_cast<size_t>(lay.n_tiles) * 4, 256);
  size_t end = 0;
  if (lay.kind == MapKind::kDirect) {
    lay.table_bytes = align_up(lay.cells * 4, 256);
    lay.rows_off = lay.table_off + lay.table_bytes;
    end = lay.rows_off;
  } else if (lay.kind == MapKind::kBrick) {
    const uint64_t dir_n = static_cast<uint64_t>(dir_cells);
    lay.bricks_max = std::max<uint64_t>(1, std::min<uint64_t>(static_cast<uint64_t>(n), dir_n));
    lay.table_bytes = align_up(dir_n * 4, 256);
    lay.rows_off = lay.table_off + lay.table_bytes;
    end = align_up(lay.rows_off + lay.bricks_max * kBrickCells * 4, 256);
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
  lay.et_stride = lay.pos_max + 4;  // entries for positions -1 .. pos_max, 16-byte lines
  lay.cnt_off = end;
  lay.sb_off = align_up(lay.cnt_off + static_cast<size_t>(lay.n_tiles) * 4, 256);
  const int64_t n_super = (lay.n_tiles + kSuperTiles - 1) / kSuperTiles;
  lay.hdr_off = align_up(lay.sb_off + static_cast<size_t>(n_super) * 4, 256);
  lay.pos_off = lay.hdr_off + 256;
  lay.pos_bytes = static_cast<size_t>(lay.pos_max) * 4;
  lay.et_off = align_up(lay.pos_off + lay.pos_bytes, 256);
  lay.total = align_up(lay.et_off + static_cast<size_t>(9 * lay.et_stride) * 4, 256);
  *out = lay;
  return true;
}

namespace {

template <Kind K>
void launch_build_kernels(unsigned ins_blocks, unsigned q_blocks, bool runs, const int4* c4,
                          int n, int grid, int batch, const Tables& t, int32_t* cells,
                          unsigned long long* table, int32_t* rows, int32_t* nbr, uint32_t* mask,
                          uint32_t* status, const RunCount& rc, const RunOut& ro,
                          cudaStream_t stream) {
  launch_pdl(map_insert<K>, ins_blocks, kInsertThreads, 0, stream, c4, n, grid, batch, t, cells,
             table, rows, status, rc);
  if (runs)
    launch_pdl(map_query<K, true>, q_blocks, kTileRows, 0, stream, c4, n, grid, batch, t, nbr,
               mask, status, ro);
  else
    launch_pdl(map_query<K, false>, q_blocks, kTileRows, 0, stream, c4, n, grid, batch, t, nbr,
               mask, status, ro);
}

}  // namespace

cudaError_t launch_map_build(const int32_t* coords, int64_t n, int32_t grid_dim, int32_t batch,
                             int32_t* nbr, void* workspace, const MapLayout& lay,
                             cudaStream_t stream) {
  if (n < 0 || n >= kMaxMapRows) return cudaErrorInvalidValue;
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
    ro.es = static_cast<int32_t>(lay.et_stride);
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
  const int ni = static_cast<int>(n);
  const unsigned ins_blocks = static_cast<unsigned>((n + kInsertThreads - 1) / kInsertThreads);
  const unsigned q_blocks = static_cast<unsigned>(lay.n_tiles);
  Tables t{};
  t.capmask = static_cast<uint32_t>(lay.capacity - 1);
  if (lay.kind == MapKind::kDirect) {
    t.cells = reinterpret_cast<const int32_t*>(table);
    launch_build_kernels<Kind::kDirect>(ins_blocks, q_blocks, runs, c4, ni, grid_dim, batch, t,
                                        reinterpret_cast<int32_t*>(table), nullptr, nullptr, nbr,
                                        mask, status, rc, ro, stream);
  } else if (lay.kind == MapKind::kBrick) {
    auto* dir = reinterpret_cast<int32_t*>(table);
    auto* pool = reinterpret_cast<int32_t*>(ws + lay.rows_off);
    t.cells = pool;
    t.rows = dir;
    t.bgx = lay.bgx;
    t.bgy = lay.bgy;
    t.bgz = lay.bgz;
    launch_pdl(map_brick_alloc, static_cast<unsigned>((n + kAllocThreads - 1) / kAllocThreads),
               kAllocThreads, 0, stream, c4, ni, grid_dim, batch, t, dir, pool, status);
    launch_build_kernels<Kind::kBrick>(ins_blocks, q_blocks, runs, c4, ni, grid_dim, batch, t,
                                       pool, nullptr, nullptr, nbr, mask, status, rc, ro, stream);
  } else if (lay.compact) {
    t.table = reinterpret_cast<const unsigned long long*>(table);
    launch_build_kernels<Kind::kCompact>(ins_blocks, q_blocks, runs, c4, ni, grid_dim, batch, t,
                                         nullptr, reinterpret_cast<unsigned long long*>(table),
                                         nullptr, nbr, mask, status, rc, ro, stream);
  } else {
    auto* rows = reinterpret_cast<int32_t*>(ws + lay.rows_off);
    t.table = reinterpret_cast<const unsigned long long*>(table);
    t.rows = rows;
    launch_build_kernels<Kind::kWide>(ins_blocks, q_blocks, runs, c4, ni, grid_dim, batch, t,
                                      nullptr, reinterpret_cast<unsigned long long*>(table), rows,
                                      nbr, mask, status, rc, ro, stream);
  }
  return cudaGetLastError();
}

}  // namespace subm3d

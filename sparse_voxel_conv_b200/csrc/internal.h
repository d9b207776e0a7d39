// Declarations shared by the C-ABI layer (subm3d_api.cu) and the kernel files.
// Not installed; the public surface is include/subm3d.h.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

namespace subm3d {

// Programmatic dependent launch.  The library's kernels are launched with the
// programmatic-serialization attribute, so a kernel may be scheduled while the
// previous kernel on the stream is finishing; every such kernel executes
// pdl_wait() (griddepcontrol.wait: until the preceding grid has completed and
// its writes are visible) before its first global-memory access, and the map
// kernels call pdl_trigger() to let the next kernel be scheduled early.  The
// wait is a no-op for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Loads, after pdl_wait(), of data that an earlier kernel of the chain writes.
// A kernel launched with the attribute can be running while that kernel still
// writes, so such data must not go through the non-coherent read-only path
// (ld.global.nc, __ldg): that path takes the data to be unchanged for the
// reading kernel's whole lifetime, and the compiler may schedule those loads
// above griddepcontrol.wait.  (A forward that read the map's header through it,
// queued right behind the build, at times saw the value from before the build
// and skipped whole tiles.)  These are ordinary coherent loads (ld.global.ca),
// written as volatile asm so that they stay after the wait.
__device__ __forceinline__ int32_t ld_dep(const int32_t* p) {
  int32_t v;
  asm volatile("ld.global.ca.b32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ unsigned long long ld_dep(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.global.ca.b64 %0, [%1];" : "=l"(v) : "l"(p));
  return v;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Bits of the map build's device status word.
constexpr uint32_t kErrRange = 1u;
constexpr uint32_t kErrDuplicate = 2u;
constexpr uint32_t kErrTableFull = 4u;

constexpr int kTileRows = 128;  // rows per tile-mask word
constexpr int kKvol = 27;
// Largest N + 1 a map may have: row and tile arithmetic of the map kernels is
// int32 (the last tile's end, N rounded up to 128, stays below 2^31).
constexpr int64_t kMaxMapRows = (int64_t(1) << 31) - 256;

// The three lookup structures of the map build (see map_build.cu).
enum class MapKind { kDirect, kHash, kBrick };

// The direct-address table (batch * (grid_dim + 2)^3 int32 cells: each grid
// with a one-cell border) may be used while it takes at most
// max(kDirectTableMinBytes, kDirectTableBytesPerVoxel * N) bytes and at most
// kDirectTableMaxCells cells (int32 cell arithmetic in the query).  Clearing it
// costs its size in HBM writes, so it is chosen while it is small (at most
// kDirectTableMinBytes) or dense (at most kDirectCellsPerVoxel cells per
// voxel); sparser volumes take the brick table when its directory fits the
// same budget, and the hash table otherwise.
constexpr size_t kDirectTableMinBytes = size_t(64) << 20;
constexpr double kDirectTableBytesPerVoxel = 256.0;
constexpr double kDirectTableMaxCells = double(int64_t(1) << 28);
constexpr double kDirectCellsPerVoxel = 16.0;

// The brick table cuts each bordered grid into bricks of 8 (x) x 4 (y) x 2 (z)
// cells: a directory of int32 (one per brick: -1, or the brick's slot) and a
// pool of 64-cell int32 blocks, one per occupied brick (at most min(N, bricks)
// of them, so at most 256 bytes per voxel).
constexpr int kBrickCells = 64;

// Testing knobs: force one table kind (where it fits), or cap the hash
// table's capacity (which implies the hash table).
struct MapOptions {
  bool force_hash = false;
  bool force_brick = false;
  bool force_direct = false;
  uint64_t forced_capacity = 0;  // a power of two, or 0
  bool run_layout = true;        // also build the x-run layout (subm3d_forward_map)
};

// x-run position layout used by the run-padded forward.  Voxels are laid out
// in row order on a line of positions; every run of x-adjacent voxels (same
// b, z, y; consecutive x and consecutive rows) is preceded by two pad
// positions: the right neighbour slot of the previous run and the left
// neighbour slot of this one.  Positions are cut into tiles of kPosTile.
constexpr int kPosTile = 256;
// The E index table holds one line per offset pair (dz, dy), et_stride int32
// entries apart: entry q + 1 of line dz-dy is the feature row gathered as E
// row q (position q), for -1 <= q <= 256 * tiles, or -1.  A tile's E rows
// -1 .. 256 are the 258 consecutive entries from 256 * tile.
// The run layout is built for N < 2^29, so that positions (< 3N + 512) and
// position-table entries (row * 4 + tag) fit int32; larger maps go without it.
constexpr int64_t kRunLayoutMaxRows = int64_t(1) << 29;
// Tags of a position-table entry (row * 4 + tag); -1 is an empty position.
constexpr int kPosVoxel = 0, kPosLeftPad = 1, kPosRightPad = 2;

// Placement of the map build's pieces inside the caller's workspace.
struct MapLayout {
  MapKind kind = MapKind::kDirect;
  bool compact = true;      // hash: 32-bit keys in 8-byte (key, row) slots; else 64-bit keys + rows
  uint64_t capacity = 0;    // hash slots, a power of two >= 4
  uint64_t cells = 0;       // direct: batch * (grid_dim + 2)^3
  int32_t bgx = 0, bgy = 0, bgz = 0;  // brick: bricks along x, y, z of one bordered grid
  uint64_t bricks_max = 0;  // brick: pool blocks reserved, min(N, directory entries)
  size_t status_off = 0;    // uint32 status word (+ the brick counter, uint32, after it)
  size_t mask_off = 0;      // uint32 [n_tiles]
  size_t table_off = 0;     // direct: int32 [cells]; hash: uint64 [capacity] (slots or keys);
                            // brick: int32 directory [batch * bgz * bgy * bgx]
  size_t table_bytes = 0;   // bytes of the table (a multiple of 16)
  size_t rows_off = 0;      // hash, wide keys only: int32 rows [capacity];
                            // brick: int32 pool [bricks_max * kBrickCells]
  // run layout (all kinds)
  size_t cnt_off = 0;       // int32 [n_tiles]: run starts per 128-row tile
  size_t sb_off = 0;        // int32 [ceil(n_tiles / 128)]: run starts per superblock
  size_t hdr_off = 0;       // int32 [4]: runs, position tiles, positions, E line stride
  size_t pos_off = 0;       // int32 [pos_max]: position table (row * 4 + tag, or -1)
  size_t pos_bytes = 0;
  size_t et_off = 0;        // int32 [9][et_stride]: E index table
  int64_t et_stride = 0;    // entries per (dz, dy) line: pos_max + 4
  int64_t pos_max = 0;      // positions reserved: 3N rounded up to whole tiles, + one tile
  int64_t ptile_max = 0;
  size_t total = 0;         // bytes
  int64_t n_tiles = 0;
};

// Returns false when the arguments are out of the supported range.
bool map_layout(int64_t n, int32_t grid_dim, int32_t batch, const MapOptions& opt,
                MapLayout* out);

// Enqueues the map-build kernels (init, [brick allocation,] insert, query) on `stream`.
// Returns the launch error.  Accepts N < kMaxMapRows.
cudaError_t launch_map_build(const int32_t* coords, int64_t n, int32_t grid_dim, int32_t batch,
                             int32_t* nbr, void* workspace, const MapLayout& lay,
                             cudaStream_t stream);

// Activation codes of the forward epilogue (the values of subm3d_act).
enum : int { kActNone = 0, kActGelu = 1, kActSilu = 2 };

// Epilogue of a forward: out = act(acc + bias) + residual (epilogue.cuh).
// bias: [Cout] and residual: [N, Cout] in the feature dtype, each optional; act:
// 0 none, 1 exact GELU, 2 SiLU.  residual may be `out` itself.
struct Epilogue {
  const void* bias = nullptr;
  const void* residual = nullptr;
  int32_t act = 0;
};

// fp32 forward on CUDA-core FMA.
cudaError_t launch_forward_f32(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                               const float* feats, const float* weight, float* out, int32_t cin,
                               int32_t cout, int32_t flip, const Epilogue& epi,
                               cudaStream_t stream);

// What the tensor-core kernels need besides their operands: the library's
// device error word (set to 1 by a CTA whose bounded wait ran out) and the
// limit of each pipeline wait in ns (2 s unless a test asks for less).
struct DeviceCtl {
  int32_t* err_word = nullptr;
  uint64_t wait_limit_ns = 0;
};

// bf16 forward on tcgen05 tensor cores (fp32 accumulation in TMEM).
cudaError_t launch_forward_bf16(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                                const void* feats, const void* weight, void* out, int32_t cin,
                                int32_t cout, int32_t flip, const Epilogue& epi,
                                const DeviceCtl& ctl, cudaStream_t stream);

// bf16 forward over the x-run position layout (forward_bf16_runs_sm100.cu);
// Cin and Cout multiples of 16 (Cin in 64-channel chunks, the last zero-padded).
cudaError_t launch_forward_bf16_runs(const int32_t* pos, const int32_t* etable,
                                     int64_t et_stride, const int32_t* header, int64_t max_tiles,
                                     const void* feats,
                                     const void* weight, void* out, int32_t cin, int32_t cout,
                                     int32_t flip, const Epilogue& epi, const DeviceCtl& ctl,
                                     cudaStream_t stream);

// Backward (backward.cu): W [cout][27][cin] -> W^T [cin][27][cout]; and the
// weight gradient dW [cout][27][cin] fp32 (zeroed, then accumulated).
cudaError_t launch_transpose_weight(const void* w, void* wt, int32_t cout, int32_t cin,
                                    bool bf16, cudaStream_t stream);
cudaError_t launch_wgrad(const int32_t* nbr, int64_t n, const void* x, const void* dy, float* dw,
                         int32_t cin, int32_t cout, int32_t flip, bool bf16, int num_sms,
                         cudaStream_t stream);

// bf16 weight gradient over the x-run layout on tcgen05 (wgrad_bf16_runs_sm100.cu):
// Cin and Cout multiples of 16; zeroes dw, then accumulates.
cudaError_t launch_wgrad_bf16_runs(const int32_t* pos, const int32_t* etable,
                                   int64_t et_stride, const int32_t* header, const void* feats, const void* dy,
                                   float* dw, int32_t cin, int32_t cout, int32_t flip,
                                   const DeviceCtl& ctl, cudaStream_t stream);

// Resolution changes (resample.cu).  Expansion: subdivide (C-order children,
// replicated rows), upsample (masked, axis-0-fastest children, replicated) and
// channel2spatial (masked or not, channel slices); child rows are written
// parent-major.  Its workspace: per-1,024-voxel child counts, a total and, per
// child row, its source (parent * 8 + slot).
struct ExpandLayout {
  int64_t n_blocks = 0;
  size_t cnt_off = 0, total_off = 0, src_off = 0, bytes = 0;
};
ExpandLayout expand_layout(int64_t n);
// Blocking when `mask` is given (the child count is read back); *out_count = rows.
cudaError_t launch_expand(const int32_t* coords, const void* feats, const uint8_t* mask, int64_t n,
                          int64_t in_row_bytes, int64_t out_row_bytes, bool slice, bool c_order,
                          int32_t* out_coords, void* out_feats, void* workspace,
                          int64_t* out_count, cudaStream_t stream);

// Pooling to parents coord // 2 in raster order: max (0), mean (1) or
// spatial2channel (2), through the fine set's map table.  Its workspace: a flag
// per parent cell, per-4,096-cell counts and the total.
struct PoolLayout {
  int32_t G = 0;
  int64_t cells = 0, n_blocks = 0;
  size_t flags_off = 0, cnt_off = 0, total_off = 0, bytes = 0;
};
PoolLayout pool_layout(int64_t n, int32_t grid_dim, int32_t batch);
// Blocking (the parent count is read back); *out_count = parents.
cudaError_t launch_pool(const MapLayout& map_lay, const void* map_ws, int32_t grid_dim,
                        int32_t batch, const int32_t* coords, int64_t n, const void* feats,
                        int32_t channels, bool bf16, int mode, int32_t* out_coords,
                        void* out_feats, void* workspace, int64_t* out_count,
                        cudaStream_t stream);

}  // namespace subm3d

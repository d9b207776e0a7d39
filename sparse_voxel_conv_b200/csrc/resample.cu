// Resolution changes around the submanifold convolution (trellis_sparse_mrp_mlx
// commit log; lato.2_mrp_mlx notes "Key facts"), factor 2:
//
//   expand  subdivide        every voxel -> children 2 * coord + (dz, dy, dx),
//                            C order (s = 4 dz + 2 dy + dx), features replicated;
//           upsample         only the children an [N, 8] 0/1 mask flags, the
//                            child index decoded axis 0 fastest (dz = s % 2,
//                            dy = s / 2 % 2, dx = s / 4 % 2), features replicated;
//           channel2spatial  as upsample (mask optional), child s takes channels
//                            [s C, (s + 1) C) of the parent's 8 C.
//   pool    downsample       parents coord // 2 in raster order, max or mean over
//                            the children present;
//           spatial2channel  parents coord // 2, child s's features in channel
//                            slot s (axis 0 fastest), zeros for absent children.
//
// Expansion lists children parent-major by ascending child index.  With a mask
// the children's output rows come from a scan of the per-voxel child counts
// (blocks of 1,024 voxels: counts, one-block scan of the block counts, emit).
// Pooling marks the parent cells in a dense flag grid over batch x G^3 cells
// (G = ceil(grid / 2)), compacts the marked cells in raster order with the same
// three-step scan, and gathers each parent's children through the fine set's
// neighbour-map table (map_table.cuh): no sort and no atomics on features, so
// max and spatial2channel are exact and mean sums a parent's children in child
// index order.  Features move in 16-byte pieces where the row allows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "map_table.cuh"

namespace subm3d {
namespace {

constexpr int kScanThreads = 256;
constexpr int kExpandPerThread = 4;                                // voxels per thread
constexpr int kExpandBlock = kScanThreads * kExpandPerThread;      // 1,024 voxels
constexpr int kPoolPerThread = 16;                                 // cells per thread
constexpr int kPoolBlock = kScanThreads * kPoolPerThread;          // 4,096 cells

__device__ __forceinline__ void child_offsets(int s, bool c_order, int& dz, int& dy, int& dx) {
  if (c_order) {
    dz = (s >> 2) & 1;
    dy = (s >> 1) & 1;
    dx = s & 1;
  } else {
    dz = s & 1;
    dy = (s >> 1) & 1;
    dx = (s >> 2) & 1;
  }
}

__device__ __forceinline__ uint32_t mask_bits(const uint8_t* mask, int64_t i) {
  uint32_t b = 0;
#pragma unroll
  for (int s = 0; s < 8; ++s) b |= (mask[i * 8 + s] != 0 ? 1u : 0u) << s;
  return b;
}

// Block-wide exclusive scan of one int64 per thread (kScanThreads threads);
// returns this thread's exclusive prefix and, through `total`, the block sum.
__device__ __forceinline__ int64_t block_exclusive_scan(int64_t v, int64_t* total) {
  __shared__ int64_t s_warp[kScanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int64_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int64_t before = 0, sum = 0;
#pragma unroll
  for (int w = 0; w < kScanThreads / 32; ++w) {
    if (w < warp) before += s_warp[w];
    sum += s_warp[w];
  }
  __syncthreads();  // s_warp may be reused by the caller's next scan
  *total = sum;
  return before + incl - v;
}

// One-block exclusive scan of `n` int64 block counts in place; *total = the sum.
__global__ void __launch_bounds__(kScanThreads) scan_block_counts(int64_t* cnt, int64_t n,
                                                                  int64_t* total) {
  int64_t carry = 0;
  for (int64_t base = 0; base < n; base += kScanThreads) {
    const int64_t i = base + threadIdx.x;
    const int64_t v = i < n ? cnt[i] : 0;
    int64_t sum = 0;
    const int64_t ex = block_exclusive_scan(v, &sum);
    if (i < n) cnt[i] = carry + ex;
    carry += sum;
  }
  if (threadIdx.x == 0) *total = carry;
}

// ---------------------------------------------------------------- expand ----

// Children per block of kExpandBlock voxels (masked expansion).
__global__ void __launch_bounds__(kScanThreads) expand_count(const uint8_t* __restrict__ mask,
                                                             int64_t n, int64_t* block_cnt) {
  int64_t c = 0;
#pragma unroll
  for (int q = 0; q < kExpandPerThread; ++q) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kExpandBlock + threadIdx.x * kExpandPerThread + q;
    if (i < n) c += __popc(mask_bits(mask, i));
  }
  int64_t sum = 0;
  block_exclusive_scan(c, &sum);
  if (threadIdx.x == 0) block_cnt[blockIdx.x] = sum;
}

// Child coordinates and, with a mask, each child row's source (parent * 8 +
// slot).  Without a mask every voxel has 8 children at rows 8 i .. 8 i + 7.
__global__ void __launch_bounds__(kScanThreads)
    expand_emit(const int4* __restrict__ coords, const uint8_t* __restrict__ mask, int64_t n,
                const int64_t* __restrict__ block_off, int c_order, int4* __restrict__ out_coords,
                int64_t* __restrict__ child_src) {
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kExpandBlock + threadIdx.x * kExpandPerThread;
  uint32_t bits[kExpandPerThread];
  int64_t mine = 0;
#pragma unroll
  for (int q = 0; q < kExpandPerThread; ++q) {
    const int64_t i = i0 + q;
    bits[q] = i < n ? (mask ? mask_bits(mask, i) : 0xFFu) : 0u;
    mine += __popc(bits[q]);
  }
  int64_t sum = 0;
  int64_t r = block_exclusive_scan(mine, &sum) + (mask ? block_off[blockIdx.x] : 8 * static_cast<int64_t>(blockIdx.x) * kExpandBlock);
#pragma unroll
  for (int q = 0; q < kExpandPerThread; ++q) {
    const int64_t i = i0 + q;
    if (i >= n) break;
    const int4 c = coords[i];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      if (!((bits[q] >> s) & 1u)) continue;
      int dz, dy, dx;
      child_offsets(s, c_order != 0, dz, dy, dx);
      out_coords[r] = make_int4(c.x, 2 * c.y + dz, 2 * c.z + dy, 2 * c.w + dx);
      if (mask) child_src[r] = i * 8 + s;  // without a mask, row r's source is r itself
      ++r;
    }
  }
}

// out_feats[r] = the parent's row (replicate) or its slot's slice.  Each thread
// moves kCopyPieces pieces of PIECE bytes (strided by the grid, so a warp's
// accesses stay contiguous); without a child list (subdivide) row r's parent
// is r / 8 and its slot r % 8.
constexpr int kCopyPieces = 4;

template <int PIECE, bool LIST>
__global__ void __launch_bounds__(256)
    expand_copy(const uint8_t* __restrict__ feats, const int64_t* __restrict__ child_src,
                int64_t rows, int64_t in_row_bytes, int64_t out_row_bytes, int slice,
                uint8_t* __restrict__ out) {
  const int64_t pieces = out_row_bytes / PIECE;
  const int64_t total = rows * pieces;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
#pragma unroll
  for (int k = 0; k < kCopyPieces; ++k) {
    const int64_t t = t0 + k * stride;
    if (t >= total) break;
    const int64_t r = t / pieces, p = t % pieces;
    const int64_t src = LIST ? child_src[r] : r;
    const int64_t parent = src >> 3, slot = src & 7;
    const uint8_t* from =
        feats + parent * in_row_bytes + (slice ? slot * out_row_bytes : 0) + p * PIECE;
    uint8_t* to = out + r * out_row_bytes + p * PIECE;
    if constexpr (PIECE == 16)
      *reinterpret_cast<uint4*>(to) = *reinterpret_cast<const uint4*>(from);
    else if constexpr (PIECE == 4)
      *reinterpret_cast<uint32_t*>(to) = *reinterpret_cast<const uint32_t*>(from);
    else
      *reinterpret_cast<uint16_t*>(to) = *reinterpret_cast<const uint16_t*>(from);
  }
}

// ------------------------------------------------------------------ pool ----

__device__ __forceinline__ int64_t parent_cell(int4 c, int G) {
  return ((static_cast<int64_t>(c.x) * G + (c.y >> 1)) * G + (c.z >> 1)) * G + (c.w >> 1);
}

// Coordinates outside the volume (an invalid map) mark nothing.
__global__ void pool_mark(const int4* __restrict__ coords, int64_t n, int grid, int batch, int G,
                          uint8_t* __restrict__ flags) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int4 c = coords[i];
  if (in_volume(c, grid, batch)) flags[parent_cell(c, G)] = 1;
}

// Marked cells per block of kPoolBlock cells.
__global__ void __launch_bounds__(kScanThreads) pool_count(const uint8_t* __restrict__ flags,
                                                           int64_t cells, int64_t* block_cnt) {
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kPoolBlock + threadIdx.x * kPoolPerThread;
  int64_t c = 0;
#pragma unroll
  for (int q = 0; q < kPoolPerThread; ++q) c += (c0 + q < cells && flags[c0 + q]) ? 1 : 0;
  int64_t sum = 0;
  block_exclusive_scan(c, &sum);
  if (threadIdx.x == 0) block_cnt[blockIdx.x] = sum;
}

// Parents in raster (cell) order: their coordinates and cell indices.
__global__ void __launch_bounds__(kScanThreads)
    pool_emit(const uint8_t* __restrict__ flags, int64_t cells, const int64_t* __restrict__ block_off,
              int G, int4* __restrict__ out_coords, int64_t* __restrict__ parent_cells) {
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kPoolBlock + threadIdx.x * kPoolPerThread;
  uint32_t bits = 0;
#pragma unroll
  for (int q = 0; q < kPoolPerThread; ++q) bits |= (c0 + q < cells && flags[c0 + q] ? 1u : 0u) << q;
  int64_t sum = 0;
  int64_t r = block_exclusive_scan(__popc(bits), &sum) + block_off[blockIdx.x];
  const int64_t g3 = static_cast<int64_t>(G) * G * G;
#pragma unroll
  for (int q = 0; q < kPoolPerThread; ++q) {
    if (!((bits >> q) & 1u)) continue;
    const int64_t cell = c0 + q;
    const int64_t b = cell / g3, rem = cell % g3;
    const int z = static_cast<int>(rem / (static_cast<int64_t>(G) * G));
    const int y = static_cast<int>((rem / G) % G), x = static_cast<int>(rem % G);
    out_coords[r] = make_int4(static_cast<int>(b), z, y, x);
    parent_cells[r] = cell;
    ++r;
  }
}

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

enum : int { kPoolMax = 0, kPoolMean = 1, kPoolS2C = 2 };

// One warp per parent: lanes 0-7 look up the 8 children in the fine map once
// and broadcast their rows; the warp then streams the channels.  max / mean:
// over the children present, in child slot order; spatial2channel: child s's
// row (or zeros) to channel slot s.  Channels move 4 at a time (8 bytes of
// bf16, 16 of fp32: 128 channels fill the warp) when C is a multiple of 4,
// else one at a time.
template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[4]) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  v[0] = __uint_as_float(r.x << 16);
  v[1] = __uint_as_float(r.x & 0xFFFF0000u);
  v[2] = __uint_as_float(r.y << 16);
  v[3] = __uint_as_float(r.y & 0xFFFF0000u);
}
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x;
  v[1] = a.y;
  v[2] = a.z;
  v[3] = a.w;
}
template <typename T>
__device__ __forceinline__ void store4(T* p, const float (&v)[4]);
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[4]) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  *reinterpret_cast<uint2*>(p) =
      make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
}
template <>
__device__ __forceinline__ void store4<float>(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

template <Kind K, int MODE, typename T, bool VEC>
__global__ void __launch_bounds__(256)
    pool_reduce(const int64_t* __restrict__ parent_cells, int64_t parents, Tables tab, int grid,
                int batch, int G, const T* __restrict__ feats, int C, T* __restrict__ out) {
  const int64_t p = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x & 31;
  if (p >= parents) return;  // whole warps leave together
  const int64_t cell = parent_cells[p];
  const int64_t g3 = static_cast<int64_t>(G) * G * G;
  const int b = static_cast<int>(cell / g3);
  const int64_t rem = cell % g3;
  const int Z = static_cast<int>(rem / (static_cast<int64_t>(G) * G));
  const int Y = static_cast<int>((rem / G) % G), X = static_cast<int>(rem % G);
  int32_t my_row = -1;
  if (lane < 8) {  // child slot `lane`, axis 0 fastest
    const int z = 2 * Z + (lane & 1), y = 2 * Y + ((lane >> 1) & 1), x = 2 * X + ((lane >> 2) & 1);
    if (z < grid && y < grid && x < grid && b < batch) my_row = lookup<K>(tab, b, z, y, x, grid);
  }
  int32_t rows[8];
#pragma unroll
  for (int s = 0; s < 8; ++s) rows[s] = __shfl_sync(0xFFFFFFFFu, my_row, s);
  if constexpr (MODE == kPoolS2C) {
    T* o = out + p * 8 * C;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const T* src = rows[s] >= 0 ? feats + static_cast<int64_t>(rows[s]) * C : nullptr;
      if constexpr (VEC) {
        for (int c = lane * 4; c < C; c += 128) {
          float v[4] = {0.f, 0.f, 0.f, 0.f};
          if (src) load4<T>(src + c, v);
          store4<T>(o + s * C + c, v);
        }
      } else {
        for (int c = lane; c < C; c += 32) o[s * C + c] = src ? src[c] : from_f<T>(0.0f);
      }
    }
  } else {
    int count = 0;
#pragma unroll
    for (int s = 0; s < 8; ++s) count += rows[s] >= 0 ? 1 : 0;
    if constexpr (VEC) {
      for (int c = lane * 4; c < C; c += 128) {
        float acc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = MODE == kPoolMax ? -INFINITY : 0.0f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          if (rows[s] < 0) continue;
          float v[4];
          load4<T>(feats + static_cast<int64_t>(rows[s]) * C + c, v);
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[j] = MODE == kPoolMax ? fmaxf(acc[j], v[j]) : acc[j] + v[j];
        }
        if (MODE == kPoolMean) {
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[j] = count > 0 ? acc[j] / static_cast<float>(count) : 0.0f;
        }
        store4<T>(out + p * C + c, acc);
      }
    } else {
      for (int c = lane; c < C; c += 32) {
        float acc = MODE == kPoolMax ? -INFINITY : 0.0f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          if (rows[s] < 0) continue;
          const float v = to_f<T>(feats[static_cast<int64_t>(rows[s]) * C + c]);
          acc = MODE == kPoolMax ? fmaxf(acc, v) : acc + v;
        }
        if (MODE == kPoolMean) acc = count > 0 ? acc / static_cast<float>(count) : 0.0f;
        out[p * C + c] = from_f<T>(acc);
      }
    }
  }
}

template <Kind K, typename T>
cudaError_t launch_reduce(int mode, const int64_t* parent_cells, int64_t parents, const Tables& tab,
                          int grid, int batch, int G, const void* feats, int C, void* out,
                          cudaStream_t stream) {
  if (parents == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((parents * 32 + 255) / 256);
  const auto* f = static_cast<const T*>(feats);
  auto* o = static_cast<T*>(out);
  const size_t align = 4 * sizeof(T);  // one 4-channel piece
  const bool vec = C % 4 == 0 && reinterpret_cast<uintptr_t>(feats) % align == 0 &&
                   reinterpret_cast<uintptr_t>(out) % align == 0;
  auto go = [&](auto kernel) {
    kernel<<<blocks, 256, 0, stream>>>(parent_cells, parents, tab, grid, batch, G, f, C, o);
  };
  if (mode == kPoolMax)
    vec ? go(pool_reduce<K, kPoolMax, T, true>) : go(pool_reduce<K, kPoolMax, T, false>);
  else if (mode == kPoolMean)
    vec ? go(pool_reduce<K, kPoolMean, T, true>) : go(pool_reduce<K, kPoolMean, T, false>);
  else
    vec ? go(pool_reduce<K, kPoolS2C, T, true>) : go(pool_reduce<K, kPoolS2C, T, false>);
  return cudaGetLastError();
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

// ------------------------------------------------------------ host side ----

ExpandLayout expand_layout(int64_t n) {
  ExpandLayout l;
  l.n_blocks = (n + kExpandBlock - 1) / kExpandBlock;
  l.cnt_off = 0;
  l.total_off = align256(static_cast<size_t>(l.n_blocks + 1) * 8);
  l.src_off = l.total_off + 256;
  l.bytes = align256(l.src_off + static_cast<size_t>(8 * n) * 8);
  return l;
}

cudaError_t launch_expand(const int32_t* coords, const void* feats, const uint8_t* mask, int64_t n,
                          int64_t in_row_bytes, int64_t out_row_bytes, bool slice, bool c_order,
                          int32_t* out_coords, void* out_feats, void* workspace,
                          int64_t* out_count, cudaStream_t stream) {
  const ExpandLayout l = expand_layout(n);
  auto* ws = static_cast<uint8_t*>(workspace);
  auto* cnt = reinterpret_cast<int64_t*>(ws + l.cnt_off);
  auto* total = reinterpret_cast<int64_t*>(ws + l.total_off);
  auto* src = reinterpret_cast<int64_t*>(ws + l.src_off);
  const unsigned blocks = static_cast<unsigned>(l.n_blocks);
  int64_t rows = 8 * n;
  cudaError_t e;
  if (mask) {
    expand_count<<<blocks, kScanThreads, 0, stream>>>(mask, n, cnt);
    scan_block_counts<<<1, kScanThreads, 0, stream>>>(cnt, l.n_blocks, total);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaMemcpyAsync(&rows, total, sizeof(rows), cudaMemcpyDeviceToHost, stream)) !=
            cudaSuccess ||
        (e = cudaStreamSynchronize(stream)) != cudaSuccess)
      return e;
  }
  *out_count = rows;
  expand_emit<<<blocks, kScanThreads, 0, stream>>>(reinterpret_cast<const int4*>(coords), mask, n,
                                                   cnt, c_order ? 1 : 0,
                                                   reinterpret_cast<int4*>(out_coords), src);
  if ((e = cudaGetLastError()) != cudaSuccess || rows == 0) return e;
  const auto* f = static_cast<const uint8_t*>(feats);
  auto* o = static_cast<uint8_t*>(out_feats);
  const bool a16 = out_row_bytes % 16 == 0 && in_row_bytes % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(feats) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(out_feats) % 16 == 0;
  const bool a4 = out_row_bytes % 4 == 0 && in_row_bytes % 4 == 0 &&
                  reinterpret_cast<uintptr_t>(feats) % 4 == 0 &&
                  reinterpret_cast<uintptr_t>(out_feats) % 4 == 0;
  const int piece = a16 ? 16 : (a4 ? 4 : 2);
  const int64_t work = rows * (out_row_bytes / piece);
  const unsigned cblocks =
      static_cast<unsigned>((work + 256 * kCopyPieces - 1) / (256 * kCopyPieces));
  auto go = [&](auto kernel) {
    kernel<<<cblocks, 256, 0, stream>>>(f, src, rows, in_row_bytes, out_row_bytes, slice ? 1 : 0,
                                        o);
  };
  const bool list = mask != nullptr;
  if (piece == 16)
    list ? go(expand_copy<16, true>) : go(expand_copy<16, false>);
  else if (piece == 4)
    list ? go(expand_copy<4, true>) : go(expand_copy<4, false>);
  else
    list ? go(expand_copy<2, true>) : go(expand_copy<2, false>);
  return cudaGetLastError();
}

PoolLayout pool_layout(int64_t n, int32_t grid_dim, int32_t batch) {
  PoolLayout l;
  l.G = (grid_dim + 1) / 2;
  l.cells = static_cast<int64_t>(batch) * l.G * l.G * l.G;
  l.n_blocks = (l.cells + kPoolBlock - 1) / kPoolBlock;
  l.flags_off = 0;
  l.cnt_off = align256(static_cast<size_t>(l.cells));
  l.total_off = align256(l.cnt_off + static_cast<size_t>(l.n_blocks + 1) * 8);
  l.cells_off = l.total_off + 256;
  l.bytes = align256(l.cells_off + static_cast<size_t>(n > 0 ? n : 1) * 8);
  return l;
}

cudaError_t launch_pool(const MapLayout& map_lay, const void* map_ws, int32_t grid_dim,
                        int32_t batch, const int32_t* coords, int64_t n, const void* feats,
                        int32_t channels, bool bf16, int mode, int32_t* out_coords,
                        void* out_feats, void* workspace, int64_t* out_count,
                        cudaStream_t stream) {
  const PoolLayout l = pool_layout(n, grid_dim, batch);
  auto* ws = static_cast<uint8_t*>(workspace);
  auto* flags = ws + l.flags_off;
  auto* cnt = reinterpret_cast<int64_t*>(ws + l.cnt_off);
  auto* total = reinterpret_cast<int64_t*>(ws + l.total_off);
  auto* pcells = reinterpret_cast<int64_t*>(ws + l.cells_off);
  cudaError_t e = cudaMemsetAsync(flags, 0, static_cast<size_t>(l.cells), stream);
  if (e != cudaSuccess) return e;
  if (n > 0)
    pool_mark<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
        reinterpret_cast<const int4*>(coords), n, grid_dim, batch, l.G, flags);
  const unsigned blocks = static_cast<unsigned>(l.n_blocks);
  pool_count<<<blocks, kScanThreads, 0, stream>>>(flags, l.cells, cnt);
  scan_block_counts<<<1, kScanThreads, 0, stream>>>(cnt, l.n_blocks, total);
  pool_emit<<<blocks, kScanThreads, 0, stream>>>(flags, l.cells, cnt, l.G,
                                                 reinterpret_cast<int4*>(out_coords), pcells);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int64_t parents = 0;
  if ((e = cudaMemcpyAsync(&parents, total, sizeof(parents), cudaMemcpyDeviceToHost, stream)) !=
          cudaSuccess ||
      (e = cudaStreamSynchronize(stream)) != cudaSuccess)
    return e;
  *out_count = parents;
  const uint8_t* mws = static_cast<const uint8_t*>(map_ws);
  Tables t{};
  t.capmask = static_cast<uint32_t>(map_lay.capacity - 1);
  if (map_lay.kind == MapKind::kDirect) {
    t.cells = reinterpret_cast<const int32_t*>(mws + map_lay.table_off);
    return bf16 ? launch_reduce<Kind::kDirect, __nv_bfloat16>(mode, pcells, parents, t, grid_dim,
                                                              batch, l.G, feats, channels,
                                                              out_feats, stream)
                : launch_reduce<Kind::kDirect, float>(mode, pcells, parents, t, grid_dim, batch,
                                                      l.G, feats, channels, out_feats, stream);
  }
  t.table = reinterpret_cast<const unsigned long long*>(mws + map_lay.table_off);
  if (map_lay.compact)
    return bf16 ? launch_reduce<Kind::kCompact, __nv_bfloat16>(mode, pcells, parents, t,
                                                               grid_dim, batch, l.G, feats,
                                                               channels, out_feats, stream)
                : launch_reduce<Kind::kCompact, float>(mode, pcells, parents, t, grid_dim, batch,
                                                       l.G, feats, channels, out_feats, stream);
  t.rows = reinterpret_cast<const int32_t*>(mws + map_lay.rows_off);
  return bf16 ? launch_reduce<Kind::kWide, __nv_bfloat16>(mode, pcells, parents, t, grid_dim,
                                                          batch, l.G, feats, channels, out_feats,
                                                          stream)
              : launch_reduce<Kind::kWide, float>(mode, pcells, parents, t, grid_dim, batch, l.G,
                                                  feats, channels, out_feats, stream);
}

}  // namespace subm3d

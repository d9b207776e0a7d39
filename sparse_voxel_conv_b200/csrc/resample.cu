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

// out_feats[r] = the parent's row (replicate) or its slot's slice.  A warp
// takes 8 consecutive output rows per step (grid-stride over such chunks): L
// lanes per row (L the power of two >= the row's pieces, at most 32), 32 / L
// rows at a time.  Without a child list (subdivide, or channel2spatial on all
// children) chunk c is exactly voxel c's children, so the warp also writes their
// coordinates and, when replicating a row of at most 32 pieces, loads the
// parent's pieces once for all 8 rows.
template <typename P, bool LIST>
__global__ void __launch_bounds__(256)
    expand_rows(const int4* __restrict__ coords, const P* __restrict__ feats,
                const int64_t* __restrict__ child_src, int64_t rows, int in_ppr, int ppr,
                int lanes_per_row, int slice, int c_order, int4* __restrict__ out_coords,
                P* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int L = lanes_per_row, sub0 = lane / L, j0 = lane % L;
  const int64_t chunks = (rows + 7) / 8;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
  for (int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; c < chunks;
       c += warps) {
    if constexpr (!LIST) {
      if (lane < 8) {  // chunk c = voxel c's 8 children
        const int4 pc = __ldg(coords + c);
        int dz, dy, dx;
        child_offsets(lane, c_order != 0, dz, dy, dx);
        out_coords[8 * c + lane] = make_int4(pc.x, 2 * pc.y + dz, 2 * pc.z + dy, 2 * pc.w + dx);
      }
      if (!slice && ppr <= 32) {  // every row of the chunk is the parent's row
        if (j0 < ppr) {
          const P v = __ldg(feats + c * in_ppr + j0);
          P* dst = out + (8 * c) * ppr + j0;
#pragma unroll
          for (int sub = sub0; sub < 8; sub += 32 / L) dst[static_cast<int64_t>(sub) * ppr] = v;
        }
        continue;
      }
    }
    for (int sub = sub0; sub < 8; sub += 32 / L) {
      const int64_t r = 8 * c + sub;
      if (r >= rows) break;
      const int64_t src = LIST ? __ldg(child_src + r) : r;
      const P* from = feats + (src >> 3) * in_ppr + (slice ? (src & 7) * ppr : 0);
      P* to = out + r * ppr;
      for (int j = j0; j < ppr; j += L) to[j] = __ldg(from + j);
    }
  }
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cached[dev] = v;
  }
  return cached[dev];
}

// Blocks for a grid-stride kernel of 256 threads over `work_warps` warp-sized
// items: enough for 8 resident blocks per SM, fewer when there is less work.
unsigned stride_blocks(int64_t work_warps) {
  const int64_t want = (work_warps + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
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

// Flags of cells c0 .. c0 + 15 (c0 a multiple of 16) as bits, one 16-byte load:
// the flag region is padded to 256 bytes, and bits at or past `cells` (bytes
// the clear does not cover) are dropped.
static_assert(kPoolPerThread == 16, "one 16-byte flag load per thread");
__device__ __forceinline__ uint32_t flag_bits(const uint8_t* __restrict__ flags, int64_t c0,
                                              int64_t cells) {
  if (c0 >= cells) return 0u;
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(flags + c0));
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  uint32_t bits = 0;
#pragma unroll
  for (int q = 0; q < 16; ++q) bits |= ((words[q >> 2] >> (8 * (q & 3))) & 0xFFu ? 1u : 0u) << q;
  const int64_t left = cells - c0;
  return left >= 16 ? bits : bits & ((1u << left) - 1u);
}

// Marked cells per block of kPoolBlock cells.
__global__ void __launch_bounds__(kScanThreads) pool_count(const uint8_t* __restrict__ flags,
                                                           int64_t cells, int64_t* block_cnt) {
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kPoolBlock + threadIdx.x * kPoolPerThread;
  int64_t sum = 0;
  block_exclusive_scan(__popc(flag_bits(flags, c0, cells)), &sum);
  if (threadIdx.x == 0) block_cnt[blockIdx.x] = sum;
}

// Parents in raster (cell) order: their coordinates.
__global__ void __launch_bounds__(kScanThreads)
    pool_emit(const uint8_t* __restrict__ flags, int64_t cells, const int64_t* __restrict__ block_off,
              int G, int4* __restrict__ out_coords) {
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kPoolBlock + threadIdx.x * kPoolPerThread;
  uint32_t bits = flag_bits(flags, c0, cells);
  int64_t sum = 0;
  int64_t r = block_exclusive_scan(__popc(bits), &sum) + block_off[blockIdx.x];
  // cells < 2^30 (the workspace query refuses more): 32-bit decode
  const uint32_t g = static_cast<uint32_t>(G);
  while (bits) {
    const int q = __ffs(bits) - 1;
    bits &= bits - 1u;
    uint32_t cell = static_cast<uint32_t>(c0 + q);
    const uint32_t x = cell % g;
    cell /= g;
    const uint32_t y = cell % g;
    cell /= g;
    const uint32_t z = cell % g;
    out_coords[r] = make_int4(static_cast<int>(cell / g), static_cast<int>(z),
                              static_cast<int>(y), static_cast<int>(x));
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

// A warp takes 4 parents at a time (grid-stride; the parent count is read from
// device memory, so no host round trip precedes the launch).  Lane l serves
// parent l / 8: it looks up child slot l % 8 in the fine map (axis 0 fastest),
// takes the parent's 8 child rows from its 7 partner lanes, and then moves the
// row's 16-byte pieces l % 8, l % 8 + 8, ...: one load per child, so the 4
// parents' 32 child rows are in flight together.  max / mean: over the children
// present, in child slot order; spatial2channel: child s's row (or zeros) to
// channel slot s.  Rows whose size or address is not a multiple of 16 bytes go
// one channel per lane instead.
// 16 bytes of channels: kN of them, unpacked to fp32 one at a time.
template <typename T>
struct Piece;
template <>
struct Piece<__nv_bfloat16> {
  static constexpr int kN = 8;
  static __device__ __forceinline__ float get(const uint4& r, int k) {
    const uint32_t w = k < 2 ? r.x : (k < 4 ? r.y : (k < 6 ? r.z : r.w));
    return __uint_as_float((k & 1) ? (w & 0xFFFF0000u) : (w << 16));
  }
  static __device__ __forceinline__ uint4 pack(const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Piece<float> {
  static constexpr int kN = 4;
  static __device__ __forceinline__ float get(const uint4& r, int k) {
    return __uint_as_float(k == 0 ? r.x : (k == 1 ? r.y : (k == 2 ? r.z : r.w)));
  }
  static __device__ __forceinline__ uint4 pack(const float (&v)[4]) {
    return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                      __float_as_uint(v[3]));
  }
};

// Parent p's output from its child rows (-1: absent); `j0`, `step`: the pieces
// (VEC) or channels (scalar) this lane moves.
template <int MODE, typename T, bool VEC>
__device__ __forceinline__ void pool_parent(const int32_t (&rows)[8], int64_t p, int j0, int step,
                                            const T* __restrict__ feats, int C,
                                            T* __restrict__ out) {
  int count = 0;
#pragma unroll
  for (int s = 0; s < 8; ++s) count += rows[s] >= 0 ? 1 : 0;
  if constexpr (VEC) {
    using Pc = Piece<T>;
    constexpr int W = Pc::kN;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
    for (int c = j0 * W; c < C; c += step * W) {
      uint4 r[8];  // the children's pieces, all loads in flight together
#pragma unroll
      for (int s = 0; s < 8; ++s)
        r[s] = rows[s] >= 0
                   ? __ldg(reinterpret_cast<const uint4*>(feats + static_cast<int64_t>(rows[s]) * C + c))
                   : zero;
      if constexpr (MODE == kPoolS2C) {
#pragma unroll
        for (int s = 0; s < 8; ++s) *reinterpret_cast<uint4*>(out + (p * 8 + s) * C + c) = r[s];
      } else {
        float acc[W];
#pragma unroll
        for (int k = 0; k < W; ++k) acc[k] = MODE == kPoolMax ? -INFINITY : 0.0f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          if (rows[s] < 0) continue;
#pragma unroll
          for (int k = 0; k < W; ++k)
            acc[k] = MODE == kPoolMax ? fmaxf(acc[k], Pc::get(r[s], k)) : acc[k] + Pc::get(r[s], k);
        }
        if (MODE == kPoolMean) {
#pragma unroll
          for (int k = 0; k < W; ++k)
            acc[k] = count > 0 ? acc[k] / static_cast<float>(count) : 0.0f;
        }
        *reinterpret_cast<uint4*>(out + p * C + c) = Pc::pack(acc);
      }
    }
  } else {
    for (int c = j0; c < C; c += step) {
      if constexpr (MODE == kPoolS2C) {
#pragma unroll
        for (int s = 0; s < 8; ++s)
          out[(p * 8 + s) * C + c] =
              rows[s] >= 0 ? feats[static_cast<int64_t>(rows[s]) * C + c] : from_f<T>(0.0f);
      } else {
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

template <Kind K, int MODE, typename T, bool VEC>
__global__ void __launch_bounds__(256, 4)
    pool_reduce(const int4* __restrict__ parent_coords, const int64_t* __restrict__ parent_count,
                Tables tab, int grid, int batch, const T* __restrict__ feats, int C,
                T* __restrict__ out) {
  constexpr int kGroup = 4;  // parents per warp step, 8 lanes each
  const int lane = threadIdx.x & 31, g = lane >> 3, j = lane & 7;
  const int64_t parents = __ldg(parent_count);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
  for (int64_t p0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32 * kGroup;
       p0 < parents; p0 += warps * kGroup) {
    const int64_t p = p0 + g;
    int32_t my_row = -1;
    if (p < parents) {
      const int4 pc = __ldg(parent_coords + p);
      const int z = 2 * pc.y + (j & 1), y = 2 * pc.z + ((j >> 1) & 1), x = 2 * pc.w + ((j >> 2) & 1);
      if (z < grid && y < grid && x < grid && pc.x < batch)
        my_row = lookup<K>(tab, pc.x, z, y, x, grid);
    }
    int32_t rows[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) rows[s] = __shfl_sync(0xFFFFFFFFu, my_row, (g << 3) + s);
    if (p < parents) pool_parent<MODE, T, VEC>(rows, p, j, 8, feats, C, out);
  }
}

template <Kind K, typename T>
cudaError_t launch_reduce(int mode, const int4* parent_coords, const int64_t* parent_count,
                          int64_t max_parents, const Tables& tab, int grid, int batch,
                          const void* feats, int C, void* out, cudaStream_t stream) {
  if (max_parents == 0) return cudaSuccess;
  const unsigned blocks = stride_blocks((max_parents + 3) / 4);
  const auto* f = static_cast<const T*>(feats);
  auto* o = static_cast<T*>(out);
  // 16-byte pieces: C a multiple of 8 (bf16) or 4 (fp32), both buffers aligned
  const bool vec = (static_cast<size_t>(C) * sizeof(T)) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(feats) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(out) % 16 == 0;
  auto go = [&](auto kernel) {
    kernel<<<blocks, 256, 0, stream>>>(parent_coords, parent_count, tab, grid, batch, f, C, o);
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
  const bool list = mask != nullptr;
  if (list)  // coordinates and each child row's source; without a mask expand_rows writes both
    expand_emit<<<blocks, kScanThreads, 0, stream>>>(reinterpret_cast<const int4*>(coords), mask,
                                                     n, cnt, c_order ? 1 : 0,
                                                     reinterpret_cast<int4*>(out_coords), src);
  if ((e = cudaGetLastError()) != cudaSuccess || rows == 0) return e;
  const bool a16 = out_row_bytes % 16 == 0 && in_row_bytes % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(feats) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(out_feats) % 16 == 0;
  const bool a4 = out_row_bytes % 4 == 0 && in_row_bytes % 4 == 0 &&
                  reinterpret_cast<uintptr_t>(feats) % 4 == 0 &&
                  reinterpret_cast<uintptr_t>(out_feats) % 4 == 0;
  const int piece = a16 ? 16 : (a4 ? 4 : 2);
  const int ppr = static_cast<int>(out_row_bytes / piece);
  const int in_ppr = static_cast<int>(in_row_bytes / piece);
  int lanes = 1;
  while (lanes < ppr && lanes < 32) lanes <<= 1;
  const unsigned cblocks = stride_blocks((rows + 7) / 8);
  auto go = [&](auto kernel, auto piece_type) {
    using P = decltype(piece_type);
    kernel<<<cblocks, 256, 0, stream>>>(
        reinterpret_cast<const int4*>(coords), static_cast<const P*>(feats), src, rows, in_ppr,
        ppr, lanes, slice ? 1 : 0, c_order ? 1 : 0, reinterpret_cast<int4*>(out_coords),
        static_cast<P*>(out_feats));
  };
  if (piece == 16)
    list ? go(expand_rows<uint4, true>, uint4{}) : go(expand_rows<uint4, false>, uint4{});
  else if (piece == 4)
    list ? go(expand_rows<uint32_t, true>, uint32_t{}) : go(expand_rows<uint32_t, false>, uint32_t{});
  else
    list ? go(expand_rows<uint16_t, true>, uint16_t{}) : go(expand_rows<uint16_t, false>, uint16_t{});
  return cudaGetLastError();
}

PoolLayout pool_layout(int64_t n, int32_t grid_dim, int32_t batch) {
  (void)n;
  PoolLayout l;
  l.G = (grid_dim + 1) / 2;
  l.cells = static_cast<int64_t>(batch) * l.G * l.G * l.G;
  l.n_blocks = (l.cells + kPoolBlock - 1) / kPoolBlock;
  l.flags_off = 0;
  l.cnt_off = align256(static_cast<size_t>(l.cells));
  l.total_off = align256(l.cnt_off + static_cast<size_t>(l.n_blocks + 1) * 8);
  l.bytes = l.total_off + 256;
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
  cudaError_t e = cudaMemsetAsync(flags, 0, static_cast<size_t>(l.cells), stream);
  if (e != cudaSuccess) return e;
  if (n > 0)
    pool_mark<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
        reinterpret_cast<const int4*>(coords), n, grid_dim, batch, l.G, flags);
  const unsigned blocks = static_cast<unsigned>(l.n_blocks);
  pool_count<<<blocks, kScanThreads, 0, stream>>>(flags, l.cells, cnt);
  scan_block_counts<<<1, kScanThreads, 0, stream>>>(cnt, l.n_blocks, total);
  pool_emit<<<blocks, kScanThreads, 0, stream>>>(flags, l.cells, cnt, l.G,
                                                 reinterpret_cast<int4*>(out_coords));
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // the reduction reads the parent count on the device (there are at most N)
  const auto* pc = reinterpret_cast<const int4*>(out_coords);
  const uint8_t* mws = static_cast<const uint8_t*>(map_ws);
  Tables t{};
  t.capmask = static_cast<uint32_t>(map_lay.capacity - 1);
  if (map_lay.kind == MapKind::kDirect) {
    t.cells = reinterpret_cast<const int32_t*>(mws + map_lay.table_off);
    e = bf16 ? launch_reduce<Kind::kDirect, __nv_bfloat16>(mode, pc, total, n, t, grid_dim, batch,
                                                           feats, channels, out_feats, stream)
             : launch_reduce<Kind::kDirect, float>(mode, pc, total, n, t, grid_dim, batch, feats,
                                                   channels, out_feats, stream);
  } else if (map_lay.kind == MapKind::kBrick) {
    t.rows = reinterpret_cast<const int32_t*>(mws + map_lay.table_off);   // directory
    t.cells = reinterpret_cast<const int32_t*>(mws + map_lay.rows_off);   // blocks
    t.bgx = map_lay.bgx;
    t.bgy = map_lay.bgy;
    t.bgz = map_lay.bgz;
    e = bf16 ? launch_reduce<Kind::kBrick, __nv_bfloat16>(mode, pc, total, n, t, grid_dim, batch,
                                                          feats, channels, out_feats, stream)
             : launch_reduce<Kind::kBrick, float>(mode, pc, total, n, t, grid_dim, batch, feats,
                                                  channels, out_feats, stream);
  } else if (map_lay.compact) {
    t.table = reinterpret_cast<const unsigned long long*>(mws + map_lay.table_off);
    e = bf16 ? launch_reduce<Kind::kCompact, __nv_bfloat16>(mode, pc, total, n, t, grid_dim,
                                                            batch, feats, channels, out_feats,
                                                            stream)
             : launch_reduce<Kind::kCompact, float>(mode, pc, total, n, t, grid_dim, batch, feats,
                                                    channels, out_feats, stream);
  } else {
    t.table = reinterpret_cast<const unsigned long long*>(mws + map_lay.table_off);
    t.rows = reinterpret_cast<const int32_t*>(mws + map_lay.rows_off);
    e = bf16 ? launch_reduce<Kind::kWide, __nv_bfloat16>(mode, pc, total, n, t, grid_dim, batch,
                                                         feats, channels, out_feats, stream)
             : launch_reduce<Kind::kWide, float>(mode, pc, total, n, t, grid_dim, batch, feats,
                                                 channels, out_feats, stream);
  }
  if (e != cudaSuccess) return e;
  int64_t parents = 0;
  if ((e = cudaMemcpyAsync(&parents, total, sizeof(parents), cudaMemcpyDeviceToHost, stream)) !=
          cudaSuccess ||
      (e = cudaStreamSynchronize(stream)) != cudaSuccess)
    return e;
  *out_count = parents;
  return cudaSuccess;
}

}  // namespace subm3d

// Backward of the submanifold 3x3x3 convolution.
//
// Input gradient.  With out[i] = sum_k Wf[:, k, :] . x[nbr[i][k]], the gradient
// of x[j] collects Wf[:, k, :]^T dy[i] over every (i, k) with nbr[i][k] = j.
// The map is symmetric, nbr[i][k] = j <=> nbr[j][26-k] = i, so
//   dx[j] = sum_k V[:, k, :] . dy[nbr[j][k]],   V[c][k][o] = Wf[o][26-k][c],
// which is the forward itself on dy with the transposed weight W^T[c][k][o] =
// W[o][k][c] and the opposite orientation.  transpose_weight() writes W^T and
// the forward kernels do the rest (tensor cores for bf16).
//
// Weight gradient.  dW[o][kw][c] = sum_i dy[i][o] * x[nbr[i][k]][c], kw = k or
// 26-k under flip: for each offset a [Cout x N] . [N x Cin] product whose
// reduction runs over the voxels.  wgrad_kernel: a block takes a 128 x 128
// (o, c) tile of one offset and a slice of the voxels, stages 32-voxel slices of
// dy and of the gathered x rows (zero where nbr = -1) in shared memory,
// accumulates an 8 x 8 fp32 register tile per thread and adds the block's
// partial tile into the fp32 dW with atomics (dW is zeroed first).  CUDA-core
// FMA; bf16 inputs are widened to fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace subm3d {
namespace {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// W [cout][27][cin] -> W^T [cin][27][cout], one 32 x 32 tile per block.
template <typename T>
__global__ void __launch_bounds__(256) transpose_weight_kernel(const T* __restrict__ w,
                                                               T* __restrict__ wt, int cout,
                                                               int cin) {
  __shared__ T tile[32][33];
  const int k = blockIdx.z;
  const int c0 = blockIdx.x * 32, o0 = blockIdx.y * 32;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;  // 32 x 8 threads
  for (int r = ty; r < 32; r += 8) {
    const int o = o0 + r, c = c0 + tx;
    if (o < cout && c < cin) tile[r][tx] = w[(static_cast<int64_t>(o) * 27 + k) * cin + c];
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int c = c0 + r, o = o0 + tx;
    if (o < cout && c < cin) wt[(static_cast<int64_t>(c) * 27 + k) * cout + o] = tile[tx][r];
  }
}

// Weight-gradient tile: 128 output x 128 input channels of one offset per block,
// 256 threads with an 8 x 8 register tile each (o = 4 ty .. 4 ty + 3 and
// 64 + 4 ty ..; c likewise with tx), K = the voxels of the block's slice in
// steps of 32.  Both operands are voxel-major rows -- dy[i][o0 ..] and the
// gathered x[nbr[i][k]][c0 ..] (zero where nbr = -1) -- so a step stages them
// with 16-byte stores as they come, in two shared buffers; the next step loads
// into registers in four 8-voxel parts while this step's FMAs run.
constexpr int WB = 128, WK = 32, WT = 256, WP = 8;
constexpr int kWgradFloats = WK * WB;                       // one operand, one buffer
constexpr size_t kWgradSmemBytes = 4 * kWgradFloats * 4;    // two operands x two buffers

// Four consecutive values at p (converted to fp32), zeros where past `limit`.
template <typename T, bool VEC>
__device__ __forceinline__ float4 load4_row(const T* __restrict__ p, int first, int limit) {
  if (first >= limit) return make_float4(0.f, 0.f, 0.f, 0.f);
  if constexpr (VEC) {
    if constexpr (sizeof(T) == 4) {
      return __ldg(reinterpret_cast<const float4*>(p));
    } else {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
      return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xFFFF0000u),
                         __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xFFFF0000u));
    }
  } else {
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = first + j < limit ? to_f32(p[j]) : 0.f;
    return make_float4(v[0], v[1], v[2], v[3]);
  }
}

// Two fp32 FMAs in one instruction (each lane of the pair rounded as fmaf):
// d = a * b + c on (lo, hi) pairs held in 64-bit registers.
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                  unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
  return (static_cast<unsigned long long>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}

template <typename T, bool VEC>
__global__ void __launch_bounds__(WT, 2)
    wgrad_kernel(const int32_t* __restrict__ nbr, int64_t n, const T* __restrict__ x,
                 const T* __restrict__ dy, float* __restrict__ dw, int cin, int cout, int flip,
                 int64_t rows_per_split) {
  extern __shared__ float4 smem_w4[];
  auto s_a = reinterpret_cast<float (*)[WK][WB]>(smem_w4);                       // [2] dy
  auto s_b = reinterpret_cast<float (*)[WK][WB]>(reinterpret_cast<float*>(smem_w4) +
                                                 2 * kWgradFloats);             // [2] x
  const int k = blockIdx.y;
  const int n_ct = (cin + WB - 1) / WB;
  const int o0 = (blockIdx.x / n_ct) * WB, c0 = (blockIdx.x % n_ct) * WB;
  const int64_t i_begin = static_cast<int64_t>(blockIdx.z) * rows_per_split;
  const int64_t i_end = i_begin + rows_per_split < n ? i_begin + rows_per_split : n;
  const int steps = static_cast<int>((i_end - i_begin + WK - 1) / WK);
  const int t = threadIdx.x;
  // staging role: voxel t / 32 of the part, channels 4 (t % 32) .. + 3
  const int sv = t >> 5, sg = (t & 31) * 4;
  // compute role
  const int ty = t >> 4, tx = t & 15;

  float4 ra, rb;
  auto fetch = [&](int step, int part) {
    const int v = part * WP + sv;
    const int64_t i = i_begin + static_cast<int64_t>(step) * WK + v;
    if (i < i_end) {
      ra = load4_row<T, VEC>(dy + i * cout + o0 + sg, o0 + sg, cout);
      const int32_t j = __ldg(nbr + i * kKvol + k);
      rb = j >= 0 ? load4_row<T, VEC>(x + static_cast<int64_t>(j) * cin + c0 + sg, c0 + sg, cin)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      ra = rb = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto stage = [&](int buf, int part) {
    const int v = part * WP + sv;
    *reinterpret_cast<float4*>(&s_a[buf][v][sg]) = ra;
    *reinterpret_cast<float4*>(&s_b[buf][v][sg]) = rb;
  };
  // accumulator pairs: acc2[m][p] holds columns 2p, 2p + 1 of row m
  unsigned long long acc2[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m)
#pragma unroll
    for (int p = 0; p < 4; ++p) acc2[m][p] = 0ull;

  if (steps > 0) {
#pragma unroll 1
    for (int part = 0; part < WK / WP; ++part) {
      fetch(0, part);
      stage(0, part);
    }
    __syncthreads();
  }
  for (int s = 0; s < steps; ++s) {
    const int buf = s & 1;
    const bool more = s + 1 < steps;
#pragma unroll
    for (int part = 0; part < WK / WP; ++part) {
      if (more) fetch(s + 1, part);
#pragma unroll
      for (int q = 0; q < WP; ++q) {
        const int kk = part * WP + q;
        const float4 a0 = *reinterpret_cast<const float4*>(&s_a[buf][kk][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&s_a[buf][kk][64 + ty * 4]);
        const ulonglong2 b0 = *reinterpret_cast<const ulonglong2*>(&s_b[buf][kk][tx * 4]);
        const ulonglong2 b1 = *reinterpret_cast<const ulonglong2*>(&s_b[buf][kk][64 + tx * 4]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const unsigned long long bp[4] = {b0.x, b0.y, b1.x, b1.y};
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const unsigned long long am = pack2(av[m], av[m]);
#pragma unroll
          for (int p = 0; p < 4; ++p) acc2[m][p] = fma2(am, bp[p], acc2[m][p]);
        }
      }
      if (more) stage(buf ^ 1, part);
    }
    __syncthreads();
  }
  const int kw = flip ? 26 - k : k;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int o = o0 + (m < 4 ? ty * 4 + m : 64 + ty * 4 + m - 4);
    if (o >= cout) continue;
    float* row = dw + (static_cast<int64_t>(o) * kKvol + kw) * cin;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int c = c0 + (r < 4 ? tx * 4 + r : 64 + tx * 4 + r - 4);
      const unsigned long long pr = acc2[m][r >> 1];
      if (c < cin)
        atomicAdd(row + c, __uint_as_float(static_cast<uint32_t>((r & 1) ? (pr >> 32) : pr)));
    }
  }
}

template <typename T, bool VEC>
cudaError_t launch_wgrad_kernel(dim3 grid, cudaStream_t stream, const int32_t* nbr, int64_t n,
                                const void* x, const void* dy, float* dw, int cin, int cout,
                                int flip, int64_t rows) {
  static bool attr_set[64] = {};  // per device and instantiation; a repeat set is harmless
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(wgrad_kernel<T, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kWgradSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  wgrad_kernel<T, VEC><<<grid, WT, kWgradSmemBytes, stream>>>(
      nbr, n, static_cast<const T*>(x), static_cast<const T*>(dy), dw, cin, cout, flip, rows);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_transpose_weight(const void* w, void* wt, int32_t cout, int32_t cin,
                                    bool bf16, cudaStream_t stream) {
  const dim3 grid((cin + 31) / 32, (cout + 31) / 32, kKvol);
  if (bf16)
    transpose_weight_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(w), static_cast<__nv_bfloat16*>(wt), cout, cin);
  else
    transpose_weight_kernel<float><<<grid, 256, 0, stream>>>(
        static_cast<const float*>(w), static_cast<float*>(wt), cout, cin);
  return cudaGetLastError();
}

cudaError_t launch_wgrad(const int32_t* nbr, int64_t n, const void* x, const void* dy, float* dw,
                         int32_t cin, int32_t cout, int32_t flip, bool bf16, int num_sms,
                         cudaStream_t stream) {
  cudaError_t e =
      cudaMemsetAsync(dw, 0, static_cast<size_t>(cout) * kKvol * cin * sizeof(float), stream);
  if (e != cudaSuccess || n == 0) return e;
  const int tiles = ((cout + WB - 1) / WB) * ((cin + WB - 1) / WB);
  // split the voxels so that the grid covers the SMs (two blocks each) about 4 times
  int64_t splits = (static_cast<int64_t>(num_sms) * 8 + tiles * kKvol - 1) / (tiles * kKvol);
  if (splits < 1) splits = 1;
  int64_t rows = (n + splits - 1) / splits;
  rows = (rows + WK - 1) / WK * WK;
  splits = (n + rows - 1) / rows;
  const dim3 grid(static_cast<unsigned>(tiles), kKvol, static_cast<unsigned>(splits));
  // 16-byte (fp32) or 8-byte (bf16) row pieces where the rows allow
  const size_t esz = bf16 ? 2 : 4;
  const bool vec = cin % 4 == 0 && cout % 4 == 0 &&
                   reinterpret_cast<uintptr_t>(x) % (4 * esz) == 0 &&
                   reinterpret_cast<uintptr_t>(dy) % (4 * esz) == 0;
  if (bf16)
    return vec ? launch_wgrad_kernel<__nv_bfloat16, true>(grid, stream, nbr, n, x, dy, dw, cin,
                                                         cout, flip, rows)
               : launch_wgrad_kernel<__nv_bfloat16, false>(grid, stream, nbr, n, x, dy, dw, cin,
                                                          cout, flip, rows);
  return vec ? launch_wgrad_kernel<float, true>(grid, stream, nbr, n, x, dy, dw, cin, cout, flip,
                                                rows)
             : launch_wgrad_kernel<float, false>(grid, stream, nbr, n, x, dy, dw, cin, cout, flip,
                                                 rows);
}

}  // namespace subm3d

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
// reduction runs over the voxels.  wgrad_kernel: a block takes a 64 x 64 (o, c)
// tile of one offset and a slice of the voxels, stages 16-voxel slices of dy and
// of the gathered x rows (zero where nbr = -1) in shared memory, accumulates a
// 4 x 4 fp32 register tile per thread and adds the block's partial tile into
// the fp32 dW with atomics (dW is zeroed first).  CUDA-core FMA; bf16 inputs are
// widened to fp32.
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

constexpr int WB = 64, WK = 16, WT = 256;  // tile 64 x 64, 16 voxels per slice, 256 threads

template <typename T>
__global__ void __launch_bounds__(WT)
    wgrad_kernel(const int32_t* __restrict__ nbr, int64_t n, const T* __restrict__ x,
                 const T* __restrict__ dy, float* __restrict__ dw, int cin, int cout, int flip,
                 int64_t rows_per_split) {
  __shared__ __align__(16) float s_a[WK][WB];  // dy slice: [voxel][o]
  __shared__ __align__(16) float s_b[WK][WB];  // gathered x slice: [voxel][c]
  const int k = blockIdx.y;
  const int n_ct = (cin + WB - 1) / WB;
  const int o0 = (blockIdx.x / n_ct) * WB, c0 = (blockIdx.x % n_ct) * WB;
  const int64_t i_begin = static_cast<int64_t>(blockIdx.z) * rows_per_split;
  const int64_t i_end = i_begin + rows_per_split < n ? i_begin + rows_per_split : n;
  const int t = threadIdx.x, tx = t % 16, ty = t / 16;
  float acc[4][4] = {};
  for (int64_t i0 = i_begin; i0 < i_end; i0 += WK) {
    // 16 voxels x 64 channels of each operand: 1024 elements, 4 per thread
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int idx = t + e * WT;
      const int v = idx / WB, col = idx % WB;
      const int64_t i = i0 + v;
      float a = 0.0f, b = 0.0f;
      if (i < i_end) {
        if (o0 + col < cout) a = to_f32(dy[i * cout + o0 + col]);
        const int32_t j = nbr[i * kKvol + k];
        if (j >= 0 && c0 + col < cin) b = to_f32(x[static_cast<int64_t>(j) * cin + c0 + col]);
      }
      s_a[v][col] = a;
      s_b[v][col] = b;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < WK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) av[m] = s_a[kk][ty * 4 + m];
#pragma unroll
      for (int m = 0; m < 4; ++m) bv[m] = s_b[kk][tx * 4 + m];
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[m][q] = fmaf(av[m], bv[q], acc[m][q]);
    }
    __syncthreads();
  }
  const int kw = flip ? 26 - k : k;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int o = o0 + ty * 4 + m;
    if (o >= cout) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + tx * 4 + q;
      if (c < cin) atomicAdd(dw + (static_cast<int64_t>(o) * kKvol + kw) * cin + c, acc[m][q]);
    }
  }
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
  // split the voxels so that the grid covers the SMs about 8 times over
  int64_t splits = (static_cast<int64_t>(num_sms) * 8 + tiles * kKvol - 1) / (tiles * kKvol);
  if (splits < 1) splits = 1;
  int64_t rows = (n + splits - 1) / splits;
  rows = (rows + WK - 1) / WK * WK;
  splits = (n + rows - 1) / rows;
  const dim3 grid(static_cast<unsigned>(tiles), kKvol, static_cast<unsigned>(splits));
  if (bf16)
    wgrad_kernel<__nv_bfloat16><<<grid, WT, 0, stream>>>(
        nbr, n, static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(dy), dw,
        cin, cout, flip, rows);
  else
    wgrad_kernel<float><<<grid, WT, 0, stream>>>(nbr, n, static_cast<const float*>(x),
                                                 static_cast<const float*>(dy), dw, cin, cout,
                                                 flip, rows);
  return cudaGetLastError();
}

}  // namespace subm3d

// fp32 forward of the submanifold 3x3x3 convolution on CUDA-core FMA.
//
// out[i] = act( sum_k Wf[:, k, :] . x[nbr[i][k]] + bias ) + residual[i],
// Wf[:, k] = W[:, k] or W[:, 26-k] with flip (correlation / mirrored kernel,
// lato.2_mrp_mlx commit 97dcdfb54a message); bias and residual optional.  Implicit gather-GEMM: a 64-row x 64-column output tile
// per block, 256 threads with a 4x4 register tile each.  For every offset the
// tile needs, 16-channel slices of the 64 gathered input rows (zero where
// nbr = -1) and of the weight slice are staged in shared memory and
// contracted; the accumulators stay in registers across all 27 offsets, so
// there is no scatter and no atomics.  Any Cin, Cout >= 1.
//
// fp32 FMA rather than TF32 tensor cores: TF32's 10-bit mantissa cannot meet a
// 1e-5 relative tolerance over 27*Cin terms.
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "internal.h"

namespace subm3d {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

// out may alias residual (an in-place residual add): neither is __restrict__.
template <int ACT>
__global__ void __launch_bounds__(NT)
    fwd_f32_kernel(const int32_t* __restrict__ nbr, const uint32_t* __restrict__ tile_mask,
                   int64_t n, const float* __restrict__ x, const float* __restrict__ w,
                   float* out, int cin, int cout, int flip, const float* bias,
                   const float* residual) {
  __shared__ int32_t s_nbr[BM * kKvol];
  __shared__ __align__(16) float s_a[BK][BM];
  __shared__ __align__(16) float s_b[BK][BN];

  const int t = threadIdx.x;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * BM;
  const int col0 = blockIdx.y * BN;
  for (int e = t; e < BM * kKvol; e += NT) {
    const int64_t r = row0 + e / kKvol;
    s_nbr[e] = (r < n) ? nbr[row0 * kKvol + e] : -1;
  }
  const uint32_t mask = tile_mask ? tile_mask[row0 / kTileRows] : 0x7FFFFFFu;
  __syncthreads();

  const int ty = t / 16, tx = t % 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  uint32_t m = mask;
  while (m) {
    const int k = __ffs(m) - 1;
    m &= m - 1;
    const int kw = flip ? (kKvol - 1 - k) : k;
    for (int c0 = 0; c0 < cin; c0 += BK) {
#pragma unroll
      for (int e = 0; e < (BM * BK) / NT; ++e) {
        const int idx = t + e * NT;
        const int r = idx / BK, kk = idx % BK;
        const int src = s_nbr[r * kKvol + k];
        const int c = c0 + kk;
        s_a[kk][r] = (src >= 0 && c < cin) ? __ldg(x + static_cast<int64_t>(src) * cin + c) : 0.f;
      }
#pragma unroll
      for (int e = 0; e < (BN * BK) / NT; ++e) {
        const int idx = t + e * NT;
        const int col = idx / BK, kk = idx % BK;
        const int o = col0 + col, c = c0 + kk;
        s_b[kk][col] = (o < cout && c < cin)
                           ? __ldg(w + (static_cast<int64_t>(o) * kKvol + kw) * cin + c)
                           : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        const float4 a4 = *reinterpret_cast<const float4*>(&s_a[kk][ty * 4]);
        const float4 b4 = *reinterpret_cast<const float4*>(&s_b[kk][tx * 4]);
        const float av[4] = {a4.x, a4.y, a4.z, a4.w};
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      __syncthreads();
    }
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = row0 + ty * 4 + i;
    if (r >= n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = col0 + tx * 4 + j;
      if (o >= cout) continue;
      float v = activate<ACT>(acc[i][j] + (bias ? bias[o] : 0.0f));
      if (residual) v += residual[r * cout + o];
      out[r * cout + o] = v;
    }
  }
}

}  // namespace

cudaError_t launch_forward_f32(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                               const float* feats, const float* weight, float* out, int32_t cin,
                               int32_t cout, int32_t flip, const Epilogue& epi,
                               cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((n + BM - 1) / BM),
                  static_cast<unsigned>((cout + BN - 1) / BN));
  const auto* bias = static_cast<const float*>(epi.bias);
  const auto* res = static_cast<const float*>(epi.residual);
  if (epi.act == kActGelu)
    fwd_f32_kernel<kActGelu><<<grid, NT, 0, stream>>>(nbr, tile_mask, n, feats, weight, out, cin,
                                                      cout, flip, bias, res);
  else if (epi.act == kActSilu)
    fwd_f32_kernel<kActSilu><<<grid, NT, 0, stream>>>(nbr, tile_mask, n, feats, weight, out, cin,
                                                      cout, flip, bias, res);
  else
    fwd_f32_kernel<kActNone><<<grid, NT, 0, stream>>>(nbr, tile_mask, n, feats, weight, out, cin,
                                                      cout, flip, bias, res);
  return cudaGetLastError();
}

}  // namespace subm3d

// fp32 forward of the submanifold 3x3x3 convolution on CUDA-core FMA.
//
// out[i] = act( sum_k Wf[:, k, :] . x[nbr[i][k]] + bias ) + residual[i],
// Wf[:, k] = W[:, k] or W[:, 26-k] with flip (correlation / mirrored kernel,
// lato.2_mrp_mlx commit 97dcdfb54a message); bias and residual optional.
//
// Implicit gather-GEMM, one 128-row x 128-column output tile per block (the
// rows are one tile-mask tile): 256 threads with an 8 x 8 register tile each
// (rows 4 ty .. 4 ty + 3 and 64 + 4 ty ..; columns likewise with tx).  The K
// loop runs over the offsets present in the tile (its mask word) and, for each,
// 32-channel slices of Cin.  A step stages the 128 gathered input rows' slice
// (zeros where nbr = -1) and the weight slice in shared memory, k-major with a
// 4-float pad so that the transposing stores are conflict-free; the next step's
// slices load into registers, 8 channels at a time, while this step's 64 FMAs
// per thread and channel run, with two shared buffers and one barrier per step.  The accumulators stay
// in registers across all 27 offsets: no scatter, no atomics.  Any Cin, Cout
// >= 1; 16-byte loads and stores where Cin and Cout are multiples of 4.
//
// fp32 FMA rather than TF32 tensor cores: TF32's 10-bit mantissa cannot meet a
// 1e-5 relative tolerance over 27*Cin terms.
#include <cuda_runtime.h>

#include "epilogue.cuh"
#include "internal.h"

namespace subm3d {
namespace {

constexpr int BM = 128, BN = 128, BK = 32, HK = 8, NP = BK / HK, NT = 256, PAD = 4;
// dynamic shared memory: two k-major buffers of each operand, then the tile's nbr rows
constexpr int kOperandFloats = BK * (BM + PAD);  // BN == BM
constexpr size_t kSmemBytes = (4 * kOperandFloats + BM * kKvol + kKvol + 1) * 4;
static_assert(BM == kTileRows, "one tile-mask word per block");

// The four channels c .. c + 3 of row `src` (zeros past cin or for src < 0).
template <bool VEC>
__device__ __forceinline__ float4 load4(const float* __restrict__ base, int64_t src, int c,
                                        int cin) {
  if (src < 0 || c >= cin) return make_float4(0.f, 0.f, 0.f, 0.f);
  const float* p = base + src * cin + c;
  if constexpr (VEC) {
    return __ldg(reinterpret_cast<const float4*>(p));
  } else {
    float v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = c + j < cin ? __ldg(p + j) : 0.f;
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

// out may alias residual (an in-place residual add): neither is __restrict__.
template <int ACT, bool VEC>
__global__ void __launch_bounds__(NT, 2)
    fwd_f32_kernel(const int32_t* __restrict__ nbr, const uint32_t* __restrict__ tile_mask,
                   int64_t n, const float* __restrict__ x, const float* __restrict__ w,
                   float* out, int cin, int cout, int flip, const float* bias,
                   const float* residual) {
  extern __shared__ float4 smem_f4[];
  auto s_a = reinterpret_cast<float (*)[BK][BM + PAD]>(smem_f4);                       // [2]
  auto s_b = reinterpret_cast<float (*)[BK][BN + PAD]>(reinterpret_cast<float*>(smem_f4) +
                                                       2 * kOperandFloats);           // [2]
  int32_t* s_nbr = reinterpret_cast<int32_t*>(smem_f4) + 4 * kOperandFloats;
  int32_t* s_off = s_nbr + BM * kKvol;

  const int t = threadIdx.x;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * BM;
  const int col0 = blockIdx.y * BN;
  for (int e = t; e < BM * kKvol; e += NT) {
    const int64_t r = row0 + e / kKvol;
    s_nbr[e] = (r < n) ? __ldg(nbr + row0 * kKvol + e) : -1;
  }
  if (t == 0) {
    const uint32_t mask = tile_mask ? __ldg(tile_mask + blockIdx.x) : 0x7FFFFFFu;
    int cnt = 0;
    for (int k = 0; k < kKvol; ++k)
      if ((mask >> k) & 1u) s_off[cnt++] = k;
    s_off[kKvol] = cnt;
  }
  __syncthreads();

  // staging role: row / output column t / 2, channels 4 (t % 2) .. + 3 of the slice
  const int sr = t >> 1, sh = (t & 1) * 4;
  const int so = col0 + sr;
  // compute role
  const int ty = t >> 4, tx = t & 15;
  const int steps = s_off[kKvol] * ((cin + BK - 1) / BK);

  float4 ra, rb;  // the next half-step's slices
  int f_ki = 0, f_c = 0;  // the step fetch() loads next: offset index, slice start
  // part `part` (8 channels) of the step at (f_ki, f_c); the last part advances
  auto fetch = [&](int part) {
    const int k = s_off[f_ki];
    const int kw = flip ? (kKvol - 1 - k) : k;
    const int c = f_c + part * HK + sh;
    ra = load4<VEC>(x, s_nbr[sr * kKvol + k], c, cin);
    rb = load4<VEC>(w, so < cout ? static_cast<int64_t>(so) * kKvol + kw : -1, c, cin);
    if (part == NP - 1) {
      f_c += BK;
      if (f_c >= cin) {
        f_c = 0;
        ++f_ki;
      }
    }
  };
  auto stage = [&](int buf, int part) {
    const int kk = part * HK + sh;
    s_a[buf][kk + 0][sr] = ra.x;
    s_a[buf][kk + 1][sr] = ra.y;
    s_a[buf][kk + 2][sr] = ra.z;
    s_a[buf][kk + 3][sr] = ra.w;
    s_b[buf][kk + 0][sr] = rb.x;
    s_b[buf][kk + 1][sr] = rb.y;
    s_b[buf][kk + 2][sr] = rb.z;
    s_b[buf][kk + 3][sr] = rb.w;
  };

  // accumulator pairs: acc2[i][p] holds columns 2p, 2p + 1 of row i
  unsigned long long acc2[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int p = 0; p < 4; ++p) acc2[i][p] = 0ull;
  auto compute = [&](int buf, int part) {
#pragma unroll
    for (int q = 0; q < HK; ++q) {
      const int kk = part * HK + q;
      const float4 a0 = *reinterpret_cast<const float4*>(&s_a[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&s_a[buf][kk][64 + ty * 4]);
      const ulonglong2 b0 = *reinterpret_cast<const ulonglong2*>(&s_b[buf][kk][tx * 4]);
      const ulonglong2 b1 = *reinterpret_cast<const ulonglong2*>(&s_b[buf][kk][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const unsigned long long bp[4] = {b0.x, b0.y, b1.x, b1.y};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const unsigned long long ai = pack2(av[i], av[i]);
#pragma unroll
        for (int p = 0; p < 4; ++p) acc2[i][p] = fma2(ai, bp[p], acc2[i][p]);
      }
    }
  };

  if (steps > 0) {
#pragma unroll 1
    for (int part = 0; part < NP; ++part) {
      fetch(part);
      stage(0, part);
    }
    __syncthreads();
  }
  // buffer s & 1 holds step s; step s + 1 is fetched into registers 8 channels
  // at a time and staged in the other buffer (free since the last barrier)
  for (int s = 0; s < steps; ++s) {
    const int buf = s & 1;
    const bool more = s + 1 < steps;
#pragma unroll
    for (int part = 0; part < NP; ++part) {
      if (more) fetch(part);
      compute(buf, part);
      if (more) stage(buf ^ 1, part);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t r = row0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (r >= n) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int o0 = col0 + h * 64 + tx * 4;
      float v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int o = o0 + j;
        const int col = 4 * h + j;
        const unsigned long long pr = acc2[i][col >> 1];
        const float av = __uint_as_float(static_cast<uint32_t>((col & 1) ? (pr >> 32) : pr));
        v[j] = o < cout ? activate<ACT>(av + (bias ? bias[o] : 0.0f)) : 0.0f;
      }
      float* dst = out + r * cout + o0;
      if (VEC && o0 + 3 < cout) {
        if (residual) {
          const float4 q = *reinterpret_cast<const float4*>(residual + r * cout + o0);
          v[0] += q.x;
          v[1] += q.y;
          v[2] += q.z;
          v[3] += q.w;
        }
        *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (o0 + j >= cout) break;
          dst[j] = v[j] + (residual ? residual[r * cout + o0 + j] : 0.0f);
        }
      }
    }
  }
}

template <int ACT, bool VEC>
cudaError_t launch_one(dim3 grid, cudaStream_t stream, const int32_t* nbr,
                       const uint32_t* tile_mask, int64_t n, const float* x, const float* w,
                       float* out, int cin, int cout, int flip, const float* bias,
                       const float* res) {
  static bool attr_set[64] = {};  // per device and instantiation; a repeat set is harmless
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(fwd_f32_kernel<ACT, VEC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  fwd_f32_kernel<ACT, VEC><<<grid, NT, kSmemBytes, stream>>>(nbr, tile_mask, n, x, w, out, cin,
                                                             cout, flip, bias, res);
  return cudaGetLastError();
}

template <int ACT>
cudaError_t launch_act(dim3 grid, bool vec, cudaStream_t stream, const int32_t* nbr,
                       const uint32_t* tile_mask, int64_t n, const float* x, const float* w,
                       float* out, int cin, int cout, int flip, const float* bias,
                       const float* res) {
  return vec ? launch_one<ACT, true>(grid, stream, nbr, tile_mask, n, x, w, out, cin, cout, flip,
                                     bias, res)
             : launch_one<ACT, false>(grid, stream, nbr, tile_mask, n, x, w, out, cin, cout, flip,
                                      bias, res);
}

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

}  // namespace

cudaError_t launch_forward_f32(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                               const float* feats, const float* weight, float* out, int32_t cin,
                               int32_t cout, int32_t flip, const Epilogue& epi,
                               cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((n + BM - 1) / BM),
                  static_cast<unsigned>((cout + BN - 1) / BN));
  const auto* bias = static_cast<const float*>(epi.bias);
  const auto* res = static_cast<const float*>(epi.residual);
  // 16-byte rows: feats, weight, out and residual rows start on 16 bytes
  const bool vec = cin % 4 == 0 && cout % 4 == 0 && aligned16(feats) && aligned16(weight) &&
                   aligned16(out) && (!res || aligned16(res));
  if (epi.act == kActGelu)
    return launch_act<kActGelu>(grid, vec, stream, nbr, tile_mask, n, feats, weight, out, cin,
                                cout, flip, bias, res);
  if (epi.act == kActSilu)
    return launch_act<kActSilu>(grid, vec, stream, nbr, tile_mask, n, feats, weight, out, cin,
                                cout, flip, bias, res);
  return launch_act<kActNone>(grid, vec, stream, nbr, tile_mask, n, feats, weight, out, cin, cout,
                              flip, bias, res);
}

}  // namespace subm3d

// Epilogue arithmetic shared by the forward kernels:
//   out = act(acc + bias) + residual,
// bias added to the fp32 accumulator, then the activation, then the residual,
// and a bf16 output rounded once (round to nearest even) at the end.  The
// epilogue of a sparse residual block: the first convolution takes a bias and
// an activation, the second a bias and the block's skip input as residual.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace subm3d {

// GELU in its erf form, v * Phi(v) with Phi(v) = erfc(-v / sqrt(2)) / 2, and
// erfc by the rational-times-Gaussian approximation of Abramowitz & Stegun,
// Handbook of Mathematical Functions, eq. 7.1.26 (after Hastings): for u >= 0,
//   erfc(u) ~= t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-u^2),  t = 1 / (1 + p u),
// absolute error <= 1.5e-7.  Computing erfc(|v| / sqrt 2) directly keeps the
// negative tail free of cancellation (Phi(v) = erfc / 2 there, 1 - erfc / 2 for
// v >= 0), and the form has no branch.
__device__ __forceinline__ float gelu_erf(float v) {
  constexpr float p = 0.3275911f;
  constexpr float a1 = 0.254829592f, a2 = -0.284496736f, a3 = 1.421413741f,
                  a4 = -1.453152027f, a5 = 1.061405429f;
  const float u = __fmul_rn(fabsf(v), 0.70710678118654752f);
  const float t = __fdividef(1.0f, __fmaf_rn(p, u, 1.0f));
  const float poly =
      __fmul_rn(t, __fmaf_rn(t, __fmaf_rn(t, __fmaf_rn(t, __fmaf_rn(t, a5, a4), a3), a2), a1));
  const float ec = __fmul_rn(poly, __expf(-__fmul_rn(u, u)));  // erfc(|v| / sqrt 2)
  return __fmul_rn(v, v >= 0.0f ? __fmaf_rn(-0.5f, ec, 1.0f) : __fmul_rn(0.5f, ec));
}

// Two lanes of fp32 in one 64-bit register: the packed add / multiply / fma of
// sm_100 (add / mul / fma .rn.f32x2: two independent IEEE operations each).
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2_unpack(unsigned long long d, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// gelu_erf on two values at once: the same operations in the same order (so
// the same bits), the multiplies and fmas as f32x2 pairs; the reciprocal and
// the exponential stay per value.
__device__ __forceinline__ void gelu_erf2(float& v0, float& v1) {
  const auto k = [](float c) { return f2_pack(c, c); };
  const unsigned long long u = f2_mul(f2_pack(fabsf(v0), fabsf(v1)), k(0.70710678118654752f));
  float d0, d1;
  f2_unpack(f2_fma(k(0.3275911f), u, k(1.0f)), d0, d1);
  const unsigned long long t = f2_pack(__fdividef(1.0f, d0), __fdividef(1.0f, d1));
  unsigned long long q = f2_fma(t, k(1.061405429f), k(-1.453152027f));
  q = f2_fma(t, q, k(1.421413741f));
  q = f2_fma(t, q, k(-0.284496736f));
  q = f2_fma(t, q, k(0.254829592f));
  const unsigned long long poly = f2_mul(t, q);
  float w0, w1;
  f2_unpack(f2_mul(u, u), w0, w1);
  const unsigned long long ec = f2_mul(poly, f2_pack(__expf(-w0), __expf(-w1)));
  float hi0, hi1, lo0, lo1;  // Phi for v >= 0 and for v < 0
  f2_unpack(f2_fma(k(-0.5f), ec, k(1.0f)), hi0, hi1);
  f2_unpack(f2_mul(k(0.5f), ec), lo0, lo1);
  f2_unpack(f2_mul(f2_pack(v0, v1), f2_pack(v0 >= 0.0f ? hi0 : lo0, v1 >= 0.0f ? hi1 : lo1)),
            v0, v1);
}

template <int ACT>
__device__ __forceinline__ float activate(float v) {
  if constexpr (ACT == kActGelu) {
    return gelu_erf(v);
  } else if constexpr (ACT == kActSilu) {
    // v * sigmoid(v) with the fast exponential and the fast divide (a few ulp,
    // well inside both paths' bars); for v -> -inf the divisor overflows to inf
    // and the quotient is -0
    return __fdividef(v, 1.0f + __expf(-v));
  } else {
    return v;
  }
}

// Eight fp32 values + an optional bf16 residual chunk -> eight bf16 (one rounding).
__device__ __forceinline__ uint4 finish_bf16x8(const float (&f)[8], bool has_residual,
                                               uint4 r) {
  float g[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) g[j] = f[j];
  if (has_residual) {
    const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      g[2 * j] += __uint_as_float(rw[j] << 16);
      g[2 * j + 1] += __uint_as_float(rw[j] & 0xFFFF0000u);
    }
  }
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(g[2 * j], g[2 * j + 1]);
    w[j] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Bytes of fp32 staging one bf16 epilogue warp needs: 16 positions x 32 channels
// (a 32-position chunk is staged in two halves).
constexpr int kEpiWarpStageBytes = 16 * 32 * 4;

// The epilogue of one 256-position accumulator by one warp: its 32 channels
// (TMEM lanes; lane = channel o_warp + lane) in 8 chunks of 32 positions.  Per
// chunk, in two halves of 16 positions, the values after bias and activation go
// to the warp's staging area (`stage`, kEpiWarpStageBytes), then each lane takes
// 8 channels of one position and stores 16 bytes.  With a residual they are
// staged in fp32 (a position's 128-byte row has its 16-byte halves swapped at
// odd positions, so the reads are free of bank conflicts) and the lane adds the
// residual before the one bf16 rounding; without one they are rounded first and
// staged as 64-byte bf16 rows.  The output row of position j is
// pos[j] >> 2 when pos[j] is a voxel entry (POS: the x-run layout; pads and
// empty positions are dropped), else row0 + j below n.  Latency is hidden by prefetching: position entries
// two chunks ahead and each chunk's residual rows one chunk ahead, so they load
// while the previous chunk is staged.  The chunk loop stays rolled: an
// unrolled one inlines 256 activations and slows every warp of the kernel.
template <int ACT, bool POS>
__device__ __forceinline__ void epilogue_tile_bf16(uint32_t taddr, float bias_v, uint32_t stage,
                                                   int lane, int o_warp, int cout,
                                                   const int32_t* pos, int64_t row0, int64_t n,
                                                   __nv_bfloat16* out,
                                                   const __nv_bfloat16* residual) {
  constexpr int kChunks = 8;
  const int q = lane % 4;  // this lane's 8-channel group in the store phase
  const int o = o_warp + q * 8;
  const bool o_ok = o < cout;
  // rows (int32: N < 2^31) of this lane's 4 store slots of chunk ci, -1 to skip;
  // pe = the pos entry of position ci * 32 + lane (POS)
  auto rows_of = [&](int ci, int32_t pe, int32_t (&r)[4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int jj = p * 8 + lane / 4;
      if constexpr (POS) {
        const int32_t e = __shfl_sync(0xFFFFFFFFu, pe, jj);
        r[p] = (e >= 0 && (e & 3) == kPosVoxel) ? (e >> 2) : -1;
      } else {
        const int64_t row = row0 + ci * 32 + jj;
        r[p] = row < n ? static_cast<int32_t>(row) : -1;
      }
    }
  };
  auto load_res = [&](const int32_t (&r)[4], uint4 (&v)[4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p)
      v[p] = (residual && r[p] >= 0 && o_ok)
                 ? *reinterpret_cast<const uint4*>(residual + static_cast<int64_t>(r[p]) * cout + o)
                 : make_uint4(0u, 0u, 0u, 0u);
  };
  // chunk 0's rows and residual now, chunk 1's pos entry in flight
  int32_t pe_next = POS ? ld_dep(pos + 32 + lane) : 0;
  int32_t rows[4];
  uint4 res[4];
  rows_of(0, POS ? ld_dep(pos + lane) : 0, rows);
  if (residual != nullptr) load_res(rows, res);
  if (residual == nullptr) {
    // No residual: round to bf16 before staging (the same single rounding), so
    // the staging holds 64-byte rows of 32 bf16 channels and each lane reads its
    // 8 channels with one 16-byte load -- half the shared-memory traffic.
#pragma unroll 1
    for (int ci = 0; ci < kChunks; ++ci) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + ci * 32, v);
      int32_t rows_n[4];
      if (ci + 1 < kChunks) {
        rows_of(ci + 1, pe_next, rows_n);
        if (POS && ci + 2 < kChunks) pe_next = ld_dep(pos + (ci + 2) * 32 + lane);
      }
      tmem_ld_wait();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int e = 0; e < 16; e += 2) {  // positions e, e+1 of the half
          float f0, f1;
          f2_unpack(f2_add(f2_pack(__uint_as_float(v[16 * h + e]),
                                   __uint_as_float(v[16 * h + e + 1])),
                           f2_pack(bias_v, bias_v)),
                    f0, f1);
          if constexpr (ACT == kActGelu) {
            gelu_erf2(f0, f1);
          } else {
            f0 = activate<ACT>(f0);
            f1 = activate<ACT>(f1);
          }
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(f0, f1);
          const uint32_t w = *reinterpret_cast<const uint32_t*>(&b2);
          sts_u16(stage + e * 64 + lane * 2, static_cast<uint16_t>(w & 0xFFFFu));
          sts_u16(stage + (e + 1) * 64 + lane * 2, static_cast<uint16_t>(w >> 16));
        }
        __syncwarp();
#pragma unroll
        for (int p = 2 * h; p < 2 * h + 2; ++p) {
          const int j = (p - 2 * h) * 8 + lane / 4;  // staging row
          const uint4 val = lds_16(stage + j * 64 + q * 16);
          if (rows[p] >= 0 && o_ok)
            *reinterpret_cast<uint4*>(out + static_cast<int64_t>(rows[p]) * cout + o) = val;
        }
        __syncwarp();
      }
#pragma unroll
      for (int p = 0; p < 4; ++p) rows[p] = rows_n[p];
    }
    return;
  }
#pragma unroll 1
  for (int ci = 0; ci < kChunks; ++ci) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + ci * 32, v);
    int32_t rows_n[4];
    uint4 res_n[4];
    if (ci + 1 < kChunks) {  // next chunk's rows and residual (and the pos entry after it)
      rows_of(ci + 1, pe_next, rows_n);
      load_res(rows_n, res_n);
      if (POS && ci + 2 < kChunks) pe_next = ld_dep(pos + (ci + 2) * 32 + lane);
    }
    tmem_ld_wait();
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // positions 16h .. 16h+15 of the chunk: store slots 2h, 2h+1
#pragma unroll
      for (int e = 0; e < 16; e += 2) {  // bias and activation on pairs of positions
        float f0, f1;
        f2_unpack(f2_add(f2_pack(__uint_as_float(v[16 * h + e]), __uint_as_float(v[16 * h + e + 1])),
                         f2_pack(bias_v, bias_v)),
                  f0, f1);
        if constexpr (ACT == kActGelu) {
          gelu_erf2(f0, f1);
        } else {
          f0 = activate<ACT>(f0);
          f1 = activate<ACT>(f1);
        }
        sts_u32(stage + e * 128 + (lane * 4), __float_as_uint(f0));
        sts_u32(stage + (e + 1) * 128 + ((lane * 4) ^ 16), __float_as_uint(f1));
      }
      __syncwarp();
#pragma unroll
      for (int p = 2 * h; p < 2 * h + 2; ++p) {
        const int j = (p - 2 * h) * 8 + lane / 4;  // staging row (same parity as the position)
        const uint32_t rb = stage + j * 128;
        const uint32_t sw = static_cast<uint32_t>(j & 1) << 4;
        const uint4 lo = lds_16(rb + ((q * 32) ^ sw));
        const uint4 hi = lds_16(rb + ((q * 32 + 16) ^ sw));
        if (rows[p] >= 0 && o_ok) {
          const float f[8] = {__uint_as_float(lo.x), __uint_as_float(lo.y), __uint_as_float(lo.z),
                              __uint_as_float(lo.w), __uint_as_float(hi.x), __uint_as_float(hi.y),
                              __uint_as_float(hi.z), __uint_as_float(hi.w)};
          *reinterpret_cast<uint4*>(out + static_cast<int64_t>(rows[p]) * cout + o) =
              finish_bf16x8(f, residual != nullptr, res[p]);
        }
      }
      __syncwarp();
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      rows[p] = rows_n[p];
      res[p] = res_n[p];
    }
  }
}

}  // namespace subm3d

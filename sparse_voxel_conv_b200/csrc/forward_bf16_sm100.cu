// bf16 forward of the submanifold 3x3x3 convolution on sm_100a tensor cores.
//
// out[i] = act( sum_k Wf[:, k, :] . x[nbr[i][k]] ) with Wf[:, k] = W[:, k]
// (correlation) or W[:, 26-k] (flip), W in spconv's KRSC layout
// [Cout, kz, ky, kx, Cin] (lato.2_mrp_mlx, commit 97dcdfb54a message and
// CLAUDE.md "Key facts").  An implicit gather-GEMM: no scatter, no atomics,
// no [N, 27, Cin] buffer.
//
// One CTA computes a 128-row x BN-column output tile (BN = Cout split into
// blocks of at most 256 columns) as one fp32 accumulator in tensor memory,
// summing over every (offset k, 64-channel chunk j) step the tile needs:
//
//   warps 0-3  gather: for step (k, j) copy 128 B of row nbr[r][k] of x (chunk j)
//              into the A stage with cp.async, 16-byte pieces placed at their
//              128-byte-swizzle positions; zero-fill where nbr = -1.  Lanes
//              0-7 of a warp cover one 128-byte row segment, so every request
//              is a full, aligned 128-byte line.  They then run the epilogue.
//   warp 4     TMEM allocation; lane 0 issues tcgen05.mma (M=128, N=BN, K=16)
//              and commits each stage back to the producers.
//   warp 5     lane 0 loads the weight slice Wf[n0:n0+BN, k, 64j:64j+64] with a
//              3-D TMA tiled load (128-byte swizzle), completing on the stage's
//              mbarrier.
//   epilogue   tcgen05.ld 32 columns at a time, optional exact-erf GELU,
//              round to bf16 (RNE), 16-byte stores.
//
// Offsets with no neighbour in the whole tile (bit clear in the tile's mask
// word) are skipped.  Every wait is bounded (ptx.cuh); a wait that runs out
// sets the library's device error word, the CTA drains its copies, frees its
// tensor memory and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace subm3d {
namespace {

constexpr int BM = 128;                      // output rows per tile (= TMEM lanes)
constexpr int KC = 64;                       // channels per stage: one 128-byte row
constexpr int A_STAGE_BYTES = BM * 128;      // 16 KB
constexpr int NUM_THREADS = 192;
constexpr int MMA_WARP = 4;
constexpr int TMA_WARP = 5;
constexpr int kSmemLimit = 227 * 1024;

struct FwdArgs {
  const int32_t* nbr;
  const uint32_t* tile_mask;
  int64_t n;
  const __nv_bfloat16* x;
  __nv_bfloat16* out;
  int32_t cin, cout, bn, n_kchunks, stages, flip, act;
  uint32_t tmem_cols;
  int32_t* err_word;
};

struct SmemPlan {
  int stages;
  size_t a_off, b_off, nbr_off, bar_off, bytes;
};

__host__ __device__ inline SmemPlan plan_smem(int bn, int stages) {
  SmemPlan p;
  p.stages = stages;
  p.a_off = 0;
  p.b_off = p.a_off + static_cast<size_t>(stages) * A_STAGE_BYTES;
  p.nbr_off = p.b_off + static_cast<size_t>(stages) * bn * 128;
  p.bar_off = p.nbr_off + BM * kKvol * 4;
  // full[stages], empty[stages], acc, then tmem slot + abort word
  p.bytes = p.bar_off + (2 * stages + 1) * 8 + 16 + 1024;  // + alignment slack
  return p;
}

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Waits until at most `lag` of this thread's cp.async groups are pending.
__device__ __forceinline__ void cp_async_wait_dyn(int lag) {
  switch (lag) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    default: cp_async_wait<7>(); break;
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    subm3d_fwd_bf16_sm100(const __grid_constant__ CUtensorMap wmap, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const SmemPlan plan = plan_smem(a.bn, a.stages);
  const int S = a.stages;
  uint8_t* stage_a = base + plan.a_off;
  uint8_t* stage_b = base + plan.b_off;
  int32_t* nbr_s = reinterpret_cast<int32_t*>(base + plan.nbr_off);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + plan.bar_off);
  uint64_t* empty = full + S;
  uint64_t* accbar = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int64_t tile = blockIdx.x;
  const int64_t row0 = tile * BM;
  const int n0 = blockIdx.y * a.bn;
  const uint32_t mask = a.tile_mask ? __ldg(a.tile_mask + tile) : 0x7FFFFFFu;
  const int n_iters = __popc(mask) * a.n_kchunks;
  const uint32_t b_stage_bytes = static_cast<uint32_t>(a.bn) * 128u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 128 + 1);  // 128 gather threads + the TMA thread's expect_tx
      mbar_init(&empty[s], 1);       // one tcgen05.commit
    }
    mbar_init(accbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) tma_prefetch_desc(&wmap);
  for (int e = threadIdx.x; e < BM * kKvol; e += NUM_THREADS) {
    const int64_t r = row0 + e / kKvol;
    nbr_s[e] = (r < a.n) ? __ldg(a.nbr + row0 * kKvol + e) : -1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // ---------------------------------------------------------- gather ----
    const int lag = S - 1 < 7 ? S - 1 : 7;
    const int sub = lane >> 3;    // which of 4 rows this lane serves per pass
    const int piece = lane & 7;   // which 16-byte piece of the 128-byte segment
    uint32_t m = mask;
    int it = 0;
    bool ok = true;
    while (m && ok) {
      const int k = __ffs(m) - 1;
      m &= m - 1;
      for (int j = 0; j < a.n_kchunks; ++j, ++it) {
        const int s = it % S;
        if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t a_base = smem_u32(stage_a + static_cast<size_t>(s) * A_STAGE_BYTES);
        const int ch = j * KC + piece * 8;  // first channel of this piece
        const bool piece_live = ch < a.cin;
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) {
          const int r = warp * 32 + rr * 4 + sub;
          const int32_t src = nbr_s[r * kKvol + k];
          const bool live = piece_live && src >= 0;
          const __nv_bfloat16* gp = live ? a.x + static_cast<int64_t>(src) * a.cin + ch : a.x;
          const uint32_t dst = a_base + r * 128 + ((piece ^ (r & 7)) << 4);
          if (piece_live) cp_async_16(dst, gp, live ? 16u : 0u);
        }
        cp_async_commit();
        if (it >= lag) {
          cp_async_wait_dyn(lag);
          fence_proxy_async_smem();
          mbar_arrive(&full[(it - lag) % S]);
        }
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    if (ok) {
      for (int t = (it - lag > 0 ? it - lag : 0); t < it; ++t) mbar_arrive(&full[t % S]);
    }

    // -------------------------------------------------------- epilogue ----
    // tcgen05.ld is warp-collective: take the epilogue only if the whole warp can.
    bool go = ok && n_iters > 0 && mbar_wait(accbar, 0, abort_flag);
    go = __all_sync(0xFFFFFFFFu, go);
    if (go) {
      tc_fence_after();
      const int r = warp * 32 + lane;
      const int64_t row = row0 + r;
      const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
      __nv_bfloat16* orow = a.out + row * a.cout + n0;
      for (int c0 = 0; c0 < a.bn; c0 += 32) {
        const int width = a.bn - c0 >= 32 ? 32 : 16;
        uint32_t v[32];
        if (width == 32) {
          tmem_ld_32x32b_x32(lane_addr + c0, v);
        } else {
          uint32_t h[16];
          tmem_ld_32x32b_x16(lane_addr + c0, h);
#pragma unroll
          for (int q = 0; q < 16; ++q) v[q] = h[q];
        }
        tmem_ld_wait();
        if (row < a.n) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q * 8 >= width || n0 + c0 + q * 8 >= a.cout) continue;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float acc = __uint_as_float(v[q * 8 + e]);
              f[e] = a.act ? gelu_erf(acc) : acc;
            }
            uint4 pk;
            pk.x = pack_bf16x2(f[0], f[1]);
            pk.y = pack_bf16x2(f[2], f[3]);
            pk.z = pack_bf16x2(f[4], f[5]);
            pk.w = pack_bf16x2(f[6], f[7]);
            *reinterpret_cast<uint4*>(orow + c0 + q * 8) = pk;
          }
        }
      }
    } else if (n_iters == 0 && row0 + warp * 32 + lane < a.n) {
      // A tile with no neighbours at all cannot occur for a valid map (every
      // voxel is its own centre neighbour); write act(0) = 0 for safety.
      __nv_bfloat16* orow = a.out + (row0 + warp * 32 + lane) * a.cout + n0;
      for (int c = 0; c < a.bn && n0 + c < a.cout; ++c) orow[c] = __float2bfloat16_rn(0.f);
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------- MMA ----
    if (lane == 0 && n_iters > 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, static_cast<uint32_t>(a.bn));
      uint32_t m = mask;
      int it = 0;
      bool ok = true;
      while (m && ok) {
        m &= m - 1;
        for (int j = 0; j < a.n_kchunks; ++j, ++it) {
          const int s = it % S;
          if (!mbar_wait(&full[s], (it / S) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int ksteps = (a.cin - j * KC >= KC ? KC : a.cin - j * KC) / 16;
          const uint32_t a0 = smem_u32(stage_a + static_cast<size_t>(s) * A_STAGE_BYTES);
          const uint32_t b0 = smem_u32(stage_b + static_cast<size_t>(s) * b_stage_bytes);
          for (int kk = 0; kk < ksteps; ++kk) {
            umma_bf16(tmem_base, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32),
                      idesc, (it | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
      }
      // Always commit the accumulator barrier, so that the tensor memory is
      // only released after every issued MMA has completed.
      umma_commit(accbar);
      if (!ok) {
        volatile int no_abort = 0;
        mbar_wait(accbar, 0, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------- TMA ----
    if (lane == 0 && n_iters > 0) {
      uint32_t m = mask;
      int it = 0;
      bool ok = true;
      while (m && ok) {
        const int k = __ffs(m) - 1;
        m &= m - 1;
        const int kw = a.flip ? (kKvol - 1 - k) : k;
        for (int j = 0; j < a.n_kchunks; ++j, ++it) {
          const int s = it % S;
          if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], b_stage_bytes);
          tma_load_3d(smem_u32(stage_b + static_cast<size_t>(s) * b_stage_bytes), &wmap, &full[s],
                      j * KC, kw, n0);
        }
      }
      if (!ok) __nanosleep(20000);  // let TMA loads already issued land before exit
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, a.tmem_cols);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicExch(a.err_word, 1);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Per-device one-time setup: opt in to the large dynamic shared memory size.
cudaError_t ensure_attrs(int device) {
  static std::mutex mu;
  static bool done[64] = {};
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (done[device]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(subm3d_fwd_bf16_sm100,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  if (e == cudaSuccess) done[device] = true;
  return e;
}

}  // namespace

cudaError_t launch_forward_bf16(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                                const void* feats, const void* weight, void* out, int32_t cin,
                                int32_t cout, int32_t flip, int32_t act, int32_t* err_word,
                                cudaStream_t stream) {
  EncodeTiledFn encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  if ((e = ensure_attrs(device)) != cudaSuccess) return e;

  // Split Cout into n_blocks column blocks of equal width (a multiple of 16, <= 256).
  const int n_blocks = (cout + 255) / 256;
  int bn = (cout + n_blocks - 1) / n_blocks;
  bn = (bn + 15) / 16 * 16;
  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(bn)) tmem_cols <<= 1;
  int stages = 8;
  while (stages > 2 && plan_smem(bn, stages).bytes > static_cast<size_t>(kSmemLimit)) --stages;
  const SmemPlan plan = plan_smem(bn, stages);

  CUtensorMap map;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cin), 27, static_cast<cuuint64_t>(cout)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cin) * 2,
                                 static_cast<cuuint64_t>(cin) * 27 * 2};
  const cuuint32_t box[3] = {KC, 1, static_cast<cuuint32_t>(bn)};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(weight), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  FwdArgs a;
  a.nbr = nbr;
  a.tile_mask = tile_mask;
  a.n = n;
  a.x = static_cast<const __nv_bfloat16*>(feats);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.cin = cin;
  a.cout = cout;
  a.bn = bn;
  a.n_kchunks = (cin + KC - 1) / KC;
  a.stages = stages;
  a.flip = flip;
  a.act = act;
  a.tmem_cols = tmem_cols;
  a.err_word = err_word;
  const dim3 grid(static_cast<unsigned>((n + BM - 1) / BM), static_cast<unsigned>(n_blocks));
  subm3d_fwd_bf16_sm100<<<grid, NUM_THREADS, plan.bytes, stream>>>(map, a);
  return cudaGetLastError();
}

}  // namespace subm3d

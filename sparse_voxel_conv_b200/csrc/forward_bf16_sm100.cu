// bf16 forward of the submanifold 3x3x3 convolution on sm_100a tensor cores.
//
// out[i] = act( sum_k Wf[:, k, :] . x[nbr[i][k]] + bias ) + residual[i] with
// Wf[:, k] = W[:, k]
// (correlation) or W[:, 26-k] (flip), W in spconv's KRSC layout
// [Cout, kz, ky, kx, Cin] (lato.2_mrp_mlx, commit 97dcdfb54a message and
// CLAUDE.md "Key facts").  An implicit gather-GEMM: no scatter, no atomics,
// no [N, 27, Cin] buffer.
//
// Orientation of the contraction.  A tcgen05.mma with M = 128 costs the same
// number of cycles for any N up to 256, so it reaches the tensor-core peak
// only at N = 256.  The layer widths here are 64-128 channels, so the output
// channels are the M side and a tile of 256 voxels is the N side:
//
//     D[o, v] += sum_c Wf[o, k, c] * x[nbr[v][k], c]      (D in tensor memory)
//
// with A = the weight slice (128 output channels x a channel chunk, loaded by
// TMA) and B = the gathered input rows (256 voxels x the chunk).  Both are
// K-major in the 128/64/32-byte swizzle layout matching the chunk of 64/32/16
// channels (the widest that divides Cin).
//
// Persistent kernel, one CTA per SM.  A work unit is a 256-voxel tile x a
// block of 128 output channels; its fp32 accumulator (128 lanes x 256 columns)
// sums over every step (offset k, chunk j) the tile needs.  Roles (14 warps):
//
//   warps 4-11 (gather)  256 threads fetch B: for step (k, j) the 256 rows
//       x[nbr[v][k]][chunk j] are copied with 16-byte cp.async straight into
//       their swizzled positions in the stage (zero-fill where nbr = -1); each
//       thread's cp.async.mbarrier.arrive.noinc completes the stage barrier
//       when its copies have landed.  Eight lanes cover one 128-byte row
//       segment, so every request is a whole aligned segment.
//   warp 13 (TMA)        bulk-copies each unit's nbr rows [256 x 27] into one
//       of two shared buffers ahead of use, and loads the weight slice
//       Wf[o0:o0+128, k, chunk j] of every step with a 3-D TMA tiled load
//       (rows past Cout read as zero).
//   warp 12 (MMA)        TMEM allocation (512 columns: two accumulators); lane 0
//       issues tcgen05.mma (M=128, N=256, K=16) and commits each stage back.
//   warps 0-3 (epilogue) drain the other accumulator: warp w holds channels
//       32w..32w+31; tcgen05.ld 32 voxels at a time, bias, activation (none,
//       exact GELU, SiLU), a transpose through fp32 shared memory, the
//       residual, one bf16 rounding (nearest even) and 16-byte stores of whole
//       64-byte channel runs of each voxel's row (epilogue.cuh).
//
// Offsets with no neighbour anywhere in the tile (bit clear in both 128-row
// mask words) are skipped.  Every wait is bounded (ptx.cuh).  When one runs
// out, every role leaves its loop; after a CTA-wide barrier the TMA lane waits
// (bounded) for the weight and nbr copies it issued and the MMA lane for its
// MMAs, then the CTA frees its tensor memory, sets the library's device error
// word and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "epilogue.cuh"

namespace subm3d {
namespace {

constexpr int TV = 256;  // voxels per tile (MMA N)
constexpr int TO = 128;  // output channels per unit (MMA M, TMEM lanes)
constexpr int NUM_EPI_WARPS = 4;
constexpr int NUM_GATHER_WARPS = 8;
constexpr int GATHER_WARP0 = 4;
constexpr int MMA_WARP = GATHER_WARP0 + NUM_GATHER_WARPS;
constexpr int TMA_WARP = MMA_WARP + 1;
constexpr int NUM_THREADS = (TMA_WARP + 1) * 32;
constexpr int GATHER_THREADS = NUM_GATHER_WARPS * 32;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kNbrTileBytes = TV * kKvol * 4;             // 27648
constexpr int kEpiStageBytes = NUM_EPI_WARPS * kEpiWarpStageBytes;  // fp32 staging per warp
constexpr uint32_t kTmemCols = 2 * TV;
constexpr uint32_t kCentreBit = 1u << 13;

struct FwdArgs {
  const int32_t* nbr;
  const uint32_t* tile_mask;  // one word per 128 rows
  const __nv_bfloat16* x;
  int64_t n;
  __nv_bfloat16* out;
  const __nv_bfloat16* bias;      // [cout] or nullptr
  const __nv_bfloat16* residual;  // [n, cout] or nullptr; may be `out`
  int32_t cin, cout, n_oblocks, n_kchunks, stages, flip;
  int64_t n_tiles;
  int32_t* err_word;
  uint64_t wait_limit_ns;
};

struct SmemPlan {
  size_t a_off, b_off, nbr_off, epi_off, bar_off, bytes;
};

__host__ __device__ inline SmemPlan plan_smem(int chunk, int stages) {
  SmemPlan p;
  const size_t a_bytes = static_cast<size_t>(TO) * chunk * 2;
  const size_t b_bytes = static_cast<size_t>(TV) * chunk * 2;
  p.a_off = 0;
  p.b_off = p.a_off + stages * a_bytes;
  p.nbr_off = p.b_off + stages * b_bytes;
  p.epi_off = p.nbr_off + 2 * kNbrTileBytes;
  p.bar_off = p.epi_off + kEpiStageBytes;
  // full[S], wfull[S], empty[S], nbr_full[2], nbr_empty[2], acc_full[2], acc_empty[2],
  // drain, WaitCtl (16 B), tmem slot
  p.bytes = p.bar_off + (3 * stages + 9) * 8 + 16 + 16 + 1024;  // + base alignment slack
  return p;
}

// The sequence of (unit, offset k, chunk j) steps a CTA runs; every role walks
// the same sequence.  The centre offset is always included, so every unit has
// at least one step.
struct Steps {
  int64_t u;       // current unit
  int64_t n_units;
  int local;       // index of the unit within this CTA (buffer / parity selector)
  uint32_t mask;   // offsets of the unit
  uint32_t rest;   // offsets still to come in the current chunk
  int k, j;        // current offset and chunk
  int slot;        // stage slot of the current step (step counter mod stages)
  uint32_t phase;  // parity of the slot's current use (step counter / stages, mod 2)
  bool valid;

  __device__ void load_unit(const FwdArgs& a) {
    const int64_t tile = u / a.n_oblocks;
    uint32_t m = 0x7FFFFFFu;
    if (a.tile_mask) {
      const int64_t w = 2 * tile;
      const int64_t n_words = (a.n + kTileRows - 1) / kTileRows;
      m = __ldg(a.tile_mask + w) | (w + 1 < n_words ? __ldg(a.tile_mask + w + 1) : 0u);
    }
    m |= kCentreBit;
    mask = m;
    k = __ffs(m) - 1;
    rest = m & (m - 1);
    j = 0;
  }
  __device__ void begin(const FwdArgs& a) {
    n_units = a.n_tiles * a.n_oblocks;
    u = blockIdx.x;
    local = 0;
    slot = 0;
    phase = 0;
    valid = u < n_units;
    if (valid) load_unit(a);
  }
  // Advances one step; returns true when the step moved to a new unit (or ended).
  __device__ bool next(const FwdArgs& a) {
    if (++slot == a.stages) {
      slot = 0;
      phase ^= 1u;
    }
    // chunk-major: all offsets of chunk j, then chunk j+1, so that the steps of
    // x-adjacent offsets (which gather largely the same rows, shifted by one
    // voxel) follow each other and can share cached rows
    if (rest) {
      k = __ffs(rest) - 1;
      rest &= rest - 1;
      return false;
    }
    if (++j < a.n_kchunks) {
      k = __ffs(mask) - 1;
      rest = mask & (mask - 1);
      return false;
    }
    j = 0;
    u += gridDim.x;
    ++local;
    valid = u < n_units;
    if (valid) load_unit(a);
    return true;
  }
};

template <int CHUNK, int ACT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    subm3d_fwd_bf16_sm100(const __grid_constant__ CUtensorMap wmap, const FwdArgs a) {
  constexpr int ROW_BYTES = CHUNK * 2;  // 128, 64 or 32
  constexpr int PPR = CHUNK / 8;        // 16-byte pieces per row segment
  constexpr int ROWS_PER_PASS = GATHER_THREADS / PPR;
  constexpr int PPT = TV / ROWS_PER_PASS;  // pieces per gather thread per step
  constexpr uint32_t A_STAGE = TO * ROW_BYTES;
  constexpr uint32_t B_STAGE = TV * ROW_BYTES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = a.stages;
  const SmemPlan plan = plan_smem(CHUNK, S);
  uint8_t* stage_a = base + plan.a_off;
  uint8_t* stage_b = base + plan.b_off;
  int32_t* nbr_s = reinterpret_cast<int32_t*>(base + plan.nbr_off);
  uint8_t* epi_s = base + plan.epi_off;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + plan.bar_off);  // gathered B rows
  uint64_t* wfull = full + S;                                           // TMA weight slice
  uint64_t* empty = wfull + S;
  uint64_t* nbr_full = empty + S;
  uint64_t* nbr_empty = nbr_full + 2;
  uint64_t* acc_full = nbr_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain_bar = acc_empty + 2;
  WaitCtl* wctl = reinterpret_cast<WaitCtl*>(drain_bar + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wctl + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], GATHER_THREADS);  // every gather thread's cp.async arrive
      mbar_init(&wfull[s], 1);              // the TMA lane's arrive + the slice's bytes
      mbar_init(&empty[s], 1);              // one tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&nbr_full[b], 1);
      mbar_init(&nbr_empty[b], NUM_GATHER_WARPS);
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], NUM_EPI_WARPS * 32);
    }
    mbar_init(drain_bar, 1);
    wait_ctl_init(wctl, a.wait_limit_ns);
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == TMA_WARP && lane == 0) tma_prefetch_desc(&wmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  int64_t w_issued = 0;    // weight loads issued by the TMA warp (its abort-path drain)
  int64_t nbr_issued = 0;  // nbr tiles staged by the TMA warp

  if (warp >= GATHER_WARP0 && warp < GATHER_WARP0 + NUM_GATHER_WARPS) {
    // ---------------------------------------------------------- gather ----
    // Per step: wait for the slot, read this thread's row indices, issue its
    // 16-byte cp.async copies straight into the swizzled stage (zero-fill
    // where nbr = -1), and let the hardware arrive on the stage's barrier when
    // they have landed.  No register staging: the copies of up to `stages`
    // steps are in flight at once.
    const int gt = threadIdx.x - GATHER_WARP0 * 32;
    const int piece = gt % PPR;
    const int rbase = gt / PPR;
    uint32_t dst_off[PPT];  // swizzled byte offset of each piece in a stage
#pragma unroll
    for (int q = 0; q < PPT; ++q) {
      const int r = rbase + q * ROWS_PER_PASS;
      dst_off[q] = r * ROW_BYTES + ((piece ^ ((r * ROW_BYTES >> 7) & (PPR - 1))) << 4);
    }
    Steps st;
    st.begin(a);
    int ready_local = -1;
    while (st.valid) {
      if (st.local != ready_local) {
        if (!__all_sync(0xFFFFFFFFu,
                        mbar_wait(&nbr_full[st.local & 1], (st.local >> 1) & 1, wctl)))
          break;
        ready_local = st.local;
      }
      const int s = st.slot;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], st.phase ^ 1u, wctl))) break;
      const int32_t* nb = nbr_s + (st.local & 1) * (TV * kKvol) + rbase * kKvol + st.k;
      const __nv_bfloat16* xcol = a.x + st.j * CHUNK + piece * 8;
      const uint32_t b_base = smem_u32(stage_b) + static_cast<uint32_t>(s) * B_STAGE;
#pragma unroll
      for (int q = 0; q < PPT; ++q) {
        const int32_t src = nb[q * ROWS_PER_PASS * kKvol];
        cp_async_16(b_base + dst_off[q],
                    src >= 0 ? xcol + static_cast<int64_t>(src) * a.cin : a.x, src >= 0 ? 16u : 0u);
      }
      cp_async_mbar_arrive_noinc(&full[s]);
      const int old_local = st.local;
      if (st.next(a)) {  // the unit's last copies are issued: release its nbr buffer
        __syncwarp();
        if (lane == 0) mbar_arrive(&nbr_empty[old_local & 1]);
      }
    }
    cp_async_wait_all();
  } else if (warp == TMA_WARP) {
    // ------------------------------------------------------------- TMA ----
    const int64_t n_units = a.n_tiles * a.n_oblocks;
    // Stage the nbr rows of the unit with local index l into buffer l & 1.
    auto load_nbr = [&](int64_t u, int l) -> bool {
      const int buf = l & 1;
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait(&nbr_empty[buf], ((l >> 1) & 1) ^ 1, wctl)))
        return false;
      const int64_t row0 = (u / a.n_oblocks) * TV;
      int32_t* dst = nbr_s + buf * (TV * kKvol);
      if (row0 + TV <= a.n) {
        if (lane == 0) {
          fence_proxy_async_smem();  // earlier generic reads of this buffer come first
          mbar_arrive_expect_tx(&nbr_full[buf], kNbrTileBytes);
          bulk_load(smem_u32(dst), a.nbr + row0 * kKvol, kNbrTileBytes, &nbr_full[buf]);
        }
      } else {
        const int rows = static_cast<int>(a.n - row0);
        for (int e = lane; e < TV * kKvol; e += 32)
          dst[e] = (e / kKvol < rows) ? __ldg(a.nbr + row0 * kKvol + e) : -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&nbr_full[buf]);
      }
      ++nbr_issued;
      return true;
    };
    bool ok = true;
    if (blockIdx.x < n_units) ok = load_nbr(blockIdx.x, 0);
    Steps st;
    st.begin(a);
    int unit_local = -1;
    while (ok && st.valid) {
      if (st.local != unit_local) {  // entering a unit: prefetch the next unit's nbr rows
        unit_local = st.local;
        const int64_t nu = st.u + gridDim.x;
        if (nu < n_units && !load_nbr(nu, st.local + 1)) {
          ok = false;
          break;
        }
      }
      const int s = st.slot;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], st.phase ^ 1u, wctl))) {
        ok = false;
        break;
      }
      if (lane == 0) {
        const int kw = a.flip ? (kKvol - 1 - st.k) : st.k;
        const int o0 = static_cast<int>(st.u % a.n_oblocks) * TO;
        mbar_arrive_expect_tx(&wfull[s], A_STAGE);
        tma_load_3d(smem_u32(stage_a) + static_cast<uint32_t>(s) * A_STAGE, &wmap, &wfull[s],
                    st.j * CHUNK, kw, o0);
      }
      __syncwarp();
      ++w_issued;
      st.next(a);
    }
  } else if (warp == MMA_WARP) {
    // -------------------------------------------------------------- MMA ----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(TO, TV);
      Steps st;
      st.begin(a);
      bool ok = true;
      while (ok && st.valid) {
        const int local = st.local;
        const int acc = local & 1;
        if (!mbar_wait(&acc_empty[acc], ((local >> 1) & 1) ^ 1, wctl)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * TV);
        bool first = true;
        bool unit_done = false;
        while (!unit_done) {
          const int s = st.slot;
          if (!mbar_wait(&full[s], st.phase, wctl) || !mbar_wait(&wfull[s], st.phase, wctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stage_a) + static_cast<uint32_t>(s) * A_STAGE;
          const uint32_t b0 = smem_u32(stage_b) + static_cast<uint32_t>(s) * B_STAGE;
#pragma unroll
          for (int kk = 0; kk < CHUNK / 16; ++kk) {
            umma_bf16(d, smem_desc_sw(a0 + kk * 32, ROW_BYTES),
                      smem_desc_sw(b0 + kk * 32, ROW_BYTES), idesc,
                      (first && kk == 0) ? 0u : 1u);
          }
          first = false;
          umma_commit(&empty[s]);
          unit_done = st.next(a);
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue ----
    const int64_t n_units = a.n_tiles * a.n_oblocks;
    const uint32_t stage =
        smem_u32(epi_s) + static_cast<uint32_t>(warp) * static_cast<uint32_t>(kEpiWarpStageBytes);
    int local = 0;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
      const int acc = local & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[acc], (local >> 1) & 1, wctl))) break;
      tc_fence_after();
      const int64_t row0 = (u / a.n_oblocks) * TV;
      const int o_warp = static_cast<int>(u % a.n_oblocks) * TO + warp * 32;  // this warp's channels
      const float bias_v =
          (a.bias && o_warp + lane < a.cout) ? __bfloat162float(a.bias[o_warp + lane]) : 0.0f;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(acc * TV);
      if (o_warp < a.cout)  // a warp whose 32 channels all lie past Cout has nothing to store
        epilogue_tile_bf16<ACT, false>(taddr, bias_v, stage, lane, o_warp, a.cout, nullptr,
                                       row0, a.n, a.out, a.residual);
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();  // every role has left its loop; the abort word no longer changes
  if (wait_aborted(wctl)) {
    // copies and MMAs issued before the abort may still be in flight
    if (warp == TMA_WARP && lane == 0) {
      drain_ring(wfull, S, w_issued);
      drain_ring(nbr_full, 2, nbr_issued);
    }
    if (warp == MMA_WARP && lane == 0) drain_mma(drain_bar);
    tc_fence_before();
    __syncthreads();
  }
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0 && wait_aborted(wctl)) atomicExch(a.err_word, 1);
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

// Per-device one-time setup: large dynamic shared memory opt-in and SM count.
cudaError_t device_setup(int device, int* num_sms) {
  static std::mutex mu;
  static int sms[64] = {};
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (sms[device] == 0) {
    const void* kernels[9] = {
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<64, kActNone>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<32, kActNone>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<16, kActNone>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<64, kActGelu>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<32, kActGelu>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<16, kActGelu>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<64, kActSilu>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<32, kActSilu>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_sm100<16, kActSilu>)};
    for (const void* k : kernels) {
      const cudaError_t e =
          cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
      if (e != cudaSuccess) return e;
    }
    int count = 0;
    const cudaError_t e = cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, device);
    if (e != cudaSuccess) return e;
    sms[device] = count;
  }
  *num_sms = sms[device];
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_forward_bf16(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                                const void* feats, const void* weight, void* out, int32_t cin,
                                int32_t cout, int32_t flip, const Epilogue& epi, const DeviceCtl& ctl,
                                cudaStream_t stream) {
  EncodeTiledFn encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  int num_sms = 0;
  if ((e = device_setup(device, &num_sms)) != cudaSuccess) return e;

  const int chunk = cin % 64 == 0 ? 64 : (cin % 32 == 0 ? 32 : 16);
  int stages = 12;
  while (stages > 2 && plan_smem(chunk, stages).bytes > static_cast<size_t>(kSmemLimit)) --stages;
  const SmemPlan plan = plan_smem(chunk, stages);

  // Weight viewed as [Cout][27][Cin]; a box is 128 output channels x 1 offset x
  // one channel chunk.  Output channels past Cout read as zero.
  CUtensorMap wmap;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cin), 27, static_cast<cuuint64_t>(cout)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cin) * 2,
                                 static_cast<cuuint64_t>(cin) * 27 * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(chunk), 1, static_cast<cuuint32_t>(TO)};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle swz =
      chunk == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                  : (chunk == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(weight), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  FwdArgs a;
  a.nbr = nbr;
  a.tile_mask = tile_mask;
  a.x = static_cast<const __nv_bfloat16*>(feats);
  a.n = n;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.cin = cin;
  a.cout = cout;
  a.n_oblocks = (cout + TO - 1) / TO;
  a.n_kchunks = cin / chunk;
  a.stages = stages;
  a.flip = flip;
  a.bias = static_cast<const __nv_bfloat16*>(epi.bias);
  a.residual = static_cast<const __nv_bfloat16*>(epi.residual);
  a.n_tiles = (n + TV - 1) / TV;
  a.err_word = ctl.err_word;
  a.wait_limit_ns = ctl.wait_limit_ns;
  const int64_t units = a.n_tiles * a.n_oblocks;
  const unsigned grid = static_cast<unsigned>(units < num_sms ? units : num_sms);
  auto launch = [&](auto kernel) {
    kernel<<<grid, NUM_THREADS, plan.bytes, stream>>>(wmap, a);
  };
  auto by_act = [&](auto k_none, auto k_gelu, auto k_silu) {
    if (epi.act == kActGelu)
      launch(k_gelu);
    else if (epi.act == kActSilu)
      launch(k_silu);
    else
      launch(k_none);
  };
  if (chunk == 64)
    by_act(subm3d_fwd_bf16_sm100<64, kActNone>, subm3d_fwd_bf16_sm100<64, kActGelu>,
           subm3d_fwd_bf16_sm100<64, kActSilu>);
  else if (chunk == 32)
    by_act(subm3d_fwd_bf16_sm100<32, kActNone>, subm3d_fwd_bf16_sm100<32, kActGelu>,
           subm3d_fwd_bf16_sm100<32, kActSilu>);
  else
    by_act(subm3d_fwd_bf16_sm100<16, kActNone>, subm3d_fwd_bf16_sm100<16, kActGelu>,
           subm3d_fwd_bf16_sm100<16, kActSilu>);
  return cudaGetLastError();
}

}  // namespace subm3d

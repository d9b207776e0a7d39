// bf16 weight gradient over the x-run position layout, sm_100a tensor cores.
//
//   dW[o][kw][c] = sum_i dy[i][o] * x[nbr[i][k]][c],  kw = k or 26-k (flip),
//
// the gradient of the forward's definition (lato.2_mrp_mlx, commit 97dcdfb54a
// message: KRSC weights, the --flip-kernel mirror).  Over the x-run layout of
// the map build (see forward_bf16_runs_sm100.cu) the sum over voxels becomes a
// sum over positions p:  for the offset pair (dz, dy) and dx = d - 1,
//
//   D_d[o][c] += sum_p Ydense[p][o] * E_{dz,dy}[p + d - 1][c],
//
// Ydense[p] = dy[row of the voxel at p], zero at pads and empty positions.  So
// the contraction runs over positions (MMA K), with the output channels as M
// and the input channels as N, and both operands are the natural gathered
// tiles -- rows of positions, channels contiguous -- i.e. MN-major operands.
// One gathered E tile again serves all three dx, here inside one MMA: the B
// operand's N dimension holds three 64-channel atoms whose stride (LBO) is one
// 128-byte row, so atom d is the tile shifted by d rows (the 128-byte swizzle
// is keyed on address bits, so a view shifted by whole rows of an aligned slot
// is the same layout).
//
// A unit is (tile range, pair, 128 output channels, 128 input channels).  Each
// CTA takes units in turn; a unit's steps are half tiles (128 positions):
//   warps 4-11 (gather)  Y: 128 rows x 128 channels of dy, E: 130 rows (E rows
//       -1 .. 128 of the half) x 128 channels of x, 16-byte cp.async into two
//       64-channel 128-byte-swizzle slots each (zero-fill where absent),
//       completing the stage's barrier with cp.async.mbarrier.arrive.noinc.
//   warp 12 (MMA)        8 x 2 tcgen05.mma (M=128, N=192, K=16) per step into
//       two accumulators (384 TMEM columns), one per 64-channel chunk; the
//       B operand's three 64-channel atoms are set 128 bytes (one row) apart,
//       so they are the chunk's E rows shifted by dx = -1, 0, +1.
//   warps 0-3 (epilogue) at the end of a unit: tcgen05.ld of the two
//       accumulators and red.global.add.v4.f32 into the fp32 dW (zeroed by the
//       launcher), the unit's partial sum over its tile range.
// Every wait is bounded (ptx.cuh): a wait that runs out sets the library's
// device error word; the CTA lets its copies land, frees TMEM and exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace subm3d {
namespace {

constexpr int HP = 128;             // positions per step (half a position tile): MMA K per step
constexpr int OB = 128;             // output channels per unit: MMA M, TMEM lanes
constexpr int CB = 128;             // input channels per unit: MMA N
constexpr int ROW = 128;            // bytes per slot row: 64 bf16 channels
constexpr int YROWS = HP;           // Y rows per step
constexpr int EROWS = HP + 2;       // E rows per step: -1 .. 128 of the half
constexpr uint32_t Y_CHUNK = YROWS * ROW;                                   // 16384
constexpr uint32_t E_CHUNK = ((EROWS * ROW + 1023) / 1024) * 1024;           // 17408
constexpr uint32_t STAGE = 2 * Y_CHUNK + 2 * E_CHUNK;                        // 67584
constexpr int NSTAGE = 3;
constexpr int NUM_EPI_WARPS = 4;
constexpr int NUM_GATHER_WARPS = 8;
constexpr int GATHER_WARP0 = 4;
constexpr int MMA_WARP = GATHER_WARP0 + NUM_GATHER_WARPS;
constexpr int NUM_THREADS = (MMA_WARP + 1) * 32;
constexpr int GATHER_THREADS = NUM_GATHER_WARPS * 32;
constexpr uint32_t kAccCols = 192;   // per 64-channel chunk: dx-major, 3 x 64 columns
constexpr uint32_t kTmemCols = 512;  // two accumulators (the two chunks of a block)
constexpr size_t kSmemBytes = 1024 + NSTAGE * STAGE + 256;
static_assert(kSmemBytes <= 227 * 1024, "stages exceed shared memory");
static_assert(GATHER_THREADS == 16 * 16, "gather mapping: 16 pieces x 16 rows per pass");

struct WgradArgs {
  const int32_t* pos;  // position table
  const int32_t* et;   // E index table: 9 lines (one per dz-dy pair), `es` entries apart
  int64_t es;          // E line stride (entries)
  const int32_t* hdr;  // [runs, position tiles, positions, 0]
  const __nv_bfloat16* x;
  const __nv_bfloat16* dy;
  float* dw;           // [cout][27][cin], zeroed
  int32_t cin, cout, n_ob, n_cb, ranges, flip;
  int32_t* err_word;
  uint64_t wait_limit_ns;
};

// The step sequence of a CTA, walked identically by every role: units
// u = blockIdx.x, blockIdx.x + gridDim.x, ...; a unit's steps are the two halves
// of each tile of its range.  Units whose range is empty are skipped.
struct WSteps {
  int64_t u, n_units, n_tiles, per_range;
  int local;             // unit count within the CTA (accumulator phase)
  int pair, ob, cb;
  int64_t tile, tile_end;
  int half;
  int slot;
  uint32_t phase;
  bool valid;
  __device__ void set_unit(int n_ob, int n_cb) {
    while (u < n_units) {
      int64_t v = u;
      cb = static_cast<int>(v % n_cb);
      v /= n_cb;
      ob = static_cast<int>(v % n_ob);
      v /= n_ob;
      pair = static_cast<int>(v % 9);
      const int64_t r = v / 9;
      tile = r * per_range;
      tile_end = tile + per_range < n_tiles ? tile + per_range : n_tiles;
      if (tile < tile_end) break;
      u += gridDim.x;
    }
    valid = u < n_units;
    half = 0;
  }
  __device__ void begin(int64_t tiles, int ranges, int n_ob, int n_cb) {
    n_tiles = tiles;
    per_range = (tiles + ranges - 1) / ranges;
    n_units = static_cast<int64_t>(ranges) * 9 * n_ob * n_cb;
    u = blockIdx.x;
    local = 0;
    slot = 0;
    phase = 0;
    set_unit(n_ob, n_cb);
  }
  // Advances one step; returns true when it moved to a new unit (or ended).
  __device__ bool next(int n_ob, int n_cb) {
    if (++slot == NSTAGE) {
      slot = 0;
      phase ^= 1u;
    }
    if (++half < 2) return false;
    half = 0;
    if (++tile < tile_end) return false;
    u += gridDim.x;
    ++local;
    set_unit(n_ob, n_cb);
    return true;
  }
};

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1) subm3d_wgrad_bf16_runs_sm100(const WgradArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = base;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + NSTAGE * STAGE);
  uint64_t* empty = full + NSTAGE;
  uint64_t* acc_full = empty + NSTAGE;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain_bar = acc_empty + 1;
  WaitCtl* wctl = reinterpret_cast<WaitCtl*>(drain_bar + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wctl + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], GATHER_THREADS);  // every gather thread's cp.async arrive
      mbar_init(&empty[s], 1);              // one tcgen05.commit
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, NUM_EPI_WARPS * 32);
    mbar_init(drain_bar, 1);
    wait_ctl_init(wctl, a.wait_limit_ns);
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  const int64_t n_tiles = ld_dep(a.hdr + 1);

  if (warp >= GATHER_WARP0 && warp < MMA_WARP) {
    // ---------------------------------------------------------- gather ----
    const int gt = threadIdx.x - GATHER_WARP0 * 32;
    const int piece = gt % 16;       // 16-byte piece of a 256-byte (128-channel) row
    const int chunk = piece / 8;     // 64-channel slot
    const int col = piece % 8;       // 16-byte column within the 128-byte row
    const int rbase = gt / 16;       // 0..15: rows rbase, rbase + 16, ...
    WSteps st;
    st.begin(n_tiles, a.ranges, a.n_ob, a.n_cb);
    while (st.valid) {
      const int s = st.slot;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[s], st.phase ^ 1u, wctl))) break;
      const uint32_t y_base = smem_u32(ring) + static_cast<uint32_t>(s) * STAGE;
      const uint32_t e_base = y_base + 2 * Y_CHUNK;
      const int o = st.ob * OB + chunk * 64 + col * 8;   // dy channel of this piece
      const int c = st.cb * CB + chunk * 64 + col * 8;   // x channel of this piece
      const int32_t* posp = a.pos + st.tile * kPosTile + st.half * HP;
      const int32_t* etp = a.et + st.pair * a.es + st.tile * kPosTile + st.half * HP;
#pragma unroll
      for (int q = 0; q < YROWS / 16; ++q) {
        const int r = rbase + 16 * q;
        const int32_t e = ld_dep(posp + r);
        const bool ok = e >= 0 && (e & 3) == kPosVoxel && o < a.cout;
        const uint32_t dst = y_base + chunk * Y_CHUNK + r * ROW + ((col ^ (r & 7)) << 4);
        cp_async_16(dst, ok ? a.dy + static_cast<int64_t>(e >> 2) * a.cout + o : a.dy,
                    ok ? 16u : 0u);
      }
#pragma unroll
      for (int q = 0; q <= HP / 16; ++q) {
        const int r = rbase + 16 * q;  // E slot row r = E row r - 1 of the half
        if (q == HP / 16 && r >= EROWS) break;
        const int32_t e = ld_dep(etp + r);
        const bool ok = e >= 0 && c < a.cin;
        const uint32_t dst = e_base + chunk * E_CHUNK + r * ROW + ((col ^ (r & 7)) << 4);
        cp_async_16(dst, ok ? a.x + static_cast<int64_t>(e) * a.cin + c : a.x, ok ? 16u : 0u);
      }
      cp_async_mbar_arrive_noinc(&full[s]);
      st.next(a.n_ob, a.n_cb);
    }
    cp_async_wait_all();
  } else if (warp == MMA_WARP) {
    // -------------------------------------------------------------- MMA ----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32_mn(OB, kAccCols);
      WSteps st;
      st.begin(n_tiles, a.ranges, a.n_ob, a.n_cb);
      bool ok = true;
      while (ok && st.valid) {
        // the accumulators are free once the previous unit's epilogue has read them
        if (!mbar_wait(acc_empty, (st.local & 1) ^ 1, wctl)) break;
        tc_fence_after();
        bool first = true;
        bool unit_done = false;
        while (!unit_done) {
          const int s = st.slot;
          if (!mbar_wait(&full[s], st.phase, wctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t y_base = smem_u32(ring) + static_cast<uint32_t>(s) * STAGE;
          const uint32_t e_base = y_base + 2 * Y_CHUNK;
#pragma unroll
          for (int kk = 0; kk < HP / 16; ++kk) {
            const uint64_t da = smem_desc_mn_sw128(y_base + kk * 16 * ROW, Y_CHUNK, 1024);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              // N = 192: three 64-channel atoms ROW bytes apart = E rows shifted by
              // d = 0, 1, 2, i.e. dx = -1, 0, +1 of the same chunk in one MMA
              const uint64_t db =
                  smem_desc_mn_sw128(e_base + j * E_CHUNK + kk * 16 * ROW, ROW, 1024);
              umma_bf16(tmem_base + static_cast<uint32_t>(j * kAccCols), da, db, idesc,
                        (first && kk == 0) ? 0u : 1u);
            }
          }
          first = false;
          umma_commit(&empty[s]);
          unit_done = st.next(a.n_ob, a.n_cb);
        }
        if (!ok) break;
        umma_commit(acc_full);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue ----
    WSteps st;
    st.begin(n_tiles, a.ranges, a.n_ob, a.n_cb);
    while (st.valid) {
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(acc_full, st.local & 1, wctl))) break;
      tc_fence_after();
      const int o = st.ob * OB + warp * 32 + lane;
      const int c0 = st.cb * CB;
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
#pragma unroll 1
        for (int cc = 0; cc < static_cast<int>(kAccCols); cc += 32) {
          const int d = cc / 64;                  // column = d * 64 + channel in the chunk
          const int c = c0 + j * 64 + cc % 64;    // first input channel of these 32 columns
          const int k = 3 * st.pair + d;
          const int kw = a.flip ? (kKvol - 1 - k) : k;
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) +
                                 static_cast<uint32_t>(j * kAccCols + cc),
                             v);
          tmem_ld_wait();
          if (o < a.cout && c < a.cin) {
            float* dst = a.dw + (static_cast<int64_t>(o) * kKvol + kw) * a.cin + c;
            // cin is a multiple of 16: each 4-channel group is inside or past it
#pragma unroll
            for (int t = 0; t < 32; t += 4)
              if (c + t < a.cin)
                red_add_v4(dst + t, __uint_as_float(v[t]), __uint_as_float(v[t + 1]),
                           __uint_as_float(v[t + 2]), __uint_as_float(v[t + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
      // skip to the next unit: walk the steps of this one
      while (!st.next(a.n_ob, a.n_cb)) {
      }
    }
  }

  tc_fence_before();
  __syncthreads();  // every role has left its loop; the abort word no longer changes
  if (wait_aborted(wctl)) {
    // MMAs issued before the abort may still be running (the gather threads have
    // already waited for their own copies)
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

}  // namespace

cudaError_t launch_wgrad_bf16_runs(const int32_t* pos, const int32_t* etable,
                                   int64_t et_stride, const int32_t* header, const void* feats, const void* dy,
                                   float* dw, int32_t cin, int32_t cout, int32_t flip,
                                   const DeviceCtl& ctl, cudaStream_t stream) {
  static std::mutex mu;
  static int sms[64] = {0};
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (sms[device] == 0) {
      e = cudaFuncSetAttribute(subm3d_wgrad_bf16_runs_sm100,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmemBytes));
      if (e != cudaSuccess) return e;
      int count = 0;
      e = cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, device);
      if (e != cudaSuccess) return e;
      sms[device] = count;
    }
  }
  const int num_sms = sms[device];
  e = cudaMemsetAsync(dw, 0, static_cast<size_t>(cout) * kKvol * cin * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  WgradArgs a;
  a.pos = pos;
  a.et = etable;
  a.es = et_stride;
  a.hdr = header;
  a.x = static_cast<const __nv_bfloat16*>(feats);
  a.dy = static_cast<const __nv_bfloat16*>(dy);
  a.dw = dw;
  a.cin = cin;
  a.cout = cout;
  a.n_ob = (cout + OB - 1) / OB;
  a.n_cb = (cin + CB - 1) / CB;
  // one unit per SM: tile ranges x 9 pairs x channel blocks ~ the SM count
  const int combos = 9 * a.n_ob * a.n_cb;
  a.ranges = num_sms / combos > 0 ? num_sms / combos : 1;
  a.flip = flip;
  a.err_word = ctl.err_word;
  a.wait_limit_ns = ctl.wait_limit_ns;
  const int64_t units = static_cast<int64_t>(a.ranges) * combos;
  const unsigned grid = static_cast<unsigned>(units < num_sms ? units : num_sms);
  return launch_pdl(subm3d_wgrad_bf16_runs_sm100, grid, NUM_THREADS, kSmemBytes, stream, a);
}

}  // namespace subm3d

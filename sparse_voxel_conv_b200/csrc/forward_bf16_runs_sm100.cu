// bf16 forward over the x-run position layout, sm_100a tensor cores.
//
// Same op as forward_bf16_sm100.cu: out[i] = act( sum_k Wf[:, k, :] .
// x[nbr[i][k]] + bias ) + residual[i], Wf[:, k] = W[:, k] or W[:, 26-k] (flip), KRSC weights
// (lato.2_mrp_mlx, commit 97dcdfb54a message and CLAUDE.md "Key facts").
//
// The map build lays the voxels out on a line of positions in row order, with
// two pad positions before every run of x-adjacent voxels (the right pad of the
// previous run, the left pad of this one), and cuts the line into tiles of 256
// positions.  For a tile and an offset pair (dz, dy) it stores the E index
// list: E row p holds the (dz, dy, 0) neighbour of the voxel at position p, the
// (dz, dy, -1) neighbour of a left pad's voxel, the (dz, dy, +1) neighbour of a
// right pad's voxel, and rows -1 and 256 complete the tile's edges.  For every
// voxel at position p, E rows p-1, p and p+1 are therefore its dx = -1, 0, +1
// neighbours, so ONE gathered E tile serves three offsets: the MMA for offset
// (dz, dy, dx) reads B = E shifted by dx rows.  Gathered bytes drop ~3x against
// one gather per offset; the price is MMA work on the pad columns.
//
// With the output channels as M (128) and the 256 positions as N, the tile's
// fp32 accumulator D[o, p] (128 lanes x 256 columns) lives in tensor memory:
//
//     D[o, p] += sum_c Wf[o, k, c] * E_{dz,dy}[p + dx][c],  k = (dz, dy, dx)
//
// Persistent kernel, one CTA per SM; a work unit is a position tile x a block
// of 128 output channels.  Roles (14 warps):
//
//   warp 13 (TMA)   per E step (chunk j, pair dz-dy): loads the three weight
//       slices Wf[o0:o0+128, k, chunk j], dx = -1, 0, +1, into the W ring with
//       3-D TMA tiled loads (128-byte swizzle).
//   warps 4-11      gather E: once the E slot is free, 258 rows x 128 bytes with
//       16-byte cp.async into the 128-byte-swizzle layout (zero-fill for absent
//       rows), completing the slot's barrier with cp.async.mbarrier.arrive.noinc.
//       Each thread reads the E index entries of its rows straight from global
//       memory into registers one step ahead, so a freed slot waits for one
//       memory round trip (the rows), not two (the index list, then the rows).
//   warp 12 (MMA)   per E step, for dx = -1, 0, +1: 4 x tcgen05.mma (M=128,
//       N=256, K=16) with the B descriptor started dx rows into the E slot.
//       The 128-byte swizzle XORs with address bits [7,10) of each row's own
//       address, so a view shifted by whole 128-byte rows in a 1024-aligned
//       slot is the same swizzled layout: base offset 0, start + dx * 128.
//   warps 0-3       epilogue of the other accumulator: tcgen05.ld, bias,
//       activation (none, exact GELU, SiLU), a transpose through fp32 shared
//       memory, the residual, one bf16 rounding and 16-byte stores to the rows
//       of the voxel positions (pad columns are dropped).
//
// Every wait is bounded (ptx.cuh).  When one runs out, every role leaves its
// loop; after a CTA-wide barrier the TMA lane waits (bounded) for the weight
// loads it issued and the MMA lane commits to a drain barrier and waits for
// its MMAs, so that no copy or MMA is in flight when the CTA frees its tensor
// memory and exits; the library's device error word is then set.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "epilogue.cuh"

namespace subm3d {
namespace {

constexpr int TP = kPosTile;  // positions per tile (MMA N)
constexpr int TO = 128;       // output channels per unit (MMA M, TMEM lanes)
constexpr int CHUNK = 64;     // channels per step: one 128-byte swizzle row
constexpr int ROW_BYTES = CHUNK * 2;
constexpr int NUM_EPI_WARPS = 4;
constexpr int NUM_GATHER_WARPS = 8;
constexpr int GATHER_WARP0 = 4;
constexpr int MMA_WARP = GATHER_WARP0 + NUM_GATHER_WARPS;
constexpr int TMA_WARP = MMA_WARP + 1;
constexpr int NUM_THREADS = (TMA_WARP + 1) * 32;
constexpr int GATHER_THREADS = NUM_GATHER_WARPS * 32;
constexpr int kSmemLimit = 227 * 1024;
constexpr int kERows = TP + 2;                                   // rows -1 .. 256
constexpr uint32_t E_SLOT = ((kERows * ROW_BYTES + 1023) / 1024) * 1024;  // 33792
constexpr uint32_t A_SLOT = TO * ROW_BYTES;                      // 16384
constexpr int kEpiStageBytes = NUM_EPI_WARPS * kEpiWarpStageBytes;
constexpr uint32_t kTmemCols = 2 * TP;

struct RunArgs {
  const int32_t* pos;     // position table
  const int32_t* et;      // E index table: 9 lines (one per dz-dy pair), `es` entries apart
  const int32_t* hdr;     // [runs, position tiles, positions, 0]
  const __nv_bfloat16* x;
  __nv_bfloat16* out;
  const __nv_bfloat16* bias;      // [cout] or nullptr
  const __nv_bfloat16* residual;  // [N, cout] or nullptr; may be `out`
  int64_t es;             // E line stride (entries)
  int32_t cin, cout, n_oblocks, n_kchunks, se, sw, flip;
  int32_t* err_word;
  uint64_t wait_limit_ns;
};

struct SmemPlan {
  size_t e_off, w_off, epi_off, bar_off, bytes;
};

__host__ __device__ inline SmemPlan plan_smem(int se, int sw) {
  SmemPlan p;
  p.e_off = 0;
  p.w_off = p.e_off + static_cast<size_t>(se) * E_SLOT;
  p.epi_off = p.w_off + static_cast<size_t>(sw) * A_SLOT;
  p.bar_off = p.epi_off + kEpiStageBytes;
  // e_full[se], e_empty[se], w_full[sw], w_empty[sw], acc_full[2], acc_empty[2],
  // drain, WaitCtl (16 B), tmem slot
  p.bytes = p.bar_off + (2 * se + 2 * sw + 5) * 8 + 16 + 16 + 1024;
  return p;
}

// The (unit, chunk j, pair dzdy) E steps of a CTA, walked by every role.
struct ESteps {
  int64_t u, n_units;
  int local;         // unit index within the CTA (accumulator / parity selector)
  int j, dzdy;       // current chunk and offset pair
  int slot;          // E ring slot
  uint32_t phase;    // parity of that slot's current use
  bool valid;
  __device__ void begin(int64_t units) {
    n_units = units;
    u = blockIdx.x;
    local = 0;
    j = 0;
    dzdy = 0;
    slot = 0;
    phase = 0;
    valid = u < n_units;
  }
  // Advances one E step; returns true when it moved to a new unit (or ended).
  __device__ bool next(int n_kchunks, int se) {
    if (++slot == se) {
      slot = 0;
      phase ^= 1u;
    }
    if (++dzdy < 9) return false;
    dzdy = 0;
    if (++j < n_kchunks) return false;
    j = 0;
    u += gridDim.x;
    ++local;
    valid = u < n_units;
    return true;
  }
};

// A ring counter for the W slots (three per E step).
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  __device__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

template <int ACT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    subm3d_fwd_bf16_runs_sm100(const __grid_constant__ CUtensorMap wmap, const RunArgs a) {
  constexpr int PPR = CHUNK / 8;                       // 16-byte pieces per row: 8
  constexpr int ROWS_PER_PASS = GATHER_THREADS / PPR;  // 32
  constexpr int PPT = TP / ROWS_PER_PASS;              // 8 pieces per thread (+1 edge piece)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int SE = a.se, SW = a.sw;
  const SmemPlan plan = plan_smem(SE, SW);
  uint8_t* e_ring = base + plan.e_off;
  uint8_t* w_ring = base + plan.w_off;
  uint8_t* epi_s = base + plan.epi_off;
  uint64_t* e_full = reinterpret_cast<uint64_t*>(base + plan.bar_off);
  uint64_t* e_empty = e_full + SE;
  uint64_t* w_full = e_empty + SE;
  uint64_t* w_empty = w_full + SW;
  uint64_t* acc_full = w_empty + SW;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain_bar = acc_empty + 2;
  WaitCtl* wctl = reinterpret_cast<WaitCtl*>(drain_bar + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wctl + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SE; ++s) {
      mbar_init(&e_full[s], GATHER_THREADS);  // every gather thread's cp.async arrive
      mbar_init(&e_empty[s], 1);              // one tcgen05.commit
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
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
  pdl_wait();  // the setup above overlaps the map build's tail; global reads start here
  const int64_t n_tiles = ld_dep(a.hdr + 1);
  const int64_t n_units = n_tiles * a.n_oblocks;
  int64_t w_issued = 0;  // weight loads the TMA warp has issued (its abort-path drain)

  if (warp >= GATHER_WARP0 && warp < GATHER_WARP0 + NUM_GATHER_WARPS) {
    // ---------------------------------------------------------- gather ----
    const int gt = threadIdx.x - GATHER_WARP0 * 32;
    const int piece = gt % PPR;
    const int rbase = gt / PPR;                // 0..31
    const bool edge = rbase < 2;               // also copies E row 256 + rbase (rows -1 / 256 ...)
    uint32_t dst_off[PPT + 1];
#pragma unroll
    for (int q = 0; q <= PPT; ++q) {
      const int i = q < PPT ? rbase + q * ROWS_PER_PASS : TP + rbase;  // E index row 0..257
      dst_off[q] = i * ROW_BYTES + ((piece ^ (i & 7)) << 4);
    }
    // the E index entries of this thread's rows for the step `t` points at
    auto load_src = [&](const ESteps& t, int32_t (&v)[PPT + 1]) {
      // entries 256 tile .. 256 tile + 257 of the pair's line: E rows -1 .. 256
      const int32_t* list = a.et + t.dzdy * a.es + (t.u / a.n_oblocks) * TP;
#pragma unroll
      for (int q = 0; q <= PPT; ++q) {
        const int i = q < PPT ? rbase + q * ROWS_PER_PASS : TP + rbase;
        v[q] = (q < PPT || edge) ? ld_dep(list + i) : -1;
      }
    };
    ESteps st;
    st.begin(n_units);
    int32_t src[PPT + 1];
    if (st.valid) load_src(st, src);
    while (st.valid) {
      const int s = st.slot;
      // the E slot is free once the MMAs that read it are done
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&e_empty[s], st.phase ^ 1u, wctl))) break;
      const __nv_bfloat16* xcol = a.x + st.j * CHUNK + piece * 8;
      const uint32_t e_base = smem_u32(e_ring) + static_cast<uint32_t>(s) * E_SLOT;
      if (st.j * CHUNK + piece * 8 < a.cin) {
#pragma unroll
        for (int q = 0; q <= PPT; ++q) {
          if (q == PPT && !edge) break;
          cp_async_16(e_base + dst_off[q],
                      src[q] >= 0 ? xcol + static_cast<int64_t>(src[q]) * a.cin : a.x,
                      src[q] >= 0 ? 16u : 0u);
        }
      } else {
        // a piece past cin (the last chunk of a cin that is not a multiple of
        // 64): zeros, so that the chunk's four K steps add nothing there (the
        // weight slice's columns past cin are zero-filled by the TMA load)
#pragma unroll
        for (int q = 0; q <= PPT; ++q) {
          if (q == PPT && !edge) break;
          cp_async_16(e_base + dst_off[q], a.x, 0u);
        }
      }
      cp_async_mbar_arrive_noinc(&e_full[s]);
      st.next(a.n_kchunks, SE);
      if (st.valid) load_src(st, src);  // the next step's entries load while this slot fills
    }
    cp_async_wait_all();
  } else if (warp == TMA_WARP) {
    // ------------------------------------------------------------- TMA ----
    ESteps st;
    st.begin(n_units);
    Ring w;
    bool ok = true;
    while (ok && st.valid) {
      const int o0 = static_cast<int>(st.u % a.n_oblocks) * TO;
      for (int dx = 0; dx < 3; ++dx) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&w_empty[w.slot], w.phase ^ 1u, wctl))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          const int k = 3 * st.dzdy + dx;
          const int kw = a.flip ? (kKvol - 1 - k) : k;
          mbar_arrive_expect_tx(&w_full[w.slot], A_SLOT);
          tma_load_3d(smem_u32(w_ring) + static_cast<uint32_t>(w.slot) * A_SLOT, &wmap,
                      &w_full[w.slot], st.j * CHUNK, kw, o0);
        }
        __syncwarp();
        w.next(SW);
        ++w_issued;
      }
      st.next(a.n_kchunks, SE);
    }
  } else if (warp == MMA_WARP) {
    // -------------------------------------------------------------- MMA ----
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(TO, TP);
      ESteps st;
      st.begin(n_units);
      Ring w;
      bool ok = true;
      while (ok && st.valid) {
        const int local = st.local;
        const int acc = local & 1;
        if (!mbar_wait(&acc_empty[acc], ((local >> 1) & 1) ^ 1, wctl)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * TP);
        bool first = true;
        bool unit_done = false;
        while (!unit_done) {
          const int s = st.slot;
          if (!mbar_wait(&e_full[s], st.phase, wctl)) {
            ok = false;
            break;
          }
          const uint32_t e_base = smem_u32(e_ring) + static_cast<uint32_t>(s) * E_SLOT;
          for (int dx = 0; dx < 3; ++dx) {
            if (!mbar_wait(&w_full[w.slot], w.phase, wctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(w_ring) + static_cast<uint32_t>(w.slot) * A_SLOT;
            const uint32_t b0 = e_base + static_cast<uint32_t>(dx) * ROW_BYTES;  // E row dx-1
#pragma unroll
            for (int kk = 0; kk < CHUNK / 16; ++kk) {
              umma_bf16(d, smem_desc_sw(a0 + kk * 32, ROW_BYTES),
                        smem_desc_sw(b0 + kk * 32, ROW_BYTES), idesc,
                        (first && kk == 0) ? 0u : 1u);
              first = false;
            }
            umma_commit(&w_empty[w.slot]);
            w.next(SW);
          }
          if (!ok) break;
          umma_commit(&e_empty[s]);
          unit_done = st.next(a.n_kchunks, SE);
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue ----
    const uint32_t stage =
        smem_u32(epi_s) + static_cast<uint32_t>(warp) * static_cast<uint32_t>(kEpiWarpStageBytes);
    int local = 0;
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++local) {
      const int acc = local & 1;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[acc], (local >> 1) & 1, wctl))) break;
      tc_fence_after();
      const int64_t tile = u / a.n_oblocks;
      const int o_warp = static_cast<int>(u % a.n_oblocks) * TO + warp * 32;
      const float bias_v =
          (a.bias && o_warp + lane < a.cout) ? __bfloat162float(a.bias[o_warp + lane]) : 0.0f;
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(acc * TP);
      // voxel positions store to their row; pads and empty positions are dropped
      if (o_warp < a.cout)  // a warp whose 32 channels all lie past Cout has nothing to store
        epilogue_tile_bf16<ACT, true>(taddr, bias_v, stage, lane, o_warp, a.cout,
                                      a.pos + tile * TP, 0, 0, a.out, a.residual);
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();  // every role has left its loop; the abort word no longer changes
  if (wait_aborted(wctl)) {
    // copies and MMAs issued before the abort may still be in flight
    if (warp == TMA_WARP && lane == 0) drain_ring(w_full, SW, w_issued);
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

cudaError_t device_setup(int device, int* num_sms) {
  static std::mutex mu;
  static int sms[64] = {};
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (sms[device] == 0) {
    const void* kernels[3] = {
        reinterpret_cast<const void*>(subm3d_fwd_bf16_runs_sm100<kActNone>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_runs_sm100<kActGelu>),
        reinterpret_cast<const void*>(subm3d_fwd_bf16_runs_sm100<kActSilu>)};
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

cudaError_t launch_forward_bf16_runs(const int32_t* pos, const int32_t* etable,
                                     int64_t et_stride, const int32_t* header, int64_t max_tiles,
                                     const void* feats,
                                     const void* weight, void* out, int32_t cin, int32_t cout,
                                     int32_t flip, const Epilogue& epi, const DeviceCtl& ctl,
                                     cudaStream_t stream) {
  EncodeTiledFn encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  int num_sms = 0;
  if ((e = device_setup(device, &num_sms)) != cudaSuccess) return e;

  int se = 3, sw = 7;
  while (sw > 3 && plan_smem(se, sw).bytes > static_cast<size_t>(kSmemLimit)) --sw;
  const SmemPlan plan = plan_smem(se, sw);

  CUtensorMap wmap;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cin), 27, static_cast<cuuint64_t>(cout)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cin) * 2,
                                 static_cast<cuuint64_t>(cin) * 27 * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(CHUNK), 1, static_cast<cuuint32_t>(TO)};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (encode(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(weight), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  RunArgs a;
  a.pos = pos;
  a.et = etable;
  a.es = et_stride;
  a.hdr = header;
  a.x = static_cast<const __nv_bfloat16*>(feats);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.cin = cin;
  a.cout = cout;
  a.n_oblocks = (cout + TO - 1) / TO;
  a.n_kchunks = (cin + CHUNK - 1) / CHUNK;
  a.se = se;
  a.sw = sw;
  a.flip = flip;
  a.bias = static_cast<const __nv_bfloat16*>(epi.bias);
  a.residual = static_cast<const __nv_bfloat16*>(epi.residual);
  a.err_word = ctl.err_word;
  a.wait_limit_ns = ctl.wait_limit_ns;
  // the tile count lives on the device; launch for the largest possible count
  // and let each CTA read the actual one
  const int64_t units = max_tiles * a.n_oblocks;
  const unsigned grid = static_cast<unsigned>(units < num_sms ? units : num_sms);
  if (epi.act == kActGelu)
    return launch_pdl(subm3d_fwd_bf16_runs_sm100<kActGelu>, grid, NUM_THREADS, plan.bytes, stream,
                      wmap, a);
  if (epi.act == kActSilu)
    return launch_pdl(subm3d_fwd_bf16_runs_sm100<kActSilu>, grid, NUM_THREADS, plan.bytes, stream,
                      wmap, a);
  return launch_pdl(subm3d_fwd_bf16_runs_sm100<kActNone>, grid, NUM_THREADS, plan.bytes, stream,
                    wmap, a);
}

}  // namespace subm3d

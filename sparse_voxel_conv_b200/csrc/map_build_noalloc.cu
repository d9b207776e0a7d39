// Allocation-free variant of the neighbour-map build (subm3d_build_map_noalloc).
//
// subm3d_build_map() needs a workspace that the caller allocates.  Some callers
// cannot allocate device memory at the point where they build a map: a plugin
// running inside a host framework that owns and accounts for every device
// allocation, or a serving loop that must never call cudaMalloc/cudaFree once
// it is running, because those calls synchronise the device and take hundreds
// of microseconds.  This entry point needs no workspace: its scratch space (the
// status word and the hash table) is the file-scope device array below, which
// the CUDA runtime creates when the library is loaded, on every GPU the process
// uses, and keeps until the process exits.  Nothing here calls cudaMalloc,
// cudaFree or any other allocating routine.
//
// Set-up: the first call on each device looks up the array's device address
// with cudaGetSymbolAddress (with that device current) and caches it; host code
// never passes the array's name to a kernel, because in host code that name is
// only a host-side stand-in.  All calls on a device share the one array, so two
// calls whose work overlaps on the GPU (different streams, no ordering between
// them) race; every call re-initialises the table and the status word first.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "subm3d.h"

namespace {

// Scratch layout, as subm3d::map_layout() places it for the hash table:
// status word (256 B), tile masks (one word per 128 rows), the hash table
// (capacity 2 * max voxels, 8-byte slots) and, for wide keys, an int32 row
// per slot.  Sized for SUBM3D_NOALLOC_MAX_VOXELS voxels: about 12 MB.
constexpr size_t kMaxVoxels = SUBM3D_NOALLOC_MAX_VOXELS;
constexpr size_t kMaskBytes = (kMaxVoxels / subm3d::kTileRows) * 4;
constexpr size_t kSlots = 2 * kMaxVoxels;
constexpr size_t kScratchBytes = 256 + ((kMaskBytes + 255) / 256) * 256 + kSlots * 8 + kSlots * 4;

}  // namespace

static __device__ __align__(256) unsigned char g_map_scratch[kScratchBytes];

namespace {

// Device address of g_map_scratch on `device`, looked up once per device.
cudaError_t scratch_address(int device, void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_map_scratch);
    if (e != cudaSuccess) return e;
    addr[device] = p;
  }
  *out = addr[device];
  return cudaSuccess;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" {

subm3d_status subm3d_build_map_noalloc(const int32_t* coords, int64_t n, int32_t grid_dim,
                                       int32_t batch, int32_t* nbr, uint32_t* tile_mask,
                                       void* stream) {
  if (n < 0) return SUBM3D_E_INVALID;
  if (n > 0 && (!coords || !nbr || !tile_mask)) return SUBM3D_E_INVALID;
  if (n > static_cast<int64_t>(kMaxVoxels)) return SUBM3D_E_UNSUPPORTED;  // beyond the scratch
  subm3d::MapOptions opt;
  opt.force_hash = true;  // the hash table's size depends on N only, never on the volume
  opt.run_layout = false;  // nbr and tile masks are all subm3d_forward() needs
  subm3d::MapLayout lay;
  if (!subm3d::map_layout(n, grid_dim, batch, opt, &lay))
    return (grid_dim < 1 || batch < 1) ? SUBM3D_E_INVALID : SUBM3D_E_UNSUPPORTED;
  if (lay.total > kScratchBytes) return SUBM3D_E_UNSUPPORTED;
  if (n > 0 && (!aligned(coords, 16) || !aligned(nbr, 16) || !aligned(tile_mask, 4)))
    return SUBM3D_E_INVALID;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return SUBM3D_E_CUDA;
  void* scratch = nullptr;
  if (scratch_address(device, &scratch) != cudaSuccess) return SUBM3D_E_CUDA;
  auto s = static_cast<cudaStream_t>(stream);
  if (subm3d::launch_map_build(coords, n, grid_dim, batch, nbr, scratch, lay, s) != cudaSuccess)
    return SUBM3D_E_CUDA;
  if (n > 0 &&
      cudaMemcpyAsync(tile_mask, static_cast<unsigned char*>(scratch) + lay.mask_off,
                      static_cast<size_t>(lay.n_tiles) * 4, cudaMemcpyDeviceToDevice,
                      s) != cudaSuccess)
    return SUBM3D_E_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, static_cast<unsigned char*>(scratch) + lay.status_off, sizeof(word),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SUBM3D_E_CUDA;
  if (word & subm3d::kErrRange) return SUBM3D_E_RANGE;
  if (word & subm3d::kErrDuplicate) return SUBM3D_E_DUPLICATE;
  if (word & subm3d::kErrTableFull) return SUBM3D_E_TABLE_FULL;
  return SUBM3D_OK;
}

}  // extern "C"

// C ABI of the submanifold 3x3x3 sparse convolution (include/subm3d.h):
// argument checks, workspace sizing, the map handle, and kernel dispatch.
// No device memory is allocated here; every buffer belongs to the caller.
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "subm3d.h"

// The library's device error word: set to 1 by a forward kernel whose bounded
// wait ran out; read and cleared by subm3d_device_status().
static __device__ int32_t g_subm3d_error_word;

struct subm3d_map {
  const int32_t* nbr;
  const uint32_t* tile_mask;
  const uint32_t* status_word;
  const int32_t* pos;     // x-run position table
  const int32_t* et;      // E index table
  const int32_t* hdr;     // [runs, position tiles, positions, 0]
  int64_t ptile_max;      // position tiles reserved in the workspace
  const void* workspace;  // the build's workspace, laid out as `layout`
  subm3d::MapLayout layout;
  int64_t n;
  int32_t grid_dim;
  int32_t batch;
  cudaStream_t stream;
};

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Testing knobs read from the environment at every call:
//   SUBM3D_TABLE_CAPACITY=<slots>  caps the hash table (and selects it), so that
//                                  a full table can be exercised;
//   SUBM3D_MAP_KIND=hash           uses the hash table even where the direct
//                                  or brick table would fit;
//   SUBM3D_MAP_KIND=brick|direct   uses that table wherever it fits (within
//                                  the direct table's size budget).
subm3d::MapOptions options_from_env() {
  subm3d::MapOptions o;
  const char* cap = std::getenv("SUBM3D_TABLE_CAPACITY");
  if (cap && *cap) o.forced_capacity = std::strtoull(cap, nullptr, 10);
  const char* kind = std::getenv("SUBM3D_MAP_KIND");
  if (kind && std::strcmp(kind, "hash") == 0) o.force_hash = true;
  if (kind && std::strcmp(kind, "brick") == 0) o.force_brick = true;
  if (kind && std::strcmp(kind, "direct") == 0) o.force_direct = true;
  return o;
}

// 1 when the current device is sm_100 (B200 class), 0 when it is not, -1 on error.
int device_is_sm100(int* device_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  static std::mutex mu;
  static signed char cache[64];
  static bool init = false;
  std::lock_guard<std::mutex> lock(mu);
  if (!init) {
    std::memset(cache, -1, sizeof(cache));
    init = true;
  }
  if (device_out) *device_out = dev;
  if (dev >= 0 && dev < 64 && cache[dev] >= 0) return cache[dev];
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return -1;
  const int ok = (major == 10 && minor == 0) ? 1 : 0;
  if (dev >= 0 && dev < 64) cache[dev] = static_cast<signed char>(ok);
  return ok;
}

// Limit of each pipeline wait inside the tensor-core kernels: 2 s, or the
// testing knob SUBM3D_WAIT_LIMIT_NS=<ns> (read at every call), with which a
// test makes the waits run out and checks the timeout path.
uint64_t wait_limit_from_env() {
  const char* v = std::getenv("SUBM3D_WAIT_LIMIT_NS");
  if (v && *v) {
    const unsigned long long ns = std::strtoull(v, nullptr, 10);
    if (ns > 0) return ns;
  }
  return 2000000000ull;
}

int32_t* device_error_word() {
  static std::mutex mu;
  static int32_t* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_subm3d_error_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int32_t*>(p);
  }
  return addr[dev];
}

}  // namespace

extern "C" {

int32_t subm3d_abi_version(void) { return SUBM3D_ABI_VERSION; }

const char* subm3d_status_string(int32_t status) {
  switch (status) {
    case SUBM3D_OK: return "ok";
    case SUBM3D_E_INVALID: return "invalid argument";
    case SUBM3D_E_RANGE: return "coordinate out of range";
    case SUBM3D_E_DUPLICATE: return "duplicate coordinate";
    case SUBM3D_E_TABLE_FULL: return "hash table full";
    case SUBM3D_E_UNSUPPORTED: return "unsupported shape, alignment or device";
    case SUBM3D_E_CUDA: return "CUDA runtime error";
    case SUBM3D_E_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

size_t subm3d_map_workspace_bytes(int64_t n, int32_t grid_dim, int32_t batch) {
  subm3d::MapLayout lay;
  if (!subm3d::map_layout(n, grid_dim, batch, options_from_env(), &lay)) return 0;
  return lay.total;
}

subm3d_status subm3d_build_map(const int32_t* coords, int64_t n, int32_t grid_dim,
                               int32_t batch, int32_t* nbr, void* workspace,
                               size_t workspace_bytes, void* stream, subm3d_map** out_map) {
  if (!out_map) return SUBM3D_E_INVALID;
  *out_map = nullptr;
  if (n < 0 || !workspace) return SUBM3D_E_INVALID;
  if (n > 0 && (!coords || !nbr)) return SUBM3D_E_INVALID;
  subm3d::MapLayout lay;
  if (!subm3d::map_layout(n, grid_dim, batch, options_from_env(), &lay))
    return (grid_dim < 1 || batch < 1) ? SUBM3D_E_INVALID : SUBM3D_E_UNSUPPORTED;
  if (workspace_bytes < lay.total) return SUBM3D_E_INVALID;
  if (!aligned(coords, 16) || !aligned(nbr, 16) || !aligned(workspace, 256))
    return SUBM3D_E_INVALID;
  auto* h = new (std::nothrow) subm3d_map;
  if (!h) return SUBM3D_E_INVALID;
  auto* ws = static_cast<uint8_t*>(workspace);
  h->nbr = nbr;
  h->tile_mask = reinterpret_cast<const uint32_t*>(ws + lay.mask_off);
  h->status_word = reinterpret_cast<const uint32_t*>(ws + lay.status_off);
  const bool runs = lay.ptile_max > 0;
  h->pos = runs ? reinterpret_cast<const int32_t*>(ws + lay.pos_off) : nullptr;
  h->et = runs ? reinterpret_cast<const int32_t*>(ws + lay.et_off) : nullptr;
  h->hdr = runs ? reinterpret_cast<const int32_t*>(ws + lay.hdr_off) : nullptr;
  h->ptile_max = lay.ptile_max;
  h->workspace = workspace;
  h->layout = lay;
  h->n = n;
  h->grid_dim = grid_dim;
  h->batch = batch;
  h->stream = static_cast<cudaStream_t>(stream);
  if (subm3d::launch_map_build(coords, n, grid_dim, batch, nbr, workspace, lay,
                               h->stream) != cudaSuccess) {
    delete h;
    return SUBM3D_E_CUDA;
  }
  *out_map = h;
  return SUBM3D_OK;
}

subm3d_status subm3d_map_status(const subm3d_map* map) {
  if (!map) return SUBM3D_E_INVALID;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, map->status_word, sizeof(word), cudaMemcpyDeviceToHost,
                      map->stream) != cudaSuccess ||
      cudaStreamSynchronize(map->stream) != cudaSuccess)
    return SUBM3D_E_CUDA;
  if (word & subm3d::kErrRange) return SUBM3D_E_RANGE;
  if (word & subm3d::kErrDuplicate) return SUBM3D_E_DUPLICATE;
  if (word & subm3d::kErrTableFull) return SUBM3D_E_TABLE_FULL;
  return SUBM3D_OK;
}

const int32_t* subm3d_map_nbr(const subm3d_map* map) { return map ? map->nbr : nullptr; }
const uint32_t* subm3d_map_tile_mask(const subm3d_map* map) {
  return map ? map->tile_mask : nullptr;
}
int64_t subm3d_map_size(const subm3d_map* map) { return map ? map->n : -1; }
int32_t subm3d_map_table(const subm3d_map* map) {
  if (!map) return -1;
  switch (map->layout.kind) {
    case subm3d::MapKind::kDirect: return SUBM3D_TABLE_DIRECT;
    case subm3d::MapKind::kBrick: return SUBM3D_TABLE_BRICK;
    default: return SUBM3D_TABLE_HASH;
  }
}
void subm3d_map_destroy(subm3d_map* map) { delete map; }

namespace {

bool overlaps(const void* p, size_t p_bytes, const void* q, size_t q_bytes) {
  const auto* a = static_cast<const uint8_t*>(p);
  const auto* b = static_cast<const uint8_t*>(q);
  return a < b + q_bytes && b < a + p_bytes;
}

// Kernel choice for a map with an x-run layout: the x-run kernel when Cin >= 48.
// It does tensor work on every position (voxels and pads) for all 27 offsets,
// the per-offset kernel on every voxel for the offsets present in its 256-row
// tile but with ~3x the gathered bytes; timed with the GELU epilogue on three
// sets (x-runs of 9.3 and 4.0 voxels, 1.22 and 1.50 positions per voxel) at 64
// and 128 input and output channels, the x-run kernel was faster in every case,
// by 14% (4 x 256^3 shells, 64 -> 128) to 2.1x; with a partial last chunk it is
// 2.0-2.3x faster at 48 and 80 input channels on the headline set and 1.4x at
// 96 -> 64 on the decoder-stack set, but at 32 channels (half of its only
// chunk zeros) it is no faster than the per-offset kernel, which keeps Cin < 48.
// Testing knob SUBM3D_FORWARD_KERNEL (read at every call): "gather" takes the
// per-offset kernel even where the x-run kernel applies.
bool prefer_gather() {
  const char* knob = std::getenv("SUBM3D_FORWARD_KERNEL");
  return knob && std::strcmp(knob, "gather") == 0;
}

// The forward of every entry point: map may be null (nbr-only callers), in
// which case the x-run kernel is not available.
subm3d_status forward_impl(const subm3d_map* map, const int32_t* nbr, const uint32_t* tile_mask,
                           int64_t n, const void* feats, const void* weight, const void* bias,
                           const void* residual, void* out, int32_t cin, int32_t cout,
                           subm3d_dtype dtype, int32_t flip, subm3d_act act, void* stream) {
  if (n < 0 || cin < 1 || cout < 1) return SUBM3D_E_INVALID;
  if (dtype != SUBM3D_F32 && dtype != SUBM3D_BF16) return SUBM3D_E_INVALID;
  if (act != SUBM3D_ACT_NONE && act != SUBM3D_ACT_GELU && act != SUBM3D_ACT_SILU)
    return SUBM3D_E_INVALID;
  if (n > 0 && (!nbr || !feats || !weight || !out)) return SUBM3D_E_INVALID;
  if (n >= 0x7FFFFFFFll) return SUBM3D_E_UNSUPPORTED;
  if (n == 0) return SUBM3D_OK;
  const size_t esz = dtype == SUBM3D_BF16 ? 2 : 4;
  const size_t out_bytes = static_cast<size_t>(n) * cout * esz;
  if (overlaps(feats, static_cast<size_t>(n) * cin * esz, out, out_bytes))
    return SUBM3D_E_INVALID;  // out overlaps feats
  if (residual && residual != out && overlaps(residual, out_bytes, out, out_bytes))
    return SUBM3D_E_INVALID;  // a residual partly overlapping out would race
  auto s = static_cast<cudaStream_t>(stream);
  const int flip01 = flip ? 1 : 0;
  subm3d::Epilogue epi;
  epi.bias = bias;
  epi.residual = residual;
  epi.act = act == SUBM3D_ACT_GELU ? subm3d::kActGelu
                                   : (act == SUBM3D_ACT_SILU ? subm3d::kActSilu : subm3d::kActNone);
  if (dtype == SUBM3D_F32) {
    if (!aligned(nbr, 4) || !aligned(feats, 4) || !aligned(weight, 4) || !aligned(out, 4) ||
        (tile_mask && !aligned(tile_mask, 4)) || !aligned(bias, 4) || !aligned(residual, 4))
      return SUBM3D_E_INVALID;
    return subm3d::launch_forward_f32(nbr, tile_mask, n, static_cast<const float*>(feats),
                                      static_cast<const float*>(weight), static_cast<float*>(out),
                                      cin, cout, flip01, epi, s) == cudaSuccess
               ? SUBM3D_OK
               : SUBM3D_E_CUDA;
  }
  if (cin % 16 != 0 || cout % 16 != 0) return SUBM3D_E_UNSUPPORTED;
  if (!aligned(nbr, 16) || !aligned(feats, 16) || !aligned(weight, 16) || !aligned(out, 16) ||
      (tile_mask && !aligned(tile_mask, 4)) || !aligned(bias, 2) || !aligned(residual, 16))
    return SUBM3D_E_UNSUPPORTED;
  const int sm100 = device_is_sm100(nullptr);
  if (sm100 < 0) return SUBM3D_E_CUDA;
  if (sm100 == 0) return SUBM3D_E_UNSUPPORTED;
  subm3d::DeviceCtl ctl;
  ctl.err_word = device_error_word();
  if (!ctl.err_word) return SUBM3D_E_CUDA;
  ctl.wait_limit_ns = wait_limit_from_env();
  cudaError_t e;
  if (map && map->pos && cin >= 48 && !prefer_gather())  // cin % 16 == 0 (checked above)
    e = subm3d::launch_forward_bf16_runs(map->pos, map->et, map->layout.et_stride, map->hdr,
                                         map->ptile_max, feats,
                                         weight, out, cin, cout, flip01, epi, ctl, s);
  else
    e = subm3d::launch_forward_bf16(nbr, tile_mask, n, feats, weight, out, cin, cout, flip01, epi,
                                    ctl, s);
  if (e == cudaErrorNotSupported) return SUBM3D_E_UNSUPPORTED;
  return e == cudaSuccess ? SUBM3D_OK : SUBM3D_E_CUDA;
}

}  // namespace

subm3d_status subm3d_forward(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                             const void* feats, const void* weight, void* out, int32_t cin,
                             int32_t cout, subm3d_dtype dtype, int32_t flip, subm3d_act act,
                             void* stream) {
  return forward_impl(nullptr, nbr, tile_mask, n, feats, weight, nullptr, nullptr, out, cin, cout,
                      dtype, flip, act, stream);
}

subm3d_status subm3d_map_run_layout(const subm3d_map* map, const int32_t** pos,
                                    const int32_t** etable, const int32_t** header) {
  if (!map || !pos || !etable || !header) return SUBM3D_E_INVALID;
  if (!map->pos) return SUBM3D_E_UNSUPPORTED;
  *pos = map->pos;
  *etable = map->et;
  *header = map->hdr;
  return SUBM3D_OK;
}

subm3d_status subm3d_forward_map(const subm3d_map* map, const void* feats, const void* weight,
                                 void* out, int32_t cin, int32_t cout, subm3d_dtype dtype,
                                 int32_t flip, subm3d_act act, void* stream) {
  if (!map) return SUBM3D_E_INVALID;
  return forward_impl(map, map->nbr, map->tile_mask, map->n, feats, weight, nullptr, nullptr, out,
                      cin, cout, dtype, flip, act, stream);
}

subm3d_status subm3d_forward_fused(const subm3d_map* map, const void* feats, const void* weight,
                                   const void* bias, const void* residual, void* out, int32_t cin,
                                   int32_t cout, subm3d_dtype dtype, int32_t flip, subm3d_act act,
                                   void* stream) {
  if (!map) return SUBM3D_E_INVALID;
  return forward_impl(map, map->nbr, map->tile_mask, map->n, feats, weight, bias, residual, out,
                      cin, cout, dtype, flip, act, stream);
}

subm3d_status subm3d_backward_data(const subm3d_map* map, const void* dy, const void* weight,
                                   void* weight_t, void* dx, int32_t cin, int32_t cout,
                                   subm3d_dtype dtype, int32_t flip, void* stream) {
  if (!map || cin < 1 || cout < 1) return SUBM3D_E_INVALID;
  if (dtype != SUBM3D_F32 && dtype != SUBM3D_BF16) return SUBM3D_E_INVALID;
  if (map->n == 0) return SUBM3D_OK;
  if (!dy || !weight || !weight_t || !dx) return SUBM3D_E_INVALID;
  const size_t esz = dtype == SUBM3D_BF16 ? 2 : 4;
  const size_t w_bytes = static_cast<size_t>(cout) * 27 * cin * esz;
  if (overlaps(weight, w_bytes, weight_t, w_bytes)) return SUBM3D_E_INVALID;
  if (!aligned(weight, esz) || !aligned(weight_t, 16)) return SUBM3D_E_INVALID;
  auto s = static_cast<cudaStream_t>(stream);
  if (subm3d::launch_transpose_weight(weight, weight_t, cout, cin, dtype == SUBM3D_BF16, s) !=
      cudaSuccess)
    return SUBM3D_E_CUDA;
  // dx = forward of dy with W^T (Cout -> Cin) and the opposite orientation
  return forward_impl(map, map->nbr, map->tile_mask, map->n, dy, weight_t, nullptr, nullptr, dx,
                      cout, cin, dtype, flip ? 0 : 1, SUBM3D_ACT_NONE, stream);
}

subm3d_status subm3d_backward_weight(const subm3d_map* map, const void* feats, const void* dy,
                                     float* dweight, int32_t cin, int32_t cout,
                                     subm3d_dtype dtype, int32_t flip, void* stream) {
  if (!map || cin < 1 || cout < 1 || !dweight) return SUBM3D_E_INVALID;
  if (dtype != SUBM3D_F32 && dtype != SUBM3D_BF16) return SUBM3D_E_INVALID;
  const int64_t n = map->n;
  if (n > 0 && (!feats || !dy)) return SUBM3D_E_INVALID;
  const size_t esz = dtype == SUBM3D_BF16 ? 2 : 4;
  if (!aligned(feats, esz) || !aligned(dy, esz) || !aligned(dweight, 4)) return SUBM3D_E_INVALID;
  const size_t dw_bytes = static_cast<size_t>(cout) * 27 * cin * 4;
  if (n > 0 && (overlaps(dweight, dw_bytes, feats, static_cast<size_t>(n) * cin * esz) ||
                overlaps(dweight, dw_bytes, dy, static_cast<size_t>(n) * cout * esz)))
    return SUBM3D_E_INVALID;
  auto s = static_cast<cudaStream_t>(stream);
  if (n > 0 && dtype == SUBM3D_BF16 && map->pos && cin % 16 == 0 && cout % 16 == 0 &&
      aligned(feats, 16) && aligned(dy, 16) && aligned(dweight, 16) && device_is_sm100(nullptr) == 1) {
    subm3d::DeviceCtl ctl;
    ctl.err_word = device_error_word();
    if (!ctl.err_word) return SUBM3D_E_CUDA;
    ctl.wait_limit_ns = wait_limit_from_env();
    return subm3d::launch_wgrad_bf16_runs(map->pos, map->et, map->layout.et_stride, map->hdr,
                                          feats, dy, dweight, cin,
                                          cout, flip ? 1 : 0, ctl, s) == cudaSuccess
               ? SUBM3D_OK
               : SUBM3D_E_CUDA;
  }
  int device = 0, sms = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return SUBM3D_E_CUDA;
  return subm3d::launch_wgrad(map->nbr, n, feats, dy, dweight, cin, cout, flip ? 1 : 0,
                              dtype == SUBM3D_BF16, sms, s) ==
                 cudaSuccess
             ? SUBM3D_OK
             : SUBM3D_E_CUDA;
}

size_t subm3d_expand_workspace_bytes(int64_t n) {
  if (n < 0 || n >= (int64_t(1) << 28)) return 0;
  return subm3d::expand_layout(n).bytes;
}

subm3d_status subm3d_expand(const int32_t* coords, const void* feats, const uint8_t* mask,
                            int64_t n, int32_t channels_out, subm3d_dtype dtype,
                            subm3d_expand_mode mode, int32_t* out_coords, void* out_feats,
                            void* workspace, size_t workspace_bytes, int64_t* out_count,
                            void* stream) {
  if (!out_count || n < 0 || channels_out < 1) return SUBM3D_E_INVALID;
  *out_count = 0;
  if (dtype != SUBM3D_F32 && dtype != SUBM3D_BF16) return SUBM3D_E_INVALID;
  if (mode != SUBM3D_EXPAND_SUBDIVIDE && mode != SUBM3D_EXPAND_UPSAMPLE &&
      mode != SUBM3D_EXPAND_CHANNEL2SPATIAL)
    return SUBM3D_E_INVALID;
  if ((mode == SUBM3D_EXPAND_SUBDIVIDE && mask) || (mode == SUBM3D_EXPAND_UPSAMPLE && !mask))
    return SUBM3D_E_INVALID;
  if (n >= (int64_t(1) << 28)) return SUBM3D_E_UNSUPPORTED;
  if (n == 0) return SUBM3D_OK;
  if (!coords || !feats || !out_coords || !out_feats || !workspace) return SUBM3D_E_INVALID;
  if (workspace_bytes < subm3d::expand_layout(n).bytes) return SUBM3D_E_INVALID;
  const size_t esz = dtype == SUBM3D_BF16 ? 2 : 4;
  if (!aligned(coords, 16) || !aligned(out_coords, 16) || !aligned(workspace, 256) ||
      !aligned(feats, esz) || !aligned(out_feats, esz))
    return SUBM3D_E_INVALID;
  const bool slice = mode == SUBM3D_EXPAND_CHANNEL2SPATIAL;
  const int64_t out_row = static_cast<int64_t>(channels_out) * esz;
  const int64_t in_row = slice ? 8 * out_row : out_row;
  const cudaError_t e = subm3d::launch_expand(
      coords, feats, mask, n, in_row, out_row, slice, mode == SUBM3D_EXPAND_SUBDIVIDE, out_coords,
      out_feats, workspace, out_count, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SUBM3D_OK : SUBM3D_E_CUDA;
}

size_t subm3d_pool_workspace_bytes(int64_t n, int32_t grid_dim, int32_t batch) {
  if (n < 0 || grid_dim < 1 || grid_dim > 65535 || batch < 1 || batch > 65535) return 0;
  const subm3d::PoolLayout l = subm3d::pool_layout(n, grid_dim, batch);
  if (l.cells > (int64_t(1) << 30)) return 0;
  return l.bytes;
}

subm3d_status subm3d_pool(const subm3d_map* fine, const int32_t* coords, const void* feats,
                          int32_t channels, subm3d_dtype dtype, subm3d_pool_mode mode,
                          int32_t* out_coords, void* out_feats, void* workspace,
                          size_t workspace_bytes, int64_t* out_count, void* stream) {
  if (!fine || !out_count || channels < 1) return SUBM3D_E_INVALID;
  *out_count = 0;
  if (dtype != SUBM3D_F32 && dtype != SUBM3D_BF16) return SUBM3D_E_INVALID;
  if (mode != SUBM3D_POOL_MAX && mode != SUBM3D_POOL_MEAN && mode != SUBM3D_POOL_SPATIAL2CHANNEL)
    return SUBM3D_E_INVALID;
  const int64_t n = fine->n;
  const size_t need = subm3d_pool_workspace_bytes(n, fine->grid_dim, fine->batch);
  if (need == 0) return SUBM3D_E_UNSUPPORTED;
  if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return SUBM3D_E_INVALID;
  if (n > 0 && (!coords || !feats || !out_coords || !out_feats)) return SUBM3D_E_INVALID;
  const size_t esz = dtype == SUBM3D_BF16 ? 2 : 4;
  if (!aligned(coords, 16) || !aligned(out_coords, 16) || !aligned(feats, esz) ||
      !aligned(out_feats, esz))
    return SUBM3D_E_INVALID;
  const cudaError_t e = subm3d::launch_pool(
      fine->layout, fine->workspace, fine->grid_dim, fine->batch, coords, n, feats, channels,
      dtype == SUBM3D_BF16, static_cast<int>(mode), out_coords, out_feats, workspace, out_count,
      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SUBM3D_OK : SUBM3D_E_CUDA;
}

subm3d_status subm3d_device_status(void* stream) {
  int32_t* err = device_error_word();
  if (!err) return SUBM3D_E_CUDA;
  auto s = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  const int32_t zero = 0;
  if (cudaMemcpyAsync(&word, err, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(err, &zero, sizeof(zero), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SUBM3D_E_CUDA;
  return word ? SUBM3D_E_TIMEOUT : SUBM3D_OK;
}

}  // extern "C"

/*
 * subm3d.h -- C ABI of the B200 (sm_100a) submanifold 3x3x3 sparse convolution.
 *
 * The op (lato.2_mrp_mlx, commit 97dcdfb54a message and CLAUDE.md "Key facts"):
 * every SparseConv3d of the sparse-voxel generators is a submanifold
 * convolution, kernel 3x3x3, stride 1, whose output sites are exactly its input
 * sites.  For a set of N voxels p_i = (b, z, y, x):
 *
 *     out[i] = sum_{k=0}^{26} W[:, k, :] . feats[nbr[i][k]]      (nbr != -1)
 *
 * where nbr[i][k] is the row of the voxel at p_i + d_k, the 27 offsets d_k are
 * ordered kz-major, k = 9*(dz+1) + 3*(dy+1) + (dx+1), and W is spconv's KRSC
 * weight [Cout, kz, ky, kx, Cin] (same notes).  This is correlation; `flip`
 * selects the mirrored kernel W[:, 26-k, :] because the pages leave the
 * orientation unverified (same commit message, "--flip-kernel"; notes,
 * "Unresolved").  The map is built once per coordinate set and reused by
 * every layer on that set, as spconv does with indice_key (same message).
 *
 * Entry points, in order below: the map build (subm3d_map_workspace_bytes,
 * subm3d_build_map, subm3d_map_status and accessors, subm3d_build_map_noalloc);
 * the forward (subm3d_forward on nbr, subm3d_forward_map on a map,
 * subm3d_forward_fused with a residual-block epilogue); the backward
 * (subm3d_backward_data, subm3d_backward_weight); the resolution changes
 * (subm3d_expand: subdivide / upsample / channel2spatial; subm3d_pool:
 * downsample max / mean, spatial2channel); diagnostics (subm3d_map_run_layout,
 * subm3d_device_status, subm3d_status_string, subm3d_abi_version).
 *
 * Conventions for every entry point:
 *   - All buffers are caller-owned.  Pointers marked (device) must point to
 *     memory of the current CUDA device; (host) to host memory.  The library
 *     never allocates device memory; the map's scratch space is a caller
 *     workspace sized by subm3d_map_workspace_bytes().
 *   - `stream` is a cudaStream_t (0 = legacy default stream).  Work is
 *     enqueued on it and the call returns without waiting, unless noted.
 *   - Argument errors are detected on the host, before anything is enqueued,
 *     and returned synchronously.  Data errors in the coordinates are detected
 *     on the device and reported by subm3d_map_status().
 *   - Every function is safe to call from several host threads on different
 *     streams; calls that share a workspace must be ordered by the caller.
 *   - Stream order is enough: a call on a map may be enqueued right behind its
 *     build, and a build may reuse the nbr buffer and workspace of maps whose
 *     calls are enqueued before it on the same stream (those calls see their
 *     own map).  The kernels use programmatic dependent launch, read what an
 *     earlier kernel wrote only after griddepcontrol.wait, and never through
 *     the non-coherent load path.
 */
#ifndef SUBM3D_H_
#define SUBM3D_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbol visibility: the library is built with hidden visibility and exports
 * exactly the functions declared here. */
#if defined(__GNUC__)
#define SUBM3D_API __attribute__((visibility("default")))
#else
#define SUBM3D_API
#endif

#define SUBM3D_ABI_VERSION 1
/* Number of kernel offsets, 3x3x3. */
#define SUBM3D_KVOL 27
/* Rows covered by one word of the per-tile offset mask. */
#define SUBM3D_TILE_ROWS 128

typedef enum {
  SUBM3D_OK = 0,
  SUBM3D_E_INVALID = 1,     /* null pointer, negative size, too-small workspace, bad enum  */
  SUBM3D_E_RANGE = 2,       /* a coordinate lies outside [0,batch) x [0,grid_dim)^3        */
  SUBM3D_E_DUPLICATE = 3,   /* a coordinate occurs more than once                          */
  SUBM3D_E_TABLE_FULL = 4,  /* the hash table ran out of slots (only with a forced size)   */
  SUBM3D_E_UNSUPPORTED = 5, /* shape, alignment or device the kernels do not handle        */
  SUBM3D_E_CUDA = 6,        /* a CUDA runtime call failed (launch, copy, synchronize)     */
  SUBM3D_E_TIMEOUT = 7      /* a bounded device-side wait ran out; the result is invalid   */
} subm3d_status;

typedef enum { SUBM3D_F32 = 0, SUBM3D_BF16 = 1 } subm3d_dtype;
typedef enum { SUBM3D_ACT_NONE = 0, SUBM3D_ACT_GELU = 1, SUBM3D_ACT_SILU = 2 } subm3d_act;

/* Opaque handle of a built neighbour map (host memory; see subm3d_build_map). */
typedef struct subm3d_map subm3d_map;

/* ABI version of the loaded library (SUBM3D_ABI_VERSION at build time). */
SUBM3D_API int32_t subm3d_abi_version(void);

/* Static, human-readable name of a status code (never NULL). */
SUBM3D_API const char* subm3d_status_string(int32_t status);

/*
 * Workspace bytes subm3d_build_map() needs for N voxels in a batch x
 * grid_dim^3 volume: a status word, one 32-bit offset mask per 128-row tile,
 * and the lookup table -- with budget = max(64 MB, 256 bytes x N):
 *   a direct-address table of batch * (grid_dim + 2)^3 int32 cells (each grid
 *   with a one-cell border) when that fits the budget and 2^28 cells and is at
 *   most 64 MB or 16 cells per voxel;
 *   else a brick table when its directory fits the budget: one int32 per brick
 *   of 8 (x) x 4 (y) x 2 (z) bordered cells, then min(N, bricks) blocks of 64
 *   int32 cells (at most 256 bytes per voxel; only occupied bricks' blocks are
 *   written);
 *   else an open-addressing hash table of at least 2N slots (8 bytes each, 12
 *   with batch > 4 or grid_dim > 1024) --
 * and for N < 2^29 the x-run layout of subm3d_forward_map(): run-start counts
 * (an int32 per 128-row tile and per 128 tiles), a header, a position table of
 * 3N int32 (rounded up) and an E index table of 9 lines of as many int32
 * (~120 bytes per voxel).
 * Host-only, no CUDA
 * call.  Returns 0 for arguments subm3d_build_map() would
 * reject (N < 0, grid_dim < 1 or > 65535, batch < 1 or > 65535).
 */
SUBM3D_API size_t subm3d_map_workspace_bytes(int64_t n, int32_t grid_dim, int32_t batch);

/*
 * Build the neighbour map of a coordinate set ("sorted-key indice map, 27
 * lookups/voxel", lato.2_mrp_mlx commit 97dcdfb54a; here a direct-address,
 * brick or hash table on the GPU, see subm3d_map_workspace_bytes()).
 *
 *   coords     (device) int32 [N, 4] rows (b, z, y, x), 16-byte aligned, any row order.
 *   n          N >= 0; N < 2^31 - 1.
 *   grid_dim   cubic extent; valid coordinates are 0 <= z, y, x < grid_dim (<= 65535).
 *   batch      valid batch indices are 0 <= b < batch (<= 65535).
 *   nbr        (device) int32 [N, 27] output, 16-byte aligned: row of the voxel at
 *              p_i + d_k or -1 when it is absent or outside the grid.  Voxels of
 *              different batch indices are never neighbours.
 *   workspace  (device) >= subm3d_map_workspace_bytes(n, grid_dim, batch) bytes,
 *              256-byte aligned.  Its head holds the tile masks the forward reads,
 *              so it must stay alive, unmodified, as long as the handle is used.
 *   stream     stream the build is enqueued on.
 *   out_map    (host) receives a new handle; release it with subm3d_map_destroy().
 *
 * The map is bit-identical to the plain definition for every valid input and
 * does not depend on the table kind or its layout.  Coordinates outside the volume or
 * repeated are reported by subm3d_map_status(); until it returns SUBM3D_OK the
 * contents of nbr are unspecified.  Besides nbr and the tile masks the build
 * writes, for N < 2^29, the x-run position layout that subm3d_forward_map()
 * uses.  Enqueues 3 kernels (4 with the brick table); no allocation.
 * N < 2^31 - 256.
 * Testing knobs, read from the environment by this function and by
 * subm3d_map_workspace_bytes() alike: SUBM3D_MAP_KIND=direct|brick|hash
 * selects that table wherever it fits the budget (the hash table always
 * does); SUBM3D_TABLE_CAPACITY=<slots> caps
 * the hash table (and selects it) so that SUBM3D_E_TABLE_FULL can be
 * exercised -- probe loops stop after `capacity` steps instead of spinning.
 */
SUBM3D_API subm3d_status subm3d_build_map(const int32_t* coords, int64_t n, int32_t grid_dim,
                               int32_t batch, int32_t* nbr, void* workspace,
                               size_t workspace_bytes, void* stream, subm3d_map** out_map);

/*
 * Synchronizes the map's stream and returns the device-detected status of the
 * build: SUBM3D_OK, SUBM3D_E_RANGE, SUBM3D_E_DUPLICATE or SUBM3D_E_TABLE_FULL
 * (first in that order of precedence), or SUBM3D_E_CUDA.  Blocking.
 */
SUBM3D_API subm3d_status subm3d_map_status(const subm3d_map* map);

/* Accessors (host, no CUDA call).  The pointers are the caller's buffers. */
SUBM3D_API const int32_t* subm3d_map_nbr(const subm3d_map* map);        /* (device) [N, 27]          */
SUBM3D_API const uint32_t* subm3d_map_tile_mask(const subm3d_map* map); /* (device) [ceil(N/128)]    */
SUBM3D_API int64_t subm3d_map_size(const subm3d_map* map);              /* N                         */

/* The lookup table the build chose (see subm3d_map_workspace_bytes()); the
 * build enqueues 4 kernels with the brick table, 3 otherwise.  -1 for NULL. */
typedef enum { SUBM3D_TABLE_DIRECT = 0, SUBM3D_TABLE_HASH = 1, SUBM3D_TABLE_BRICK = 2 } subm3d_table;
SUBM3D_API int32_t subm3d_map_table(const subm3d_map* map);

/* Frees the host handle only; the caller's nbr and workspace are untouched. */
SUBM3D_API void subm3d_map_destroy(subm3d_map* map);

/*
 * Forward of one SubMConv3d layer over a built map (implicit gather-GEMM: the
 * rows nbr[i][k] of feats are gathered tile by tile into shared memory and
 * contracted against the weight slices; no scatter, no atomics, no [N,27,Cin]
 * buffer).  out[i] = act( sum_k Wf[:, k, :] . feats[nbr[i][k]] ), with
 * Wf[:, k] = W[:, k] (flip = 0, correlation) or W[:, 26-k] (flip != 0).
 *
 *   nbr        (device) int32 [N, 27] as written by subm3d_build_map().
 *   tile_mask  (device) uint32 [ceil(N/128)]: bit k of word t is set when some row
 *              of rows [128t, 128t+128) has nbr[.][k] != -1 (subm3d_map_tile_mask()).
 *              NULL means every offset of every tile is visited.
 *   n          N >= 0.  N = 0 enqueues nothing.
 *   feats      (device) [N, Cin] row-major.
 *   weight     (device) KRSC [Cout, 3, 3, 3, Cin] row-major.
 *   out        (device) [N, Cout] row-major; must not overlap feats (E_INVALID).
 *              feats, weight, out and nbr are 16-byte aligned for bf16 (else
 *              SUBM3D_E_UNSUPPORTED), 4-byte aligned for fp32 (else E_INVALID).
 *   dtype      SUBM3D_BF16: bf16 feats/weight/out, fp32 accumulation on the tensor
 *              cores, Cin and Cout multiples of 16 (else SUBM3D_E_UNSUPPORTED).
 *              SUBM3D_F32: fp32 throughout on CUDA-core FMA, any Cin, Cout >= 1.
 *   act        SUBM3D_ACT_NONE, SUBM3D_ACT_GELU (erf form, v * Phi(v); erfc from
 *              Abramowitz & Stegun 7.1.26, absolute error <= 1.5e-7) or
 *              SUBM3D_ACT_SILU (v * sigmoid(v)) on the fp32 sum; a bf16 output is
 *              rounded once, after the activation.
 *
 * The forward never fails on data.  SUBM3D_E_UNSUPPORTED is also returned when
 * the current device is not sm_100.  A bounded device-side wait that runs out
 * is reported by the next subm3d_device_status().
 */
SUBM3D_API subm3d_status subm3d_forward(const int32_t* nbr, const uint32_t* tile_mask, int64_t n,
                             const void* feats, const void* weight, void* out,
                             int32_t cin, int32_t cout, subm3d_dtype dtype, int32_t flip,
                             subm3d_act act, void* stream);

/*
 * Largest N subm3d_build_map_noalloc() accepts.  Its fixed scratch array holds a
 * hash table for this many voxels: about 12 MB of device memory.
 */
#define SUBM3D_NOALLOC_MAX_VOXELS 524288

/*
 * Allocation-free map build.  The paper has no counterpart to this entry point;
 * it exists for callers that cannot allocate device memory when they build a
 * map -- a plugin inside a host framework that owns and accounts for every
 * device allocation, or a serving loop that must never call cudaMalloc or
 * cudaFree once running, since those calls synchronise the device and cost
 * hundreds of microseconds.  It builds the same map as subm3d_build_map()
 * (always with the hash table) but takes no workspace: its scratch (status word
 * and hash table) is a fixed device array inside the library, about 12 MB,
 * which exists on every GPU the process loads the library on, until exit.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 *   coords     (device) int32 [N, 4] (b, z, y, x), 16-byte aligned.
 *   n          0 <= N <= SUBM3D_NOALLOC_MAX_VOXELS; a larger N returns
 *              SUBM3D_E_UNSUPPORTED before anything is enqueued.
 *   grid_dim, batch   as for subm3d_build_map().
 *   nbr        (device) int32 [N, 27] output, 16-byte aligned.
 *   tile_mask  (device) uint32 [ceil(N/128)] output, the per-tile offset masks
 *              that subm3d_forward() takes.
 *   stream     stream the work is enqueued on.
 *
 * Blocking: enqueues the build and a copy of the masks out of the scratch,
 * synchronizes `stream`, and returns the build's status (SUBM3D_OK,
 * SUBM3D_E_RANGE, SUBM3D_E_DUPLICATE, SUBM3D_E_TABLE_FULL) or an argument or
 * CUDA error.  The first call on each device looks up the scratch array's
 * device address (cudaGetSymbolAddress); make that first call before any
 * stream capture.  Every call uses the same scratch array and starts by
 * clearing it, so calls whose work overlaps on the GPU (unordered streams,
 * several host threads) race and must be serialized by the caller.
 */
SUBM3D_API subm3d_status subm3d_build_map_noalloc(const int32_t* coords, int64_t n,
                                                  int32_t grid_dim, int32_t batch, int32_t* nbr,
                                                  uint32_t* tile_mask, void* stream);

/*
 * Forward of one layer over a built map -- the same op and arguments as
 * subm3d_forward(), with N, nbr and the masks taken from the map.  For bf16
 * with Cin >= 48 (and a map of N < 2^29) it runs the x-run kernel (Cin in
 * 64-channel chunks, the last one zero-padded when Cin is not a multiple of 64),
 * which uses the map's position layout: voxels on a line of positions in row
 * order, two pad positions before every run of x-adjacent voxels, tiles of
 * 256 positions, and per tile and (dz, dy) one gathered tile of feature rows
 * whose rows p-1, p, p+1 are the dx = -1, 0, +1 neighbours of the voxel at
 * position p; the three offsets of a (dz, dy) pair share that tile through
 * row-shifted tensor-core operands, so ~3x fewer feature rows are gathered.
 * Other shapes and fp32 run subm3d_forward().  Errors as subm3d_forward().
 * Testing knobs, read at every call: SUBM3D_FORWARD_KERNEL=gather takes the
 * per-offset kernel of subm3d_forward() even where the x-run kernel applies;
 * SUBM3D_WAIT_LIMIT_NS=<ns> cuts the limit of every bounded device wait of the
 * tensor-core kernels (default 2 s) so that the timeout path can be tested.
 */
SUBM3D_API subm3d_status subm3d_forward_map(const subm3d_map* map, const void* feats,
                                            const void* weight, void* out, int32_t cin,
                                            int32_t cout, subm3d_dtype dtype, int32_t flip,
                                            subm3d_act act, void* stream);

/*
 * One layer with the epilogue of a sparse residual block fused into its store:
 *
 *   out[i] = act( sum_k Wf[:, k, :] . feats[nbr[i][k]] + bias ) + residual[i]
 *
 * -- the first convolution of a block takes a bias and an activation, the
 * second a bias and the block's skip input as residual, both on one map.  The
 * pages define the convolution only; this epilogue is the plain reading of
 * "conv + bias, activation, skip add" for the decoders' residual blocks.
 *
 *   bias      (device) [Cout] in the feature dtype, or NULL.  Added to the fp32
 *             sum before the activation.  2-byte aligned (bf16) / 4 (fp32).
 *   residual  (device) [N, Cout] in the feature dtype, or NULL.  Added after the
 *             activation, before the single rounding of a bf16 output.  It may
 *             be `out` itself (an in-place skip add) or overlap feats; a partial
 *             overlap with out is SUBM3D_E_INVALID.  16-byte aligned (bf16,
 *             else SUBM3D_E_UNSUPPORTED) / 4-byte (fp32, else E_INVALID).
 *
 * Everything else -- arguments, kernels chosen, errors -- as subm3d_forward_map().
 */
SUBM3D_API subm3d_status subm3d_forward_fused(const subm3d_map* map, const void* feats,
                                              const void* weight, const void* bias,
                                              const void* residual, void* out, int32_t cin,
                                              int32_t cout, subm3d_dtype dtype, int32_t flip,
                                              subm3d_act act, void* stream);

/*
 * Backward of one layer (the convolution itself: no bias, activation or
 * residual) over a built map.  The pages port inference only; this is the
 * plain gradient of the forward's definition.
 *
 * subm3d_backward_data: dx[j] = sum over (i, k) with nbr[i][k] = j of
 * Wf[:, k, :]^T dy[i].  By the map's symmetry (nbr[i][k] = j <=> nbr[j][26-k]
 * = i) that is the forward of dy with the transposed weight W^T[c][k][o] =
 * W[o][k][c] and the opposite flip, so it writes W^T and runs the forward
 * kernels (tensor cores for bf16: Cout and Cin multiples of 16).
 *
 *   dy        (device) [N, Cout] in the dtype; 16-byte aligned for bf16.
 *   weight    (device) KRSC [Cout, 3, 3, 3, Cin], as given to the forward.
 *   weight_t  (device) caller scratch of Cout * 27 * Cin elements, 16-byte
 *             aligned, not overlapping weight: receives W^T [Cin, 27, Cout].
 *   dx        (device) [N, Cin] output; must not overlap dy.
 *   flip      the forward's orientation.
 *
 * subm3d_backward_weight: dW[o][kw][c] = sum_i dy[i][o] * feats[nbr[i][k]][c]
 * over nbr[i][k] != -1, kw = k (flip = 0) or 26 - k.  dweight is fp32 KRSC
 * [Cout, 3, 3, 3, Cin] (device, 4-byte aligned, overwritten; fp32 for both
 * dtypes: the sum runs over all voxels).  bf16 (with the map's x-run layout)
 * runs on the tensor cores over that layout (the sum over positions as
 * the MMA K dimension, one gathered tile per (dz, dy) pair for all three dx);
 * fp32, and maps without that layout, on CUDA-core FMA.  Partial sums over voxel ranges are
 * added with fp32 atomics, so the summation order (and the last bits) vary
 * from call to call.
 *
 * Errors: SUBM3D_E_INVALID for bad arguments or overlapping buffers; otherwise
 * as subm3d_forward().  Both are asynchronous on `stream`.
 */
SUBM3D_API subm3d_status subm3d_backward_data(const subm3d_map* map, const void* dy,
                                              const void* weight, void* weight_t, void* dx,
                                              int32_t cin, int32_t cout, subm3d_dtype dtype,
                                              int32_t flip, void* stream);
SUBM3D_API subm3d_status subm3d_backward_weight(const subm3d_map* map, const void* feats,
                                                const void* dy, float* dweight, int32_t cin,
                                                int32_t cout, subm3d_dtype dtype, int32_t flip,
                                                void* stream);

/*
 * Resolution changes, factor 2 (trellis_sparse_mrp_mlx commit log; lato.2_mrp_mlx
 * notes "Key facts").  Child slot s of a parent at (b, z, y, x) lies at
 * (b, 2z + dz, 2y + dy, 2x + dx).
 *
 *   SUBM3D_EXPAND_SUBDIVIDE       every voxel emits its 8 children in C order
 *                                 (s = 4 dz + 2 dy + dx), features replicated;
 *                                 mask must be NULL.
 *   SUBM3D_EXPAND_UPSAMPLE        voxel i emits child s only where mask[i*8 + s]
 *                                 != 0; s decodes axis 0 fastest (dz = s % 2,
 *                                 dy = s / 2 % 2, dx = s / 4 % 2); features
 *                                 replicated; mask required.
 *   SUBM3D_EXPAND_CHANNEL2SPATIAL as UPSAMPLE (mask optional: NULL = all 8), child
 *                                 s takes channels [s C, (s + 1) C) of the
 *                                 parent's 8 C (C = channels_out).
 *
 * subm3d_expand: coords (device) int32 [N, 4], 16-byte aligned; feats (device)
 * [N, Cin] in dtype (Cin = channels_out, or 8 channels_out for
 * channel2spatial); mask (device) uint8 [N, 8] or NULL.  out_coords [8N, 4]
 * and out_feats [8N, channels_out] (device) receive the children parent-major,
 * by ascending s; *out_count (host) = the number written.  workspace (device)
 * >= subm3d_expand_workspace_bytes(N), 256-byte aligned.  With a mask the call
 * reads the child count back and is blocking; without one it is asynchronous.
 * N < 2^28.
 */
typedef enum {
  SUBM3D_EXPAND_SUBDIVIDE = 0,
  SUBM3D_EXPAND_UPSAMPLE = 1,
  SUBM3D_EXPAND_CHANNEL2SPATIAL = 2
} subm3d_expand_mode;
SUBM3D_API size_t subm3d_expand_workspace_bytes(int64_t n);
SUBM3D_API subm3d_status subm3d_expand(const int32_t* coords, const void* feats,
                                       const uint8_t* mask, int64_t n, int32_t channels_out,
                                       subm3d_dtype dtype, subm3d_expand_mode mode,
                                       int32_t* out_coords, void* out_feats, void* workspace,
                                       size_t workspace_bytes, int64_t* out_count, void* stream);

/*
 * Pooling to parents coord // 2, listed in raster order of (b, z, y, x):
 *
 *   SUBM3D_POOL_MAX / SUBM3D_POOL_MEAN  the element-wise max or mean over the
 *                              children present (mean: an fp32 sum in child slot
 *                              order, then one rounding); out_feats [P, C].
 *   SUBM3D_POOL_SPATIAL2CHANNEL  child s's features in channels [s C, (s+1) C) of
 *                              its parent, s = (z % 2) + 2 (y % 2) + 4 (x % 2),
 *                              zeros where the child is absent; out_feats [P, 8 C].
 *
 * fine: the map built on `coords` (its table finds the children).  coords,
 * feats [N, C] (device) are that set and its features; out_coords [N, 4] and
 * out_feats (device) must have room for P <= N parents.  workspace >=
 * subm3d_pool_workspace_bytes(N, grid_dim, batch) (a flag per parent cell of
 * batch x ceil(grid_dim/2)^3; 0 = unsupported above 2^30 cells), 256-byte
 * aligned.  Blocking: *out_count (host) = P is read back.
 */
typedef enum {
  SUBM3D_POOL_MAX = 0,
  SUBM3D_POOL_MEAN = 1,
  SUBM3D_POOL_SPATIAL2CHANNEL = 2
} subm3d_pool_mode;
SUBM3D_API size_t subm3d_pool_workspace_bytes(int64_t n, int32_t grid_dim, int32_t batch);
SUBM3D_API subm3d_status subm3d_pool(const subm3d_map* fine, const int32_t* coords,
                                     const void* feats, int32_t channels, subm3d_dtype dtype,
                                     subm3d_pool_mode mode, int32_t* out_coords, void* out_feats,
                                     void* workspace, size_t workspace_bytes, int64_t* out_count,
                                     void* stream);

/*
 * Device pointers into the map's x-run layout, for tests and tools: the
 * position table (int32, one entry per position: row * 4 + tag, tag 0 voxel,
 * 1 left pad of that row's voxel, 2 right pad, -1 empty), the E index table
 * (int32, 9 lines, one per offset pair dz-dy = 3 (dz+1) + (dy+1), `stride`
 * entries apart: entry q + 1 of a line is the feature row gathered as E row
 * q, i.e. at position q, for q = -1 .. 256 tiles, or -1) and a 4-int header
 * [runs, tiles, positions, stride].
 * Valid once the build has completed on its stream.  Host-only.
 * SUBM3D_E_UNSUPPORTED when the map has no run layout (N >= 2^29).
 */
SUBM3D_API subm3d_status subm3d_map_run_layout(const subm3d_map* map, const int32_t** pos,
                                               const int32_t** etable, const int32_t** header);

/*
 * Synchronizes `stream`, then reads and clears the library's device error word
 * of the current device: SUBM3D_E_TIMEOUT if a tensor-core kernel (forward,
 * input or weight gradient) gave up a bounded wait since the last call, else
 * SUBM3D_OK (or SUBM3D_E_CUDA).  A kernel whose wait ran out has waited for
 * the copies and MMAs it had issued and released its tensor memory before
 * exiting, so later calls run normally; its own output is invalid.
 * Blocking.
 */
SUBM3D_API subm3d_status subm3d_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SUBM3D_H_ */

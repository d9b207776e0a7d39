"""User-facing API: SparseTensor, SubMConv3d with an indice_key map cache.

The sparse-voxel generators the pages port (LATO.2, Pixal3D, the TRELLIS.2
family) hold a SparseTensor (coordinates + features) and run SparseConv3d
layers that are all submanifold 3x3x3 convolutions; the neighbour map is
cached per coordinate set "the way spconv uses indice_key" (lato.2_mrp_mlx,
commit 97dcdfb54a message).  torch provides device memory and streams only:
every step of the op runs in libsubm3d.so's kernels.
"""
from __future__ import annotations

import math

import torch

from . import _abi
from ._abi import Subm3dError

__all__ = ["MapHandle", "build_map", "forward", "backward_data", "backward_weight", "SparseTensor",
           "SubMConv3d", "SubMResBlock3d", "Subm3dError", "subdivide", "upsample",
           "channel2spatial", "spatial2channel", "downsample"]

MapHandle = _abi.MapHandle

_DTYPES = {torch.float32: _abi.SUBM3D_F32, torch.bfloat16: _abi.SUBM3D_BF16}
_ACTS = {None: _abi.SUBM3D_ACT_NONE, "none": _abi.SUBM3D_ACT_NONE, "gelu": _abi.SUBM3D_ACT_GELU,
         "silu": _abi.SUBM3D_ACT_SILU}


def _cuda_contig(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.contiguous()


def _new(t, orig):
    """t when this binding made it (an allocation or a contiguous copy), else None."""
    return None if t is orig else t


def _on_side_stream(stream, *made) -> None:
    """Before a call enqueued on `stream` when that is not torch's current stream.

    This binding allocates outputs and scratch, and makes contiguous copies, on
    the current stream; the caching allocator hands out memory that is free in
    that stream's order only.  So the side stream first waits for the work
    already queued on the current stream, and the tensors made here are
    recorded as in use by the side stream (their memory is not handed out again
    before its work has run).  `made`: only tensors created here (None skipped);
    the caller's own tensors are the caller's to manage."""
    if stream is None:
        return
    side = (stream if isinstance(stream, torch.cuda.Stream)
            else torch.cuda.ExternalStream(int(stream)))
    current = torch.cuda.current_stream()
    if side.cuda_stream == current.cuda_stream:
        return
    side.wait_stream(current)
    for t in made:
        if t is not None:
            t.record_stream(side)


def build_map(coords: torch.Tensor, grid_dim: int, batch: int = 1, stream=None,
              check: bool = True, nbr: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None) -> MapHandle:
    """Neighbour map of a coordinate set: int32 [N, 27] plus per-tile offset masks.

    coords: int32 [N, 4] (b, z, y, x) on the GPU.  With check=True the call
    waits for the build and raises Subm3dError on out-of-range or duplicate
    coordinates; with check=False it stays asynchronous (call .status later).
    nbr / workspace may be passed in to reuse memory.
    """
    coords_in, nbr_in, workspace_in = coords, nbr, workspace
    coords = _cuda_contig(coords, "coords", torch.int32)
    if coords.dim() != 2 or coords.shape[1] != 4:
        raise ValueError("coords must have shape [N, 4]")
    n = coords.shape[0]
    ws_bytes = _abi.subm3d_map_workspace_bytes(n, grid_dim, batch)
    if ws_bytes == 0:
        raise Subm3dError(_abi.SUBM3D_E_UNSUPPORTED, "subm3d_map_workspace_bytes")
    dev = coords.device
    if nbr is None:
        nbr = torch.empty((n, 27), dtype=torch.int32, device=dev)
    if workspace is None or workspace.numel() * workspace.element_size() < ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    _on_side_stream(stream, _new(coords, coords_in), _new(nbr, nbr_in),
                    _new(workspace, workspace_in))
    h = _abi.subm3d_build_map(coords, n, grid_dim, batch, nbr, workspace, ws_bytes, stream)
    h.coords = coords
    if check:
        st = _abi.subm3d_map_status(h)
        if st != _abi.SUBM3D_OK:
            raise Subm3dError(st, "subm3d_build_map")
    return h


def map_status(h: MapHandle) -> int:
    return _abi.subm3d_map_status(h)


def tile_mask_tensor(h: MapHandle) -> torch.Tensor:
    """The map's per-128-row-tile offset masks as an int32 view of its workspace."""
    off = _abi.subm3d_map_tile_mask(h) - h.workspace.data_ptr()
    n_tiles = (h.n + _abi.SUBM3D_TILE_ROWS - 1) // _abi.SUBM3D_TILE_ROWS
    return h.workspace[off:off + 4 * n_tiles].view(torch.int32)


def forward(h: MapHandle, feats: torch.Tensor, weight: torch.Tensor, flip: bool = False,
            act: str | None = None, out: torch.Tensor | None = None, stream=None,
            use_tile_mask: bool = True, kernel: str = "auto", bias: torch.Tensor | None = None,
            residual: torch.Tensor | None = None) -> torch.Tensor:
    """One SubMConv3d layer: out[i] = act(sum_k Wf[:,k,:] . feats[nbr[i,k]] + bias) + residual[i].

    feats: [N, Cin] float32 or bfloat16; weight: KRSC [Cout, 3, 3, 3, Cin] (or
    [Cout, 27, Cin]) of the same dtype.  Returns [N, Cout] of that dtype.
    act: None, "gelu" (exact erf form) or "silu".  bias: optional [Cout];
    residual: optional [N, Cout] (may be `out`), both of the feature dtype.
    kernel: "auto" runs subm3d_forward_fused (the x-run kernel for bf16 with
    Cin >= 48); "gather" runs subm3d_forward on nbr and the tile masks
    (use_tile_mask=False: no masks; no bias or residual there).
    """
    if feats.dtype not in _DTYPES:
        raise ValueError(f"unsupported feature dtype {feats.dtype}")
    given = (feats, weight, bias, residual, out)
    feats = _cuda_contig(feats, "feats")
    weight = _cuda_contig(weight, "weight", feats.dtype)
    n, cin = feats.shape
    if n != h.n:
        raise ValueError(f"feats has {n} rows but the map has {h.n}")
    cout = weight.shape[0]
    if weight.numel() != cout * 27 * cin:
        raise ValueError("weight must be KRSC [Cout, 3, 3, 3, Cin]")
    if bias is not None:
        bias = _cuda_contig(bias, "bias", feats.dtype)
        if bias.numel() != cout:
            raise ValueError("bias must have Cout elements")
    if residual is not None:
        residual = _cuda_contig(residual, "residual", feats.dtype)
        if tuple(residual.shape) != (n, cout):
            raise ValueError("residual must have shape [N, Cout]")
    if out is None:
        out = torch.empty((n, cout), dtype=feats.dtype, device=feats.device)
    _on_side_stream(stream, *(_new(t, g) for t, g in zip((feats, weight, bias, residual, out),
                                                          given)))
    if kernel == "auto" and use_tile_mask:
        _abi.subm3d_forward_fused(h, feats, weight, bias, residual, out, cin, cout,
                                  _DTYPES[feats.dtype], flip, _ACTS[act], stream)
        return out
    if kernel not in ("auto", "gather"):
        raise ValueError(f"unknown kernel {kernel!r}")
    if bias is not None or residual is not None:
        raise ValueError("bias and residual need kernel='auto'")
    mask_ptr = _abi.subm3d_map_tile_mask(h) if use_tile_mask else None
    _abi.subm3d_forward(h.nbr, mask_ptr, n, feats, weight, out, cin, cout, _DTYPES[feats.dtype],
                        flip, _ACTS[act], stream)
    return out


def backward_data(h: MapHandle, dy: torch.Tensor, weight: torch.Tensor, flip: bool = False,
                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Input gradient of the convolution: dx[j] = sum over nbr[i,k] = j of
    Wf[:,k,:]^T dy[i] -- the forward of dy with the transposed weight and the
    opposite orientation.  dy: [N, Cout]; returns [N, Cin] in dy's dtype."""
    if dy.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {dy.dtype}")
    given = (dy, weight, out)
    dy = _cuda_contig(dy, "dy")
    weight = _cuda_contig(weight, "weight", dy.dtype)
    n, cout = dy.shape
    if n != h.n or weight.shape[0] != cout:
        raise ValueError("dy must be [N, Cout] for this map and weight")
    cin = weight.numel() // (27 * cout)
    weight_t = torch.empty(weight.numel(), dtype=dy.dtype, device=dy.device)
    if out is None:
        out = torch.empty((n, cin), dtype=dy.dtype, device=dy.device)
    _on_side_stream(stream, weight_t, *(_new(t, g) for t, g in zip((dy, weight, out), given)))
    _abi.subm3d_backward_data(h, dy, weight, weight_t, out, cin, cout, _DTYPES[dy.dtype], flip,
                              stream)
    return out


def backward_weight(h: MapHandle, feats: torch.Tensor, dy: torch.Tensor, flip: bool = False,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Weight gradient: dW[o,kw,c] = sum_i dy[i,o] feats[nbr[i,k],c] (kw = k, or
    26 - k under flip), fp32 KRSC [Cout, 3, 3, 3, Cin] for either dtype."""
    if feats.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {feats.dtype}")
    given = (feats, dy, out)
    feats = _cuda_contig(feats, "feats")
    dy = _cuda_contig(dy, "dy", feats.dtype)
    n, cin = feats.shape
    cout = dy.shape[1]
    if n != h.n or dy.shape[0] != n:
        raise ValueError("feats and dy must have the map's N rows")
    if out is None:
        out = torch.empty((cout, 3, 3, 3, cin), dtype=torch.float32, device=feats.device)
    _on_side_stream(stream, *(_new(t, g) for t, g in zip((feats, dy, out), given)))
    _abi.subm3d_backward_weight(h, feats, dy, out, cin, cout, _DTYPES[feats.dtype], flip, stream)
    return out


class _SubMConvFunction(torch.autograd.Function):
    """out = conv(feats, weight) on a built map, differentiable in feats and
    weight through the library's backward kernels."""

    @staticmethod
    def forward(ctx, feats, weight, h, flip):
        ctx.save_for_backward(feats, weight)
        ctx.h, ctx.flip = h, flip
        return forward(h, feats, weight, flip=flip)

    @staticmethod
    def backward(ctx, grad_out):
        feats, weight = ctx.saved_tensors
        grad_out = grad_out.contiguous()
        dx = dw = None
        if ctx.needs_input_grad[0]:
            dx = backward_data(ctx.h, grad_out, weight, flip=ctx.flip)
        if ctx.needs_input_grad[1]:
            dw = backward_weight(ctx.h, feats, grad_out, flip=ctx.flip).to(weight.dtype)
            dw = dw.reshape(weight.shape)
        return dx, dw, None, None


def run_layout_tensors(h: MapHandle):
    """(position table [256 tiles], E index table [9, 256 tiles + 2], header) as
    int32 views of the map's workspace; call after the build has completed.
    Row dz-dy of the E table holds, at column q + 1, the feature row gathered
    as E row q (position q) for the offset pair (dz, dy), q = -1 .. 256 tiles."""
    pos_p, et_p, hdr_p = _abi.subm3d_map_run_layout(h)
    base = h.workspace.data_ptr()
    ws = h.workspace
    hdr = ws[hdr_p - base:hdr_p - base + 16].view(torch.int32)
    tiles, stride = int(hdr[1].item()), int(hdr[3].item())
    pos = ws[pos_p - base:pos_p - base + 4 * 256 * tiles].view(torch.int32)
    lines = ws[et_p - base:et_p - base + 4 * 9 * stride].view(torch.int32).view(9, stride)
    return pos, lines[:, :256 * tiles + 2], hdr


class SparseTensor:
    """Voxel coordinates int32 [N, 4] (b, z, y, x) + features [N, C] on one GPU,
    with the cache of neighbour maps built on this coordinate set."""

    def __init__(self, coords: torch.Tensor, feats: torch.Tensor, grid_dim: int,
                 batch: int = 1, cache: dict | None = None):
        if coords.shape[0] != feats.shape[0]:
            raise ValueError("coords and feats must have the same number of rows")
        self.coords = coords
        self.feats = feats
        self.grid_dim = int(grid_dim)
        self.batch = int(batch)
        self.cache = {} if cache is None else cache

    def replace(self, feats: torch.Tensor) -> "SparseTensor":
        """Same coordinate set (and map cache), new features."""
        return SparseTensor(self.coords, feats, self.grid_dim, self.batch, self.cache)

    def get_map(self, indice_key: str) -> MapHandle:
        h = self.cache.get(indice_key)
        if h is None:
            h = build_map(self.coords, self.grid_dim, self.batch)
            self.cache[indice_key] = h
        elif h.n != self.coords.shape[0]:
            raise Subm3dError(_abi.SUBM3D_E_INVALID, f"cached map {indice_key!r} size mismatch")
        return h


class SubMConv3d(torch.nn.Module):
    """Submanifold 3x3x3 convolution, stride 1, output sites = input sites.

    The weight is a KRSC parameter [Cout, 3, 3, 3, Cin].  Layers sharing an
    indice_key reuse one neighbour map per SparseTensor coordinate set.
    flip selects the mirrored kernel; act=None, "gelu" (exact erf form) or
    "silu".  bias=True adds a [Cout] bias before the activation (the pages'
    op has none; the residual blocks' convolutions do).
    """

    def __init__(self, in_channels: int, out_channels: int, indice_key: str = "subm0",
                 flip: bool = False, act: str | None = None, dtype=torch.bfloat16,
                 device=None, bias: bool = False):
        super().__init__()
        self.in_channels = in_channels
        self.out_channels = out_channels
        self.indice_key = indice_key
        self.flip = flip
        self.act = act
        w = torch.empty((out_channels, 3, 3, 3, in_channels), dtype=torch.float32)
        w.normal_(0.0, 1.0 / math.sqrt(27.0 * in_channels))
        self.weight = torch.nn.Parameter(w.to(dtype=dtype, device=device), requires_grad=False)
        if bias:
            b = torch.empty(out_channels, dtype=torch.float32).normal_(0.0, 0.1)
            self.bias = torch.nn.Parameter(b.to(dtype=dtype, device=device), requires_grad=False)
        else:
            self.bias = None

    def forward(self, x: SparseTensor, residual: torch.Tensor | None = None) -> SparseTensor:
        h = x.get_map(self.indice_key)
        wants_grad = torch.is_grad_enabled() and (self.weight.requires_grad or
                                                   x.feats.requires_grad)
        if wants_grad:
            if self.act is not None or self.bias is not None or residual is not None:
                raise NotImplementedError(
                    "gradients are implemented for the plain convolution (no act, bias, residual)")
            return x.replace(_SubMConvFunction.apply(x.feats, self.weight, h, self.flip))
        y = forward(h, x.feats, self.weight, flip=self.flip, act=self.act, bias=self.bias,
                    residual=residual)
        return x.replace(y)


class SubMResBlock3d(torch.nn.Module):
    """Two submanifold convolutions on one neighbour map with the residual
    block's epilogues fused into their stores:

        h   = act(conv1(x) + b1)
        out = conv2(h) + b2 + x

    Both convolutions share `indice_key`, so the map is built once per
    coordinate set; no separate bias, activation or add kernel runs.
    """

    def __init__(self, channels: int, indice_key: str = "subm0", act: str = "silu",
                 dtype=torch.bfloat16, device=None):
        super().__init__()
        self.conv1 = SubMConv3d(channels, channels, indice_key, act=act, dtype=dtype,
                                device=device, bias=True)
        self.conv2 = SubMConv3d(channels, channels, indice_key, act=None, dtype=dtype,
                                device=device, bias=True)

    def forward(self, x: SparseTensor) -> SparseTensor:
        return self.conv2(self.conv1(x), residual=x.feats)


# ------------------------------------------------------ resolution changes ----

def _expand(x: "SparseTensor", mask, mode: int, channels_out: int) -> "SparseTensor":
    coords = _cuda_contig(x.coords, "coords", torch.int32)
    feats = _cuda_contig(x.feats, "feats")
    if feats.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {feats.dtype}")
    n = coords.shape[0]
    if mask is not None:
        mask = _cuda_contig(mask, "mask")
        if mask.dtype != torch.uint8:
            mask = (mask != 0).to(torch.uint8)
        if tuple(mask.shape) != (n, 8):
            raise ValueError("mask must be [N, 8]")
    ws_bytes = max(_abi.subm3d_expand_workspace_bytes(n), 256)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=coords.device)
    out_c = torch.empty((8 * n, 4), dtype=torch.int32, device=coords.device)
    out_f = torch.empty((8 * n, channels_out), dtype=feats.dtype, device=coords.device)
    m = _abi.subm3d_expand(coords, feats, mask, n, channels_out, _DTYPES[feats.dtype], mode,
                           out_c, out_f, ws, ws_bytes)
    return SparseTensor(out_c[:m], out_f[:m], x.grid_dim * 2, x.batch)


def subdivide(x: "SparseTensor") -> "SparseTensor":
    """SparseSubdivide: every voxel -> its 8 children 2*coord + (dz, dy, dx) in C
    order (x fastest), features replicated; grid_dim doubles."""
    return _expand(x, None, _abi.SUBM3D_EXPAND_SUBDIVIDE, x.feats.shape[1])


def upsample(x: "SparseTensor", mask: torch.Tensor) -> "SparseTensor":
    """Masked upsample: voxel i emits child s where mask[i, s] != 0, the child
    index decoded axis 0 fastest (dz = s % 2, dy = s // 2 % 2, dx = s // 4 % 2);
    features replicated."""
    return _expand(x, mask, _abi.SUBM3D_EXPAND_UPSAMPLE, x.feats.shape[1])


def channel2spatial(x: "SparseTensor", mask: torch.Tensor | None = None) -> "SparseTensor":
    """Sparse depth-to-space: features [N, 8C] -> child s (axis 0 fastest) takes
    channels [sC, (s+1)C); all 8 children or the flagged ones."""
    c8 = x.feats.shape[1]
    if c8 % 8:
        raise ValueError("channel2spatial needs a multiple of 8 channels")
    return _expand(x, mask, _abi.SUBM3D_EXPAND_CHANNEL2SPATIAL, c8 // 8)


def _pool(x: "SparseTensor", mode: int, indice_key: str, channels_out: int) -> "SparseTensor":
    h = x.get_map(indice_key)
    coords = _cuda_contig(x.coords, "coords", torch.int32)
    feats = _cuda_contig(x.feats, "feats")
    n, c = feats.shape
    ws_bytes = _abi.subm3d_pool_workspace_bytes(n, x.grid_dim, x.batch)
    if ws_bytes == 0:
        raise Subm3dError(_abi.SUBM3D_E_UNSUPPORTED, "subm3d_pool_workspace_bytes")
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=coords.device)
    out_c = torch.empty((max(n, 1), 4), dtype=torch.int32, device=coords.device)
    out_f = torch.empty((max(n, 1), channels_out), dtype=feats.dtype, device=coords.device)
    p = _abi.subm3d_pool(h, coords, feats, c, _DTYPES[feats.dtype], mode, out_c, out_f, ws,
                         ws_bytes)
    return SparseTensor(out_c[:p], out_f[:p], (x.grid_dim + 1) // 2, x.batch)


def downsample(x: "SparseTensor", mode: str, indice_key: str = "subm0") -> "SparseTensor":
    """Parents coord // 2 in raster order with the max or the mean of their
    children's features.  The pages' models differ here (LATO.2: max, Pixal3D:
    mean by default), so the mode has no default.  Uses (or builds) the map of
    `indice_key` on x's coordinate set."""
    modes = {"max": _abi.SUBM3D_POOL_MAX, "mean": _abi.SUBM3D_POOL_MEAN}
    if mode not in modes:
        raise ValueError("mode must be 'max' or 'mean'")
    return _pool(x, modes[mode], indice_key, x.feats.shape[1])


def spatial2channel(x: "SparseTensor", indice_key: str = "subm0") -> "SparseTensor":
    """Sparse space-to-depth: parents coord // 2 (raster order), child s's
    features in channels [sC, (s+1)C), zeros for absent children."""
    return _pool(x, _abi.SUBM3D_POOL_SPATIAL2CHANNEL, indice_key, 8 * x.feats.shape[1])

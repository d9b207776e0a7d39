"""B200-native submanifold 3x3x3 sparse convolution (SubMConv3d).

The compute path lives in libsubm3d.so (C ABI in include/subm3d.h): a GPU
hash-table neighbour-map build and an implicit gather-GEMM forward on sm_100a
tcgen05 tensor cores (bf16, fp32 accumulation in TMEM), plus an fp32
CUDA-core path.  This package is the thin Python layer over it.  Importing
it loads the library and fails loudly if it is not built.
"""
from . import _abi
from ._abi import Subm3dError
from .sparse import MapHandle, SparseTensor, SubMConv3d, SubMResBlock3d, backward_data, \
    backward_weight, build_map, channel2spatial, downsample, forward, map_status, \
    run_layout_tensors, spatial2channel, subdivide, tile_mask_tensor, upsample

__all__ = ["Subm3dError", "MapHandle", "SparseTensor", "SubMConv3d", "SubMResBlock3d", "build_map",
           "forward", "backward_data", "backward_weight", "map_status", "run_layout_tensors",
           "tile_mask_tensor", "subdivide", "upsample", "channel2spatial", "spatial2channel",
           "downsample"]

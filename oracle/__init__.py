"""CPU oracle for the submanifold 3x3x3 sparse convolution (SubMConv3d).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
benchmark's CPU-baseline / reference leg may import, call, link or run
anything in this directory.  The product path (sparse_voxel_conv_b200/) never
does, and the oracle shares no code with it: no kernels, headers, helpers,
tables or pre/post-processing.  Both sides are fed by the seeded generators
in workloads.py, which hold none of the op's arithmetic.

Contents:
  subm3d_oracle.py   pure Python (dict + per-voxel, per-offset loop, fp64)
  subm3d_oracle.cpp  the same definition in C++ (std::map, OpenMP, fp64)
  cpp.py             ctypes wrapper that builds and loads the C++ oracle

Every function is pinned by tests/test_oracle.py against facts that do not
come from the oracle itself: an all-pairs brute-force map, a dense Conv3d on
fully occupied grids (submanifold equals dense there), an isolated voxel,
translation and permutation invariance, flip applied twice, linearity,
batch independence, one-hot probing of the orientation and a hand-derived
golden fixture.  Orientation relative to spconv itself is the one thing no
pin can reach (parity unpinned against spconv; the pages leave it open).
"""

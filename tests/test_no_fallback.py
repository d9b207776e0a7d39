"""The product path has no CPU fallback (CPU only): host tensors are refused
before any work, nothing in the package reaches the oracle, and a missing
shared library fails the import instead of degrading."""
import ast
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_voxel_conv_b200")


@pytest.fixture(scope="module")
def S():
    from sparse_voxel_conv_b200 import build
    build.build()
    import sparse_voxel_conv_b200 as S
    return S


def test_host_tensors_are_refused(S):
    coords = torch.zeros((4, 4), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        S.build_map(coords, 8, 1)
    x = S.SparseTensor(coords, torch.zeros((4, 16)), 8)
    conv = S.SubMConv3d(16, 16, indice_key="k")
    with pytest.raises(ValueError, match="CUDA"):
        conv(x)
    with pytest.raises(ValueError, match="CUDA"):
        S.subdivide(x)
    with pytest.raises(ValueError, match="CUDA"):
        S.downsample(x, "max")


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if not f.endswith(".py"):
                continue
            tree = ast.parse(open(os.path.join(dirpath, f)).read())
            for node in ast.walk(tree):
                if isinstance(node, ast.Import):
                    mods = [a.name for a in node.names]
                elif isinstance(node, ast.ImportFrom):
                    mods = [node.module or ""]
                else:
                    continue
                assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), (f, mods)


def test_missing_library_fails_the_import():
    code = (
        "import os, sys\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "real = os.path.exists\n"
        "os.path.exists = lambda p: False if str(p).endswith('libsubm3d.so') else real(p)\n"
        "try:\n"
        "    import sparse_voxel_conv_b200\n"
        "except ImportError as e:\n"
        "    print('ImportError', e)\n"
        "    sys.exit(0)\n"
        "sys.exit(3)\n")
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert p.returncode == 0, p.stdout + p.stderr
    assert "is not built" in p.stdout

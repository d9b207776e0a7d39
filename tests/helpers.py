"""Shared test helpers: tolerance checks and sampled-row selection."""
import numpy as np

# Per-element bar, relative to the reference's own scale:
#   |y - ref| <= rtol * (|ref| + rms(ref))
# rtol = 1e-5 for the fp32 path, 2e-2 for bf16 inputs with fp32 accumulation
# and a bf16 output.
RTOL_F32 = 1e-5
RTOL_BF16 = 2e-2


def assert_close(y, ref, rtol, what=""):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    if ref.size == 0:
        return
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(y - ref)
    bound = rtol * (np.abs(ref) + rms)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements beyond rtol={rtol}; worst at {i}: "
            f"y={y[i]!r} ref={ref[i]!r} (rms {rms:.3g}); max|y-ref|/max|ref| = "
            f"{float(err.max() / max(np.abs(ref).max(), 1e-300)):.3g}")


def sample_rows(n, k, seed=0):
    """k distinct rows: the first and last 128-row tiles (ragged tail) + random."""
    rng = np.random.default_rng(seed)
    edge = np.unique(np.concatenate([np.arange(min(n, 128)), np.arange(max(0, n - 200), n)]))
    rest = rng.choice(n, size=min(n, k), replace=False)
    return np.unique(np.concatenate([edge, rest])).astype(np.int64)


def masks_from_nbr(nbr, tile_rows=128):
    """Per-tile OR of the offsets with a neighbour, from a reference map."""
    n = nbr.shape[0]
    n_tiles = (n + tile_rows - 1) // tile_rows
    bits = (nbr >= 0).astype(np.int64) << np.arange(27, dtype=np.int64)
    per_row = np.bitwise_or.reduce(bits, axis=1) if n else np.zeros(0, np.int64)
    out = np.zeros(n_tiles, np.int64)
    for t in range(n_tiles):
        out[t] = np.bitwise_or.reduce(per_row[t * tile_rows:(t + 1) * tile_rows])
    return out

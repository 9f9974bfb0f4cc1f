"""E8 parity fixes that tie between coordinates, on the GPU (needs a B200).

When the chosen coset needs its parity fixed and several coordinates share
the largest |x - rint x| (integer coset) or the smallest (half-integer
coset), the Conway-Sloane rule moves the first of them.  Random data almost
never ties, so these tiles are built to: the rotated tile v = H (s . w) is
chosen first -- a background on a coarse grid that sets the tile's energy,
and one vector v[0:8] = t Delta with t a template of repeated quarter
integers -- and the input is w = s . (H v) / n, exact in binary32 (so the
encoder's transform gives back exactly v).  Delta comes from the oracle's
encode of the finished tile and is checked to be the one the template was
scaled by.  The fp32 stream is compared word for word with the oracle's.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from gpu_util import DEV, assert_streams_equal, fetch, gpu_encode

N, BPS, SEED = 256, 4.0, 11

# templates for x = v / Delta on one vector: repeated values tie when they
# carry the extreme |e| of a coset that needs its parity fixed
TEMPLATES = [
    [0.25, 0.25, 0, 0, 0, 0, 0, 1],
    [0.25] * 7 + [1],
    [1, 0.25, 0, 0.25, 0, 0, 0.25, 0],
    [-0.25, 0.25, 0, 0, 2, 0, 0, 1],
    [0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5, 1.5],
    [0.75, 0.75, 0.5, 0.5, 0.5, 0.5, 0.5, 0.5],
    [0.5, 0.5, 0.25, 0.25, 0.25, 0.25, 0.5, 0.5],
    [1.25, 0.25, 0.25, -0.75, 0, 0, 0, 0],
    [0.5] * 8,
    [0.25, -0.25, 0.25, -0.25, 0.25, -0.25, 0.25, 0.75],
]


def _bf16_value(bits: int) -> float:
    return float(np.array([bits << 16], np.uint32).view(np.float32)[0])


def _f32(x) -> np.float32:
    return np.float32(x)


def parity_fix_ties(x32: np.ndarray) -> bool:
    """The coset decision and parity fix of one vector restated in float32
    (identity of the exact distance difference), reporting whether the fix
    has more than one candidate coordinate."""
    R = np.rint(x32)
    F = np.floor(x32)
    ae = np.abs((x32 - R).astype(np.float32))
    s = np.float32(0.0)
    for v in ae:
        s = np.float32(s + v)
    mx, mn = ae.max(), ae.min()
    odd0, odd1 = int(R.sum()) & 1, int(F.sum()) & 1
    dd = np.float32(s - np.float32(2.0))
    if odd0:
        dd = np.float32(dd + _f32(float(mx) * -2.0 + 1.0))
    if odd1:
        dd = _f32(float(mn) * -2.0 + float(dd))
    one = dd > 0
    fix = odd1 if one else odd0
    if not fix:
        return False
    T = mn if one else mx
    return int((ae == T).sum()) > 1


def tie_tiles(count: int, seed: int):
    """Rows of fp32 tiles whose vector 0 ties; returns (rows, number of ties)."""
    rng = np.random.default_rng(seed)
    H = scipy.linalg.hadamard(N).astype(np.float64)
    s = oracle.signs(SEED, 0, N).astype(np.float64)
    c = oracle.rate_constant("E8", BPS)
    rows, ties = [], 0
    for trial in range(count):
        v = rng.integers(-24, 25, size=N).astype(np.float64) * 2.0**-5
        v[:8] = 0.0
        t = np.array(TEMPLATES[trial % len(TEMPLATES)], np.float64) * (1 if trial % 2 else -1)
        delta = None
        for _ in range(6):
            w = s * (H @ v) / N
            w32 = w.astype(np.float32)
            assert np.array_equal(w32.astype(np.float64), w)  # exact in binary32
            d = _bf16_value(oracle.tile_scale(oracle.sumsq(w32), c)[0])
            if delta == d:
                break
            delta = d
            v[:8] = t * delta
        else:
            continue
        if oracle.encode_tile(w32, "E8", BPS, SEED, 0, 0)["scale"] == 0:
            continue
        inv = np.float32(1.0) / np.float32(delta)
        x = (v[:8].astype(np.float32) * inv).astype(np.float32)
        ties += parity_fix_ties(x)
        rows.append(w32)
    return np.stack(rows), ties


def test_constructed_tiles_tie_on_the_cpu():
    """The construction (CPU only): most tiles carry a tie, every input is an
    exact binary32 transform of the planned rotated tile."""
    rows, ties = tie_tiles(60, 3)
    assert rows.shape[0] >= 50
    assert ties >= 20, ties


@pytest.mark.gpu
def test_gpu_matches_the_sequential_rule_on_ties():
    rows, ties = tie_tiles(200, 5)
    assert ties >= 60, ties
    x = torch.from_numpy(rows).to(DEV)
    s, st = gpu_encode(x, N, "E8", BPS, SEED)
    assert st == 0
    ref = oracle.encode(rows, N, "E8", BPS, SEED)
    assert_streams_equal(fetch(s), ref)

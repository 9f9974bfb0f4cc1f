"""Pins of the oracle's integer tensor-core product (CPU only).

The int8 product multiplies A = 2y (the doubled lattice coordinates, exact
integers for E8, D4 and Z) by activations rotated like the weights and
quantized per (batch row, column tile) to q = rint(x~ 127 / max|x~|).  The
pins check it against facts outside its code:
* the quantized activations against the rotation computed with scipy's
  Hadamard matrix in binary64 (|x~ - s q| <= s / 2, the extreme at +-127);
* A / 2 against the lattice points recovered from the binary64 decode;
* the product against numpy's matmul of the decoded, rotated weights and the
  dequantized activations (the integer sums are exact);
* the distance to the exact product X W_hat^T against the closed-form bound
  of the activation rounding;
* saturation of |2y| > 127, and A2 (no integer form) refused.
The fp8 variant's E4M3 rounding is pinned against torch's float8_e4m3fn
conversion (all 256 codes, every midpoint, random values), its product
against numpy's matmul of the rounded operands, and the pages' finding that
int8 beats fp8 on the rotated lattice output is checked on Gaussian weights.
"""
import math

import numpy as np
import pytest
import scipy.linalg

import oracle


def rotate64(x, seed, j, n):
    return scipy.linalg.hadamard(n).astype(np.float64) @ (oracle.signs(seed, j, n) * np.asarray(x, np.float64))


def test_activation_quantization_against_binary64_rotation():
    rng = np.random.default_rng(3)
    n = 256
    X = (rng.standard_normal((6, 3 * n)) * np.array([[0.1], [1.0], [30.0], [1e-3], [2.0], [0.5]])).astype(np.float32)
    X[4, 7] = 50.0  # an outlier coordinate
    Q, S = oracle.act_quant_i8(X, n, 11)
    for b in range(6):
        for j in range(3):
            xt = rotate64(X[b, j * n:(j + 1) * n], 11, j, n)
            s = float(S[b, j])
            assert math.isclose(s, np.abs(xt).max() / 127, rel_tol=1e-5)
            q = Q[b, j * n:(j + 1) * n].astype(np.float64)
            assert np.abs(q).max() == 127
            # rounding to the grid of step s, plus the binary32 transform's error
            assert np.all(np.abs(xt - s * q) <= 0.5 * s + 1e-5 * np.abs(xt).max())
    Z, SZ = oracle.act_quant_i8(np.zeros((1, n), np.float32), n, 1)
    assert not Z.any() and SZ[0, 0] == 0.0


@pytest.mark.parametrize("lat", ["E8", "D4", "Z"])
def test_doubled_points_are_the_decoded_lattice_points(lat):
    rng = np.random.default_rng(oracle.LATTICES[lat])
    n, seed = 128, 5
    for t in range(8):
        w = (rng.standard_normal(n) * 0.03).astype(np.float32)
        e = oracle.encode_tile(w, lat, 4.0, seed, j=0, t=t)
        st, a, sat = oracle.tile_points_i8(e["words"], n, lat, e["k"])
        assert st == 0 and sat == 0
        st, w_hat = oracle.decode_tile(e["words"], n, lat, e["scale"], e["k"], seed, 0, t)
        delta = float(np.uint32(e["scale"] << 16).view(np.float32))
        p = rotate64(w_hat, seed, 0, n) / delta  # the lattice point, up to binary64 rounding
        assert np.array_equal(a.astype(np.float64), np.rint(2 * p))
        assert np.allclose(2 * p, a, atol=1e-9)


@pytest.mark.parametrize("lat", ["E8", "D4", "Z"])
def test_product_is_matmul_of_rotated_operands_and_within_the_rounding_bound(lat):
    rng = np.random.default_rng(20 + oracle.LATTICES[lat])
    rows, cols, n, seed = 24, 768, 256, 9
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    X = rng.standard_normal((7, cols)).astype(np.float32)
    st = oracle.encode(W, n, lat, 4.0, seed)
    Y, status, sat = oracle.gemm_i8(st, rows, cols, n, lat, seed, X)
    assert status == 0 and sat == 0
    W_hat, _ = oracle.decode(st, rows, cols, n, lat, seed)
    tpr = cols // n
    Zr = np.stack([np.concatenate([rotate64(W_hat[r, j * n:(j + 1) * n], seed, j, n) for j in range(tpr)])
                   for r in range(rows)])  # Delta y per tile, rotated domain
    Q, S = oracle.act_quant_i8(X, n, seed)
    Xq = Q.astype(np.float64) * np.repeat(S.astype(np.float64), n, axis=1)  # s q
    ref = Xq @ Zr.T / n
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # against the exact product: the activation rounding moves each term by at most s / 2
    exact = X.astype(np.float64) @ W_hat.T
    bound = (np.repeat(S.astype(np.float64), n, axis=1) / 2) @ np.abs(Zr).T / n
    assert np.all(np.abs(Y - exact) <= bound * 1.0001 + 1e-5 * np.abs(exact).max())
    assert np.abs(Y - exact).max() > 0  # the int8 activations are an approximation


def test_saturation_and_a2():
    rng = np.random.default_rng(2)
    n = 128
    w = (rng.standard_normal(n)).astype(np.float32)
    e = oracle.encode_tile(w, "Z", 8.0, 1)  # 8 bps: coordinates far beyond 63
    st, a, sat = oracle.tile_points_i8(e["words"], n, "Z", e["k"])
    assert st == 0 and sat > 0 and np.abs(a.astype(int)).max() == 127
    e = oracle.encode_tile(w, "A2", 4.0, 1)
    st, a, _ = oracle.tile_points_i8(e["words"], n, "A2", e["k"])
    assert st == oracle.CORRUPT and not a.any()


# ------------------------------------------------------------ fp8 (E4M3) product
def test_e4m3_codes_and_rounding_against_torch():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_value(codes)
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~finite)
    assert np.array_equal(got[finite], ref[finite])
    # every finite code round-trips; midpoints between neighbours and random
    # values (within the saturation bound) round like torch's conversion
    vals = np.unique(ref[finite & (ref >= 0)])
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(0)
    xs = np.concatenate([vals, mids, -mids, rng.uniform(-464, 464, 3000), rng.standard_normal(2000) * 0.01,
                         [463.9, 464.0, -464.0, 2.0**-10, 3 * 2.0**-10]]).astype(np.float32)
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3(xs), want)
    assert oracle.e4m3(np.float32(1e6)) == 0x7E and oracle.e4m3(np.float32(-1e30)) == 0xFE  # saturating


def test_e4m3_activation_quantization_against_binary64_rotation():
    rng = np.random.default_rng(8)
    n = 256
    X = (rng.standard_normal((4, 2 * n)) * np.array([[0.1], [1.0], [30.0], [1e-3]])).astype(np.float32)
    Q, S = oracle.act_quant_e4m3(X, n, 4)
    for b in range(4):
        for j in range(2):
            xt = rotate64(X[b, j * n:(j + 1) * n], 4, j, n)
            s = float(S[b, j])
            assert math.isclose(s, np.abs(xt).max() / 448, rel_tol=1e-5)
            q = oracle.e4m3_value(Q[b, j * n:(j + 1) * n]).astype(np.float64)
            assert np.abs(q).max() == 448
            # E4M3 keeps 3 fraction bits: relative error at most 2^-4 above 2^-6, absolute 2^-10 below
            e = np.abs(xt / s - q)
            assert np.all(e <= np.maximum(np.abs(xt / s) * 2.0**-4, 2.0**-10) + 1e-4)


def test_e4m3_product_is_matmul_and_int8_is_closer_to_the_exact_product():
    """The pages report int8 ahead of fp8 on the lattice output after the
    rotation: with A = 2y exact in int8 but rounded beyond +-16 in E4M3, and
    the activations on 255 uniform levels against E4M3's 3 fraction bits, the
    integer product lands closer to the exact product."""
    rng = np.random.default_rng(31)
    rows, cols, n, seed = 32, 1024, 256, 2
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    X = rng.standard_normal((8, cols)).astype(np.float32)
    st = oracle.encode(W, n, "E8", 4.0, seed)
    Y8, s8, sat8 = oracle.gemm_e4m3(st, rows, cols, n, "E8", seed, X)
    assert s8 == 0 and sat8 == 0
    # reference: numpy matmul of the E4M3-rounded operands, scaled per tile
    W_hat, _ = oracle.decode(st, rows, cols, n, "E8", seed)
    tpr = cols // n
    A = np.zeros((rows, cols))
    D = np.zeros((rows, tpr))
    for r in range(rows):
        for j in range(tpr):
            t = r * tpr + j
            delta = float(np.uint32(int(st["scale"][t]) << 16).view(np.float32))
            y2 = np.rint(2 * rotate64(W_hat[r, j * n:(j + 1) * n], seed, j, n) / delta)
            A[r, j * n:(j + 1) * n] = oracle.e4m3_value(oracle.e4m3(y2.astype(np.float32)))
            D[r, j] = delta
    Q, S = oracle.act_quant_e4m3(X, n, seed)
    Qv = oracle.e4m3_value(Q).astype(np.float64)
    ref = np.einsum("btk,rtk,rt,bt->br", Qv.reshape(8, tpr, n), A.reshape(rows, tpr, n), D, S.astype(np.float64)) / (2 * n)
    assert np.allclose(Y8, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    exact = X.astype(np.float64) @ W_hat.T
    Yi, si, _ = oracle.gemm_i8(st, rows, cols, n, "E8", seed, X)
    err8 = np.linalg.norm(Y8 - exact) / np.linalg.norm(exact)
    erri = np.linalg.norm(Yi - exact) / np.linalg.norm(exact)
    assert erri < err8

"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute: a
published test vector, a library routine (scipy's Sylvester Hadamard matrix,
numpy's rint and matmul), a closed form (normalized second moments, index of
a sublattice, entropy of a finely quantized Gaussian, expected Rice cost of a
geometric source, distortion of subtractive dither), brute force over
enumerated lattice points, or a layout worked by hand.  A plausible slip in
the oracle -- a dropped sign or term, a swapped operand, a wrong constant or
tie rule -- makes at least one of them fail.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")
FACTS = json.load(open(os.path.join(GOLD, "lattice_facts.json")))
LATS = ["Z", "A2", "D4", "E8"]
SQ3 = math.sqrt(3.0)


# ------------------------------------------------------------ randomness
def test_splitmix64_published_outputs():
    g = json.load(open(os.path.join(GOLD, "splitmix64.json")))
    for i, o in zip(g["inputs"], g["outputs"]):
        assert oracle.mix64(int(i, 16)) == int(o, 16)


def test_signs_and_uniforms_are_balanced():
    s = np.concatenate([oracle.signs(7, j, 256) for j in range(64)])
    assert set(np.unique(s)) == {-1, 1}
    assert abs(s.mean()) < 4 / math.sqrt(s.size)
    r = np.array([oracle.uniform(3, t, i) for t in range(40) for i in range(128)])
    assert r.min() >= 0.0 and r.max() < 1.0
    assert abs(r.mean() - 0.5) < 4 * math.sqrt(1 / 12 / r.size)
    # 16-bit grid: r * 2^16 is an integer, and all four 16-bit fields of a hash are used
    assert np.all(np.floor(r * 2**16) == r * 2**16)
    for k in range(4):
        rk = r.reshape(40, 32, 4)[:, :, k].ravel()
        assert abs(rk.mean() - 0.5) < 4 * math.sqrt(1 / 12 / rk.size)


def test_signs_and_uniforms_match_worked_examples():
    """Worked examples of the sign vector and the dither uniforms, derived step
    by step from their definition with only the published-vector-pinned mix64
    (tests/golden/make_hash_bits.py): a swapped hash argument or a mirrored bit
    index in the oracle would change them."""
    g = json.load(open(os.path.join(GOLD, "hash_bits.json")))
    for e in g["signs"]:
        want = np.array([-1 if ch == "-" else 1 for ch in e["signs"]])
        assert np.array_equal(oracle.signs(e["seed"], e["j"], e["n"]), want), (e["seed"], e["j"])
    for e in g["uniforms"]:
        got = [oracle.uniform(e["seed"], e["t"], i) * 65536.0 for i in range(len(e["r_times_2^16"]))]
        assert got == [float(v) for v in e["r_times_2^16"]], (e["seed"], e["t"])


# ------------------------------------------------------------ Hadamard
@pytest.mark.parametrize("n", [2, 8, 64, 128, 256, 1024])
def test_fwht_is_sylvester_hadamard(n):
    H = scipy.linalg.hadamard(n).astype(np.int64)
    rng = np.random.default_rng(n)
    v = rng.integers(-1000, 1000, size=n)
    # integers well inside 2^24 are exact in binary32 at every stage
    assert np.array_equal(oracle.fwht_f32(v.astype(np.float32)).astype(np.int64), H @ v)
    assert np.array_equal(oracle.fwht_f64(v.astype(np.float64)).astype(np.int64), H @ v)
    cols = np.stack([oracle.fwht_f32(np.eye(n, dtype=np.float32)[i]) for i in range(n)])
    assert np.array_equal(cols.astype(np.int64) @ cols.T.astype(np.int64), n * np.eye(n, dtype=np.int64))


@pytest.mark.parametrize("n", [64, 128, 256, 1024])
def test_rht_round_trip_and_parseval(n):
    rng = np.random.default_rng(1 + n)
    w = rng.standard_normal(n).astype(np.float32)
    s = oracle.signs(11, 3, n).astype(np.float32)
    v = oracle.fwht_f32(s * w)
    back = s * oracle.fwht_f32(v) / n
    assert np.max(np.abs(back - w)) < 8 * math.log2(n) * 2**-24 * np.abs(w).sum() / math.sqrt(n)
    assert abs(np.sum(v.astype(np.float64) ** 2) - n * np.sum(w.astype(np.float64) ** 2)) < 1e-4 * n * np.sum(w**2)


def test_sumsq_tree():
    rng = np.random.default_rng(5)
    wi = rng.integers(-300, 300, 256).astype(np.float32)
    assert oracle.sumsq(wi) == float(np.sum(wi.astype(np.int64) ** 2))  # exact on small integers
    w = rng.standard_normal(256).astype(np.float32)
    ref = float(np.sum(w.astype(np.float64) ** 2))
    assert abs(oracle.sumsq(w) - ref) <= 10 * 2**-24 * ref


# ------------------------------------------------------------ lattices
def member(lat, y):
    """Lattice membership from the definitions (independent of the decoder)."""
    y = np.asarray(y, np.float64)
    if lat == "Z":
        return np.all(y == np.round(y))
    if lat == "D4":
        return np.all(y == np.round(y)) and int(round(y.sum())) % 2 == 0
    if lat == "E8":
        t = 2 * y
        if not np.all(t == np.round(t)):
            return False
        par = np.mod(np.round(t), 2)
        return np.all(par == par[0]) and int(round(y.sum())) % 2 == 0
    # A2: (a + c/2, (b + c/2) sqrt3)
    t0, t1 = 2 * y[0], 2 * y[1] / SQ3
    return (abs(t0 - round(t0)) < 1e-5 and abs(t1 - round(t1)) < 1e-5
            and (round(t0) - round(t1)) % 2 == 0)


def candidates(lat, x):
    """All lattice points within 1.5 of x in every coordinate (brute force)."""
    d = len(x)
    if lat == "A2":
        out = []
        for c in (0, 1):
            a0 = math.floor(x[0] - c / 2)
            b0 = math.floor(x[1] / SQ3 - c / 2)
            for a in range(a0 - 2, a0 + 3):
                for b in range(b0 - 2, b0 + 3):
                    out.append((a + c / 2, (b + c / 2) * SQ3))
        return np.array(out)
    offs = np.array(list(itertools.product((-1, 0, 1), repeat=d)), np.float64)
    pts = [np.rint(x) + offs]
    if lat == "E8":
        pts.append(np.floor(x) + 0.5 + offs)
    P = np.concatenate(pts)
    if lat in ("D4", "E8"):
        keep = np.mod(np.round(np.sum(P - (P % 1 != 0) * 0.5, axis=1)), 2) == 0
        P = P[keep]
    return P


@pytest.mark.parametrize("lat", LATS)
def test_minimal_vectors_are_fixed_points(lat):
    d = FACTS["dimension"][lat]
    norm = FACTS["min_norm"][lat]
    if lat == "A2":
        mins = [(math.cos(k * math.pi / 3), math.sin(k * math.pi / 3)) for k in range(6)]
    else:
        grid = [(-1, 0, 1)] * d if lat != "E8" else [(-1, -0.5, 0, 0.5, 1)] * d
        mins = [p for p in itertools.product(*grid)
                if abs(sum(v * v for v in p) - norm) < 1e-9 and member(lat, p)]
    assert len(mins) == FACTS["kissing"][lat]
    for p in mins:
        c, z, pt = oracle.nearest(lat, p)
        assert np.allclose(pt, p, atol=1e-6), (p, pt)


@pytest.mark.parametrize("lat", LATS)
def test_nearest_point_brute_force(lat):
    d = FACTS["dimension"][lat]
    rng = np.random.default_rng(100 + d)
    X = np.concatenate([rng.uniform(-3, 3, (600, d)), rng.standard_normal((600, d)) * 8,
                        np.round(rng.uniform(-4, 4, (200, d)) * 2) / 2,  # half-integer ties
                        np.round(rng.uniform(-4, 4, (200, d)) * 4) / 4])
    X = X.astype(np.float32)
    _, _, P = oracle.nearest_batch(lat, X)
    for x, p in zip(X.astype(np.float64), P.astype(np.float64)):
        assert member(lat, p), (x, p)
        C = candidates(lat, x)
        dmin = np.min(np.sum((C - x) ** 2, axis=1))
        dp = np.sum((p - x) ** 2)
        assert dp <= dmin + 1e-5 * (1 + np.dot(x, x)), (lat, x, p, dp, dmin)


def test_tie_rules():
    # D4 parity fix moves the first coordinate of largest |e| towards x
    c, z, _ = oracle.nearest("D4", [0.5, 0.5, 0.0, 0.0])   # rint -> 0,0,0,0 (even) -> no fix
    assert list(z) == [0, 0, 0, 0]
    c, z, _ = oracle.nearest("D4", [0.4, 1.2, 0.0, 0.0])   # rint -> 0,1 odd; |e| max at i=0
    assert list(z) == [1, 1, 0, 0]
    # E8 keeps the integer coset on exact ties: x = (1/4)^8 is equidistant
    c, z, _ = oracle.nearest("E8", np.full(8, 0.25))
    assert c == 0 and list(z) == [0] * 8
    c, z, _ = oracle.nearest("E8", np.full(8, 0.2500001))
    assert c == 1
    # an integer vector with an odd sum: every |e| is 0, so the first
    # coordinate moves, and it moves up (the "towards x" rule when x is exact)
    c, z, _ = oracle.nearest("D4", [1.0, 0.0, 0.0, 0.0])
    assert list(z) == [2, 0, 0, 0]
    c, z, _ = oracle.nearest("E8", [0.0, -3.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0])
    assert c == 0 and list(z) == [1, -3, 0, 0, 0, 0, 0, 0]
    # the half-integer coset: x all half-integers with an odd floor sum is not in
    # E8; its nearest point moves one coordinate of the nearest half-integer
    # vector by 1 (every |e| ties at 1/2, so the first), and at x - floor(x) =
    # 1/2 exactly the move is up: z = floor(x) + e_0
    c, z, pt = oracle.nearest("E8", [0.5] * 7 + [1.5])
    assert c == 1 and list(z) == [1, 0, 0, 0, 0, 0, 0, 1] and list(pt) == [1.5] + [0.5] * 6 + [1.5]


@pytest.mark.parametrize("lat", LATS)
def test_translation_invariance(lat):
    d = FACTS["dimension"][lat]
    rng = np.random.default_rng(7 + d)
    X = rng.uniform(-2, 2, (300, d)).astype(np.float32)
    _, _, P = oracle.nearest_batch(lat, X)
    # a lattice vector with a small exactly representable coordinate set
    lam = {"Z": [3.0], "A2": [1.5, 1.5 * SQ3], "D4": [1, 1, 2, 0], "E8": [0.5] * 6 + [-0.5] * 2}[lat]
    lam = np.array(lam, np.float64)
    if lat == "A2":  # keep the translation exact in binary32 for the first coordinate only
        lam = np.array([2.0, 0.0])
    Y = (X.astype(np.float64) + lam).astype(np.float32)
    _, _, P2 = oracle.nearest_batch(lat, Y)
    ok = np.all(np.abs(P2.astype(np.float64) - (P.astype(np.float64) + lam)) < 1e-4, axis=1)
    assert ok.mean() > 0.995  # only exact ties may differ


@pytest.mark.parametrize("lat", LATS)
def test_index_of_2z_sublattice_gives_cell_volume(lat):
    """Distinct Q(x) modulo a sublattice L' of known volume = vol(L')/V(lattice)."""
    d = FACTS["dimension"][lat]
    rng = np.random.default_rng(21 + d)
    X = rng.uniform(0, 2, (40000, d)).astype(np.float32)
    if lat == "A2":
        X[:, 1] *= SQ3 / 2
        X[:, 0] /= 2
    _, _, P = oracle.nearest_batch(lat, X)
    if lat == "A2":
        key = np.stack([np.mod(np.round(2 * P[:, 0]), 2), np.mod(np.round(2 * P[:, 1] / SQ3), 2)], 1)
        vol_sub = SQ3  # Z x sqrt3 Z
    else:
        key = np.mod(np.round(2 * P.astype(np.float64)), 4)
        vol_sub = 2.0**d if lat != "Z" else 1.0
        if lat == "Z":
            key = np.mod(np.round(P.astype(np.float64)), 1)
    n_cosets = len({tuple(r) for r in key})
    assert math.isclose(vol_sub / n_cosets, FACTS["cell_volume"][lat], rel_tol=1e-9)


@pytest.mark.parametrize("lat", LATS)
def test_normalized_second_moment(lat):
    d = FACTS["dimension"][lat]
    V = FACTS["cell_volume"][lat]
    rng = np.random.default_rng(31 + d)
    N = 200000
    X = rng.uniform(0, 4, (N, d))  # whole periods of a sublattice: 4Z^d, or 4Z x 4 sqrt3 Z for A2
    if lat == "A2":
        X[:, 1] *= SQ3
    _, _, P = oracle.nearest_batch(lat, X.astype(np.float32))
    e2 = np.sum((X.astype(np.float32).astype(np.float64) - P) ** 2, axis=1) / d / V ** (2 / d)
    G, se = e2.mean(), e2.std() / math.sqrt(N)
    assert abs(G - FACTS["G"][lat]) < max(4 * se, 2e-4), (G, se)


def entropy_bits(rows):
    _, cnt = np.unique(rows, axis=0, return_counts=True)
    p = cnt / cnt.sum()
    return float(-(p * np.log2(p)).sum())


@pytest.mark.parametrize("lat,R", [("Z", 3.0), ("Z", 4.0), ("Z", 5.0), ("A2", 4.0), ("D4", 3.0)])
def test_rate_constant_hits_target_entropy(lat, R):
    """Step c(R) on unit-variance Gaussian coordinates gives entropy ~ R bits/dim."""
    d = FACTS["dimension"][lat]
    c = oracle.rate_constant(lat, R)
    rng = np.random.default_rng(int(10 * R) + d)
    X = (rng.standard_normal((600000 // d, d)) / c).astype(np.float32)
    cc, z, _ = oracle.nearest_batch(lat, X)
    H = entropy_bits(np.concatenate([z, cc[:, None]], 1)) / d
    assert abs(H - R) < 0.03, H


@pytest.mark.parametrize("R", [3.0, 4.0, 5.0])
def test_e8_rate_constant_hits_target_entropy(R):
    """E8's index at step c(R) on unit Gaussian coordinates carries ~R bits per
    dimension.  The per-vector entropy E[-log2 P(Q(X))] is estimated without any
    rate formula: P(y) is the Gaussian mass of y's Voronoi cell (volume 1),
    i.e. phi(y) times the mean of phi(y + u) / phi(y) over points u uniform on
    the cell, drawn as z - Q(z) for z uniform on [0, 2)^8 (a fundamental box
    of the sublattice 2Z^8)."""
    c = oracle.rate_constant("E8", R)
    var = 1.0 / (c * c)
    rng = np.random.default_rng(int(100 * R))
    X = (rng.standard_normal((8000, 8)) / c).astype(np.float32)
    _, _, Y = oracle.nearest_batch("E8", X)
    Y = Y.astype(np.float64)
    Zb = rng.uniform(0.0, 2.0, (2048, 8)).astype(np.float32)
    _, _, QZ = oracle.nearest_batch("E8", Zb)
    U = Zb.astype(np.float64) - QZ.astype(np.float64)
    a = -(Y @ U.T) / var - (U * U).sum(1)[None, :] / (2 * var)
    am = a.max(1, keepdims=True)
    log_mean = (am[:, 0] + np.log(np.exp(a - am).mean(1)))
    log_phi = -(Y * Y).sum(1) / (2 * var) - 4.0 * math.log(2 * math.pi * var)
    H = float(-(log_phi + log_mean).mean() / math.log(2.0)) / 8
    assert abs(H - R) < 0.03, H


# ------------------------------------------------------------ E8 decision
def _d8_plain(y):
    """Conway & Sloane's D8 decoder in binary64: round every coordinate; if the
    sum is odd, round the coordinate farthest from its integer (first such
    index) the other way."""
    f = np.rint(y)
    e = y - f
    rows = np.nonzero(np.mod(f.sum(1), 2) != 0)[0]
    b = np.argmax(np.abs(e[rows]), 1)
    f[rows, b] += np.where(e[rows, b] >= 0, 1.0, -1.0)
    return f


def _plain_e8(X):
    """The plain two-candidate E8 decision in binary64: D8(x) against
    D8(x - 1/2) + 1/2, by their squared distances."""
    X64 = X.astype(np.float64)
    y0, y1 = _d8_plain(X64), _d8_plain(X64 - 0.5) + 0.5
    return ((X64 - y0) ** 2).sum(1), ((X64 - y1) ** 2).sum(1)


# The oracle decides E8's coset from an exact identity for d0 - d1 evaluated in
# binary32 (each |e| <= 1/2, at most a dozen roundings of terms below 4):
# its decision can differ from the binary64 one only within this band.
E8_BAND = 4e-6


def _check_e8_against_plain(X):
    c, _, pt = oracle.nearest_batch("E8", X)
    d0, d1 = _plain_e8(X)
    P = pt.astype(np.float64)
    # the oracle's point is in E8: all-integer or all-half-integer, even sum
    twice = 2 * P
    assert np.all(twice == np.rint(twice))
    par = np.mod(twice, 2)
    assert np.all(par == par[:, :1]) and np.all(np.mod(P.sum(1), 2) == 0)
    assert np.array_equal(c, par[:, 0].astype(np.int32))
    # outside the band the decisions agree and the oracle's point is nearest
    gap = np.abs(d0 - d1)
    plain = (d1 < d0).astype(np.int32)
    assert np.all((c == plain) | (gap <= E8_BAND))
    dor = ((X.astype(np.float64) - P) ** 2).sum(1)
    assert np.all(dor <= np.minimum(d0, d1) + E8_BAND)
    return int(np.sum(c != plain))


def test_e8_decision_agrees_with_the_plain_binary64_rule_on_random_inputs():
    """A million random vectors at several scales: every decision matches the
    plain binary64 rule (tie flips below 1e-6 of vectors)."""
    rng = np.random.default_rng(88)
    flips, total = 0, 0
    for scale in (0.3, 1.0, 3.0, 10.0, 60.0):
        X = (rng.standard_normal((200000, 8)) * scale).astype(np.float32)
        flips += _check_e8_against_plain(X)
        total += X.shape[0]
    assert flips <= 1e-6 * total, flips


def test_e8_decision_agrees_with_the_plain_binary64_rule_near_ties():
    """Points within a few binary32 ulps of the boundary between the two
    cosets (the midpoint (1/4)^8 of 0 and (1/2)^8, moved by lattice vectors
    and sign changes that keep it on the boundary, plus tiny noise): any
    disagreement with the binary64 rule lies inside the rounding band."""
    rng = np.random.default_rng(89)
    n = 100000
    base = np.full((n, 8), 0.25)
    flip = rng.integers(0, 2, (n, 8)) * 2 - 1
    flip[:, 7] = flip[:, :7].prod(1)  # an even number of minus signs keeps (1/2)^8 * signs in E8
    lam = _d8_plain(rng.normal(0, 4, (n, 8)))
    lam[:, 0] += np.mod(lam.sum(1), 2)  # an even sum: a D8 point
    X = (lam + base * flip + rng.normal(0, 1, (n, 8)) * 2.0**-21).astype(np.float32)
    _check_e8_against_plain(X)


# ------------------------------------------------------------ strip + zigzag
@pytest.mark.parametrize("lat", LATS)
def test_symbols_round_trip_and_zigzag_order(lat):
    d = FACTS["dimension"][lat]
    rng = np.random.default_rng(41 + d)
    X = (rng.standard_normal((3000, d)) * 20).astype(np.float32)
    cc, Z, _ = oracle.nearest_batch(lat, X)
    for c, z in zip(cc, Z):
        u = oracle.symbols(lat, z)
        assert np.array_equal(oracle.unsymbols(lat, u), z)
    # zigzag order 0, -1, 1, -2, 2 -> 0, 1, 2, 3, 4 (first coordinate is never halved)
    for zv, uv in [(0, 0), (-1, 1), (1, 2), (-2, 3), (2, 4), (-7, 13)]:
        z = np.zeros(d, np.int32)
        z[0] = zv
        if lat in ("D4", "E8"):
            z[1] = zv  # keep the sum even
        assert oracle.symbols(lat, z)[0] == uv
    if lat in ("D4", "E8"):  # the last coordinate is stored halved (floor)
        z = np.zeros(d, np.int32)
        z[0], z[-1] = 1, -3
        assert oracle.symbols(lat, z)[-1] == 3  # floor(-3/2) = -2 -> zigzag 3


# ------------------------------------------------------------ Rice code
def test_rice_length_closed_form_and_round_trip():
    rng = np.random.default_rng(51)
    for lat in LATS:
        d = FACTS["dimension"][lat]
        n = 256
        C = n // d if lat in ("A2", "E8") else 0
        for k in range(16):
            u = rng.geometric(0.2, n).astype(np.uint32) - 1
            u[rng.integers(0, n)] = 5000 if k < 4 else 70000
            coset = rng.integers(0, 2, n // d).astype(np.uint8) if C else np.zeros(n // d, np.uint8)
            words = oracle.pack_tile(lat, n, k, coset, u, cap_words=20000)
            bits = C + int(np.sum(u >> k)) + n * (1 + k)   # sum of (u >> k) + 1 + k, plus coset bits
            assert len(words) == (bits + 31) // 32
            st, c2, u2 = oracle.unpack_tile(lat, n, k, words)
            assert st == 0 and np.array_equal(u2, u) and np.array_equal(c2, coset)


def test_rice_layout_worked_by_hand():
    g = json.load(open(os.path.join(GOLD, "rice_layout.json")))
    for ex in g["examples"]:
        w = oracle.pack_tile(ex["lattice"], ex["n"], ex["k"], ex["coset"], ex["u"])
        assert [int(x) for x in w] == [int(h, 16) for h in ex["words"]], ex


def test_best_k_matches_expected_cost_of_geometric_source():
    """For P(u) = (1 - th) th^u, E floor(u / 2^k) = th^(2^k) / (1 - th^(2^k))."""
    rng = np.random.default_rng(61)
    for mean in [0.3, 1.0, 3.0, 10.0, 40.0, 300.0]:
        th = mean / (1 + mean)
        cost = [th ** (2**k) / (1 - th ** (2**k)) + 1 + k for k in range(16)]
        srt = sorted(cost)
        if srt[1] - srt[0] < 0.02:
            continue  # near tie in expectation: a finite sample may pick either
        u = (rng.geometric(1 - th, 200000) - 1).astype(np.uint32)
        assert oracle.best_k(u) == int(np.argmin(cost)), mean


def test_rice_cost_is_convex_in_k():
    rng = np.random.default_rng(71)
    for _ in range(200):
        u = (rng.geometric(rng.uniform(0.01, 0.9), 256) - 1).astype(np.uint32)
        c = [oracle.rice_cost(u, k) for k in range(16)]
        diffs = np.diff(c)
        assert np.all(np.diff(diffs) >= 0)
        assert oracle.best_k(u) == int(np.argmin(c))  # numpy argmin returns the first minimum


def test_unpack_rejects_corrupt_tiles():
    rng = np.random.default_rng(81)
    for seed in range(20):
        w = rng.standard_normal(256).astype(np.float32)
        r = oracle.encode_tile(w, "E8", 4.0, seed)
        words, k = r["words"], r["k"]
        st, _, u = oracle.unpack_tile("E8", 256, k, words)
        assert st == 0
        used = 32 + 256 * k + int(np.sum((u >> k) + 1))
        assert len(words) == (used + 31) // 32
        assert oracle.unpack_tile("E8", 256, k, words[:-1])[0] == oracle.CORRUPT       # truncated
        assert oracle.unpack_tile("E8", 256, k, np.append(words, 0))[0] == oracle.CORRUPT  # extra word
        assert oracle.unpack_tile("E8", 256, 16, words)[0] == oracle.CORRUPT              # k out of range
        if used % 32:
            bad = words.copy()
            bad[-1] |= np.uint32(1 << 31)                                                  # one in padding
            assert oracle.unpack_tile("E8", 256, k, bad)[0] == oracle.CORRUPT


# ------------------------------------------------------------ whole tiles
def test_tile_scale_rounds_to_bf16_like_torch():
    """Delta = bf16_rn(c sqrt(S)): with S = 1 the oracle's rounding of c to bf16
    equals torch's float32 -> bfloat16 conversion (round to nearest even),
    including values exactly halfway between two bf16 numbers."""
    import torch
    rng = np.random.default_rng(12)
    v = rng.uniform(-30, 30, 20000).astype(np.float32)
    v = np.exp2(v).astype(np.float32)
    bits = v.view(np.uint32)
    mids = (bits & 0xFFFF0000) | rng.choice(np.array([0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF], np.uint32), bits.size)
    v = np.concatenate([v, mids.view(np.float32)])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.tile_scale(1.0, float(x))[0] for x in v], np.uint16)
    assert np.array_equal(got, want)


def test_zero_and_nonfinite_tiles():
    z = oracle.encode_tile(np.zeros(256, np.float32), "E8", 4.0, 1)
    assert z["scale"] == 0 and z["k"] == 0 and z["status"] == 0
    assert [int(x) for x in z["words"]] == [0] + [0xFFFFFFFF] * 8  # 32 coset zeros, 256 unary "1"s
    w = np.ones(256, np.float32)
    w[17] = np.nan
    r = oracle.encode_tile(w, "E8", 4.0, 1)
    assert r["status"] == oracle.NONFINITE and r["scale"] == 0
    assert np.array_equal(r["words"], z["words"])
    w[17] = np.inf
    assert oracle.encode_tile(w, "E8", 4.0, 1)["status"] == oracle.NONFINITE
    st, out = oracle.decode_tile(z["words"], 256, "E8", 0, 0, 1)
    assert st == 0 and np.all(out == 0)
    # energy below 2^-96: coded as zero without a status bit; just above: a real tile
    tiny = np.zeros(256, np.float32)
    tiny[3] = 2.0**-49
    r = oracle.encode_tile(tiny, "E8", 4.0, 1)
    assert r["scale"] == 0 and r["status"] == 0 and np.array_equal(r["words"], z["words"])
    tiny[3] = 2.0**-47
    assert oracle.encode_tile(tiny, "E8", 4.0, 1)["scale"] != 0


def mse_closed_form(lat, delta, n):
    """High-resolution distortion per input element: G V^(2/d) Delta^2 / n."""
    d = FACTS["dimension"][lat]
    return FACTS["G"][lat] * FACTS["cell_volume"][lat] ** (2 / d) * delta**2 / n


def bf16_value(bits):
    return np.frombuffer((np.uint32(bits) << np.uint32(16)).tobytes(), np.float32)[0]


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("R", [4.0, 6.0])
def test_encode_decode_distortion_matches_closed_form(lat, R):
    rng = np.random.default_rng(int(R) * 10 + FACTS["dimension"][lat])
    n, ratios, bits = 256, [], 0
    for t in range(120):
        w = (rng.standard_normal(n) * rng.uniform(0.01, 3)).astype(np.float32)
        r = oracle.encode_tile(w, lat, R, 9, j=t % 3, t=t)
        st, out = oracle.decode_tile(r["words"], n, lat, r["scale"], r["k"], 9, j=t % 3, t=t)
        assert st == 0
        ratios.append(np.mean((out - w.astype(np.float64)) ** 2) / mse_closed_form(lat, bf16_value(r["scale"]), n))
        bits += 32 * len(r["words"])
    assert 0.93 < np.mean(ratios) < 1.07, np.mean(ratios)
    rate = bits / (120 * n)
    assert R - 0.1 < rate < R + 0.45, rate  # payload bits per element incl. coset bits and padding


def test_symbols_in_stream_equal_lattice_coordinates():
    rng = np.random.default_rng(91)
    for lat in LATS:
        d = FACTS["dimension"][lat]
        w = rng.standard_normal(128).astype(np.float32)
        r = oracle.encode_tile(w, lat, 3.0, 4, j=2, t=8)
        st, coset, u = oracle.unpack_tile(lat, 128, r["k"], r["words"])
        assert st == 0
        assert np.array_equal(coset, r["coset"])
        z = np.concatenate([oracle.unsymbols(lat, u[q * d:(q + 1) * d]) for q in range(128 // d)])
        assert np.array_equal(z, r["z"])


# ------------------------------------------------------------ dither
BOX_HALF_WIDTH = {"E8": [0.5] * 7 + [1.0], "D4": [0.5] * 3 + [1.0], "A2": [0.5, math.sqrt(3) / 2], "Z": [0.5]}


@pytest.mark.parametrize("lat", ["D4", "E8", "Z", "A2"])
def test_dither_is_uniform_on_a_sublattice_box(lat):
    """delta is uniform on the centred box of a sublattice's fundamental
    domain: D_d for E8 and D4, Z x sqrt3 Z for A2, Z itself; coordinate m
    spans [-w_m, w_m) with mean 0 and variance w_m^2 / 3."""
    d = FACTS["dimension"][lat]
    w = np.array(BOX_HALF_WIDTH[lat])
    D = np.array([oracle.dither(lat, 13, t, v) for t in range(500) for v in range(128 // d)]).astype(np.float64)
    assert np.all(D >= -w) and np.all(D < w)
    assert np.all(np.abs(D.mean(axis=0)) < 4 * w / math.sqrt(3 * D.shape[0]))
    assert np.all(np.abs(D.var(axis=0) / (w ** 2 / 3) - 1) < 0.06)
    # the box's volume is a whole number of lattice cells: 2 V for E8 and A2 (their sublattices
    # D8 and Z x sqrt3 Z have index 2), V for D4 and Z (the box is a fundamental domain of the lattice)
    cells = np.prod(2 * w) / FACTS["cell_volume"][lat]
    assert abs(cells - (2 if lat in ("E8", "A2") else 1)) < 1e-12


@pytest.mark.parametrize("lat", ["D4", "E8", "Z", "A2"])
def test_dither_reduced_by_the_lattice_is_uniform_on_the_cell(lat):
    """delta - Q(delta) lies in the Voronoi cell with the cell's second moment
    G V^(2/d) and mean 0: delta mod the lattice is uniform, which is what
    subtractive dither needs."""
    d = FACTS["dimension"][lat]
    D = np.array([oracle.dither(lat, 21, t, v) for t in range(500) for v in range(128 // d)])
    _, _, P = oracle.nearest_batch(lat, D)
    R = D.astype(np.float64) - P
    _, _, P2 = oracle.nearest_batch(lat, R.astype(np.float32))
    assert np.mean(np.all(P2 == 0, axis=1)) > 0.999
    m2 = np.mean(np.sum(R ** 2, axis=1)) / d
    ref = FACTS["G"][lat] * FACTS["cell_volume"][lat] ** (2 / d)
    assert abs(m2 / ref - 1) < 0.05
    assert np.all(np.abs(R.mean(axis=0)) < 0.05)


def test_sixteen_bit_dither_grid_bias_is_below_two_to_minus_sixteen():
    """Exact, by enumeration of the grid: with delta = r - 1/2 over all 2^16
    grid values r, the mean error rint(x + delta) - delta - x of the scalar
    lattice is within 2^-16 of 0 for any x (a sample of x, ties included)."""
    r = np.arange(2**16, dtype=np.float64) * 2.0**-16
    delta = r - 0.5
    for x in [0.0, 0.25, 0.5, 1e-6, 0.3333, -1.75, 123.456789, 2.0**-17, 0.5 + 2.0**-17]:
        y = x + delta
        q = np.where(y - np.floor(y) == 0.5, np.floor(y) + (np.floor(y) % 2 == 1), np.round(y))
        bias = np.mean(q - delta - x)
        assert abs(bias) <= 2.0**-16, (x, bias)
    # the oracle's scalar dither lies on that grid
    D = np.array([oracle.dither("Z", 5, t, v)[0] for t in range(50) for v in range(128)], np.float64)
    assert np.all((D + 0.5) * 2**16 == np.floor((D + 0.5) * 2**16))


def kv_rows(vec, rows):
    return np.tile(vec.astype(np.float32), (rows, 1))


@pytest.mark.parametrize("lat", ["D4", "E8"])
def test_dither_unbiased_per_vector_for_a_fixed_rotation(lat):
    """One vector k stored in many KV rows: same rotation (column tile 0),
    different dither (tile index).  <q, k_hat> - <q, k> averages to 0 with
    dither; without dither every row carries the same error."""
    rng = np.random.default_rng(3)
    n, rows, R = 128, 3000, 2.0
    kvec = rng.standard_normal(n).astype(np.float32)
    q = rng.standard_normal(n)
    X = kv_rows(kvec, rows)
    errs = {}
    for dith in (True, False):
        s = oracle.encode(X, n, lat, R, 77, dither=dith)
        out, st = oracle.decode(s, rows, n, n, lat, 77, dither=dith)
        assert st == 0
        errs[dith] = (out - kvec.astype(np.float64)) @ q
    e = errs[True]
    assert abs(e.mean()) < 4 * e.std() / math.sqrt(rows)
    assert np.ptp(errs[False]) == 0.0 and abs(errs[False][0]) > 4 * e.std() / math.sqrt(rows)


@pytest.mark.parametrize("lat", ["D4", "E8", "A2", "Z"])
def test_dithered_distortion_is_exact_at_low_rate(lat):
    """With subtractive dither the error is uniform on the cell at any rate."""
    rng = np.random.default_rng(17)
    n, rows, R = 128, 400, 1.0
    X = rng.standard_normal((rows, n)).astype(np.float32)
    s = oracle.encode(X, n, lat, R, 5, dither=True)
    out, st = oracle.decode(s, rows, n, n, lat, 5, dither=True)
    deltas = np.array([bf16_value(b) for b in s["scale"]])
    ratio = np.mean(np.mean((out - X) ** 2, axis=1) / mse_closed_form(lat, deltas, n))
    assert abs(ratio - 1) < 0.05, ratio


# ------------------------------------------------------------ matrices + GEMV
def bf16_bits_of(x):
    """Round-to-nearest-even bf16 bit patterns of float32 values (test helper)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_matrix_encode_threads_and_offsets():
    rng = np.random.default_rng(101)
    X = bf16_bits_of(rng.standard_normal((9, 512)) * 0.02)
    a = oracle.encode(X, 256, "E8", 4.0, 42, threads=1)
    b = oracle.encode(X, 256, "E8", 4.0, 42, threads=4)
    for key in ("payload", "off", "scale", "k"):
        assert np.array_equal(a[key], b[key])
    assert a["off"][0] == 0 and np.all(np.diff(a["off"].astype(np.int64)) > 0)
    assert a["off"][-1] == a["payload"].size
    for t in range(18):  # each tile's slice equals the single-tile encoding
        r, j = divmod(t, 2)
        w = (X[r, 256 * j: 256 * j + 256].astype(np.uint32) << 16).view(np.float32)
        e = oracle.encode_tile(w, "E8", 4.0, 42, j=j, t=t)
        assert np.array_equal(a["payload"][a["off"][t]: a["off"][t + 1]], e["words"])


def test_gemv_equals_decode_then_matmul():
    rng = np.random.default_rng(111)
    X = bf16_bits_of(rng.standard_normal((12, 768)) * 0.02)
    s = oracle.encode(X, 256, "E8", 4.0, 3)
    W, st = oracle.decode(s, 12, 768, 256, "E8", 3)
    x = rng.standard_normal(768)
    y = oracle.gemv(s, 12, 768, 256, "E8", 3, x)
    assert np.allclose(y, W @ x, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ KV attention
def test_kv_attention_matches_exact_attention_at_high_rate():
    """At 8 bps the compressed cache is nearly exact: the oracle's attention
    must agree with softmax attention on the raw K, V (numpy) to within the
    quantization error, and be a convex combination of the decoded rows."""
    rng = np.random.default_rng(123)
    heads, tokens, d = 2, 96, 128
    K = rng.standard_normal((heads * tokens, d)).astype(np.float32)
    V = rng.standard_normal((heads * tokens, d)).astype(np.float32)
    q = rng.standard_normal((heads, d))
    scale = 1 / math.sqrt(d)
    ks = oracle.encode(K, d, "E8", 8.0, 7, dither=True)
    vs = oracle.encode(V, d, "E8", 8.0, 8, dither=True)
    got = oracle.kv_attention(ks, vs, heads, tokens, d, "E8", 7, 8, q, scale)
    for h in range(heads):
        s = scale * (K[h * tokens:(h + 1) * tokens].astype(np.float64) @ q[h])
        p = np.exp(s - s.max())
        ref = (p / p.sum()) @ V[h * tokens:(h + 1) * tokens]
        assert np.max(np.abs(got[h] - ref)) < 0.02, np.max(np.abs(got[h] - ref))
    # swapping the value cache for the key cache changes the output (no mix-up of streams)
    other = oracle.kv_attention(ks, ks, heads, tokens, d, "E8", 7, 7, q, scale)
    assert np.max(np.abs(other - got)) > 0.05


def test_kv_attention_grouped_queries_follow_their_kv_head():
    """Grouped-query attention: query head qh reads KV head qh // group.  At
    8 bps each query's output must match exact softmax attention over the raw
    K, V of its own head, and not that of any other head."""
    rng = np.random.default_rng(321)
    heads, tokens, d, group = 3, 40, 64, 3
    K = (rng.standard_normal((heads * tokens, d)) * np.array([1.0, 3.0, 0.5]).repeat(tokens)[:, None]).astype(np.float32)
    V = (rng.standard_normal((heads * tokens, d)) + np.arange(heads).repeat(tokens)[:, None]).astype(np.float32)
    q = rng.standard_normal((heads * group, d))
    scale = 1 / math.sqrt(d)
    ks = oracle.encode(K, d, "D4", 8.0, 1, dither=True)
    vs = oracle.encode(V, d, "D4", 8.0, 2, dither=True)
    got = oracle.kv_attention(ks, vs, heads, tokens, d, "D4", 1, 2, q, scale, group=group)
    assert got.shape == (heads * group, d)

    def exact(h, qv):
        s = scale * (K[h * tokens:(h + 1) * tokens].astype(np.float64) @ qv)
        p = np.exp(s - s.max())
        return (p / p.sum()) @ V[h * tokens:(h + 1) * tokens]

    for qh in range(heads * group):
        errs = [np.max(np.abs(got[qh] - exact(h, q[qh]))) for h in range(heads)]
        assert errs[qh // group] < 0.02, errs
        assert all(e > 0.2 for h, e in enumerate(errs) if h != qh // group), errs


def test_gemm_is_decode_then_matmul_and_matches_gemv_per_row():
    """The batched product equals the decoded matrix times each activation row,
    and each of its rows equals the (separately pinned) batch-1 GEMV."""
    rng = np.random.default_rng(77)
    rows, cols = 10, 512
    X = bf16_bits_of(rng.standard_normal((rows, cols)) * 0.02)
    s = oracle.encode(X, 256, "E8", 4.0, 9)
    W, _ = oracle.decode(s, rows, cols, 256, "E8", 9)
    A = rng.standard_normal((3, cols))
    Y = oracle.gemm(s, rows, cols, 256, "E8", 9, A)
    assert Y.shape == (3, rows)
    assert np.allclose(Y, A @ W.T, rtol=1e-13, atol=1e-13)
    for b in range(3):
        assert np.allclose(Y[b], oracle.gemv(s, rows, cols, 256, "E8", 9, A[b]), rtol=1e-12, atol=1e-12)

"""Pins of the oracle's fixed-rate stream (compact headers, exact rate
control) to facts outside its search (CPU only).

The fixed-rate tile must (a) hold exactly the variable-rate tile layout at
the scale it chose -- checked by cutting the slot to the tile's own words
and running the variable-rate unpacker and decoder on them, (b) fit its
slot -- checked from the raw bits (the last one bit of a tile is its last
terminator), (c) be locally finest -- the next smaller bf16 scale does not
fit, (d) agree with a brute-force scan of every scale near the answer, and
(e) spend exactly (32 S + 20) / n bits per coordinate, side information
included.  A slip in the search (a flipped comparison, returning the wrong
end of the bracket, a skipped bisection) or in the size (a dropped coset or
terminator term) breaks one of these.
"""
import math

import numpy as np
import pytest

import oracle

LATS = ["Z", "A2", "D4", "E8"]


def _coset_bits(lattice, n):
    d = oracle.LATTICES[lattice]
    return n // d if d in (2, 8) else 0


def _bits_used(slot):
    """Bit length of a tile from its slot's raw words: highest one bit + 1."""
    nz = np.nonzero(slot)[0]
    if nz.size == 0:
        return 0
    w = int(nz[-1])
    return 32 * w + int(slot[w]).bit_length()


def _rotated(w, seed, j, n):
    return oracle.fwht_f32(oracle.signs(seed, j, n).astype(np.float32) * np.asarray(w, np.float32))


def test_slot_sizes_closed_form():
    # floor((bps n - 20) / 32) words; 20 bits of side information (bf16 Delta + 4-bit k)
    assert oracle.fixed_slot_words(256, "E8", 4.0) == 31
    assert oracle.fixed_slot_words(128, "E8", 4.0) == 15
    assert oracle.fixed_slot_words(64, "Z", 5.0) == 9
    assert oracle.fixed_slot_words(1024, "D4", 2.0) == 63
    # the all-zero tile: n terminators plus the coset bits
    assert oracle.min_slot_words(128, "E8") == math.ceil((128 + 16) / 32)
    assert oracle.min_slot_words(64, "A2") == math.ceil((64 + 32) / 32)
    assert oracle.min_slot_words(256, "D4") == 8
    assert oracle.fixed_slot_words(128, "E8", 1.0) == -1  # below the all-zero tile
    for n in (64, 128, 256, 1024):
        for bps in (2.0, 3.0, 4.0, 5.5, 8.0):
            S = oracle.fixed_slot_words(n, "E8", bps)
            assert (32 * S + 20) <= bps * n < (32 * (S + 1) + 20)


def test_k_nibbles_packed_by_hand():
    assert oracle.pack_k([1, 2, 3]).tolist() == [0x21, 0x03]
    assert oracle.pack_k([15, 0, 7, 9]).tolist() == [0x0F, 0x97]
    k = np.random.default_rng(0).integers(0, 16, 37).astype(np.uint8)
    assert np.array_equal(oracle.unpack_k(oracle.pack_k(k), 37), k)


@pytest.mark.parametrize("lattice", LATS)
@pytest.mark.parametrize("dither", [False, True])
def test_fixed_tile_is_a_variable_tile_that_fits(lattice, dither):
    rng = np.random.default_rng(oracle.LATTICES[lattice] * 10 + dither)
    for n, bps in ((64, 4.0), (128, 3.0), (256, 4.5)):
        S = oracle.fixed_slot_words(n, lattice, bps)
        C = _coset_bits(lattice, n)
        for t in range(6):
            w = (rng.standard_normal(n) * 0.05).astype(np.float32)
            e = oracle.encode_tile_fixed(w, lattice, S, 11, j=t % 3, t=t, dither=dither)
            bits = _bits_used(e["slot"])
            assert bits <= 32 * S
            nw = (bits + 31) // 32
            assert nw == e["words"]
            assert not np.any(e["slot"][nw:])
            # the variable-rate parser reads the cut slot as a canonical tile ...
            st, cos, u = oracle.unpack_tile(lattice, n, e["k"], e["slot"][:nw])
            assert st == 0
            # ... whose Rice length accounts for every bit up to the last terminator
            assert C + oracle.rice_cost(u, e["k"]) == bits
            assert e["k"] == oracle.best_k(u)
            # and decodes to what the fixed-rate decoder returns from the whole slot
            st1, a = oracle.decode_tile(e["slot"][:nw], n, lattice, e["scale"], e["k"], 11, t % 3, t, dither)
            stream = {"payload": e["slot"], "scale": np.array([e["scale"]], np.uint16),
                      "kpack": oracle.pack_k([e["k"]]), "slot": S}
            b, st2 = oracle.decode_fixed(stream, 1, n, n, lattice, 11, dither)
            assert st1 == 0 and st2 == 0
            if t % 3 == 0 and (t == 0 or not dither):  # same column tile (and dither index)
                assert np.array_equal(a, b[0])


@pytest.mark.parametrize("lattice", LATS)
def test_next_finer_scale_does_not_fit(lattice):
    rng = np.random.default_rng(5 + oracle.LATTICES[lattice])
    n, bps = 64, 4.0
    S = oracle.fixed_slot_words(n, lattice, bps)
    for t in range(12):
        w = (rng.standard_normal(n) * (0.01 + 0.1 * t)).astype(np.float32)
        e = oracle.encode_tile_fixed(w, lattice, S, 3, 0, t)
        v = _rotated(w, 3, 0, n)
        c = e["scale"]
        assert c != 0
        assert oracle.coded_bits(v, lattice, c) <= 32 * S
        assert oracle.coded_bits(v, lattice, c - 1) > 32 * S


@pytest.mark.parametrize("lattice", LATS)
def test_answer_is_first_fitting_scale_by_brute_force(lattice):
    """Scan every bf16 scale in a window around the answer: the coded size is
    nearly monotone in the scale, so the answer should be the finest fitting
    scale of the window for almost every tile."""
    rng = np.random.default_rng(17 + oracle.LATTICES[lattice])
    n, bps = 256, 4.0  # one bf16 step moves the size by about n / 128 bits, above its jitter
    S = oracle.fixed_slot_words(n, lattice, bps)
    hits = 0
    trials = 12
    for t in range(trials):
        w = (rng.standard_normal(n) * 0.03).astype(np.float32)
        c = oracle.encode_tile_fixed(w, lattice, S, 9, 0, t)["scale"]
        v = _rotated(w, 9, 0, n)
        cs = np.arange(c - 16, c + 16)
        fit = np.array([oracle.coded_bits(v, lattice, int(x)) <= 32 * S for x in cs])
        assert fit[cs == c][0]
        hits += int(cs[np.argmax(fit)] == c)
    assert hits >= trials - 2


def test_answer_against_every_scale_of_the_window():
    """Brute force over the window below the answer on 480 tiles (four
    lattices, tiles of 64, 128 and 256, with and without dither, one tile in
    five with an outlier x20): the answer always fits and its next finer
    pattern never does (a local boundary); it is the finest fitting scale of
    the window for at least 95 % of tiles, and where a finer scale fits (the
    coded size is not monotone in the scale: the lattice decision and the
    Rice parameter jitter it by a few bits) that scale is at most 16
    patterns (one eighth of an octave) finer.  The Z lattice, whose symbols
    are monotone in the scale, always gets the finest fitting scale."""
    rng = np.random.default_rng(2024)
    exact = total = 0
    for lattice in LATS:
        for n in (64, 128, 256):
            S = oracle.fixed_slot_words(n, lattice, 4.0)
            for dither in (False, True):
                for t in range(20):
                    w = (rng.standard_normal(n) * 0.03).astype(np.float32)
                    if t % 5 == 0:
                        w[rng.integers(n)] *= 20
                    c = oracle.encode_tile_fixed(w, lattice, S, 9, 0, t, dither=dither)["scale"]
                    v = _rotated(w, 9, 0, n)
                    cs = np.arange(max(0x80, c - 24), c + 1)
                    fit = np.array([oracle.coded_bits(v, lattice, int(x), 9, t, dither) <= 32 * S for x in cs])
                    assert fit[-1] and not fit[-2], (lattice, n, dither, t)
                    finest = int(cs[np.argmax(fit)])
                    assert c - finest <= 16, (lattice, n, dither, t, c - finest)
                    if lattice == "Z":
                        assert finest == c, (n, dither, t)
                    exact += int(finest == c)
                    total += 1
    assert total == 480
    assert exact >= 0.95 * total, exact


def test_search_bracket_edges():
    n, S = 64, oracle.fixed_slot_words(64, "E8", 4.0)
    rng = np.random.default_rng(1)
    v = _rotated((rng.standard_normal(n) * 0.02).astype(np.float32), 1, 0, n)
    c_good, _ = oracle.fixed_scale(v, "E8", 0x3C00, 32 * S, 1)  # start near the answer
    # a start far too fine walks up by doubling steps to the same neighbourhood
    c_up, tr_up = oracle.fixed_scale(v, "E8", c_good - 300, 32 * S, 1)
    assert oracle.coded_bits(v, "E8", c_up) <= 32 * S < oracle.coded_bits(v, "E8", c_up - 1)
    assert tr_up <= 2 + 8 + 9
    # a start far too coarse walks down
    c_dn, _ = oracle.fixed_scale(v, "E8", c_good + 300, 32 * S, 1)
    assert oracle.coded_bits(v, "E8", c_dn) <= 32 * S < oracle.coded_bits(v, "E8", c_dn - 1)
    # a budget below everything the bracket offers: the all-zero tile
    assert oracle.fixed_scale(v, "E8", c_good, 8, 1)[0] == 0
    # a budget above everything: the finest scale of the bracket (four octaves down)
    assert oracle.fixed_scale(v, "E8", c_good, 1 << 20, 1)[0] == c_good - 512
    assert oracle.fixed_scale(v, "E8", 0, 32 * S, 1) == (0, 0)


@pytest.mark.parametrize("lattice", ["E8", "A2"])
def test_zero_and_nonfinite_tiles(lattice):
    n = 128
    S = oracle.fixed_slot_words(n, lattice, 3.0)
    e = oracle.encode_tile_fixed(np.zeros(n, np.float32), lattice, S, 1)
    assert e["scale"] == 0 and e["k"] == 0 and e["status"] == 0
    # all-zero tile: C zero coset bits then n one bits (every symbol 0, k 0)
    C = _coset_bits(lattice, n)
    bits = np.unpackbits(e["slot"].view(np.uint8), bitorder="little")
    assert not bits[:C].any() and bits[C:C + n].all() and not bits[C + n:].any()
    w = np.ones(n, np.float32)
    w[3] = np.inf
    e = oracle.encode_tile_fixed(w, lattice, S, 1)
    assert e["scale"] == 0 and e["status"] == oracle.NONFINITE


def test_matrix_rate_is_exact_and_decodes():
    rng = np.random.default_rng(4)
    rows, cols, n = 24, 512, 128
    x = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    S = oracle.fixed_slot_words(n, "E8", 4.0)
    st = oracle.encode_fixed(x, n, "E8", S, 21)
    ntiles = rows * cols // n
    assert st["payload"].size == ntiles * S and st["status"] == 0
    assert st["kpack"].size == (ntiles + 1) // 2
    side_bits = 16 * st["scale"].size + 4 * ntiles
    assert (32 * st["payload"].size + side_bits) / x.size == (32 * S + 20) / n
    W, s = oracle.decode(st, rows, cols, n, "E8", 21)
    assert s == 0
    rel = np.sqrt(np.mean((W - x) ** 2) / np.mean(x ** 2))
    # E8 at (32 S - C) / n = 3.625 payload bits per coordinate: the error sits
    # near 2^-3.6 times the lattice's sqrt(12 G) sqrt(2 pi e / 12) factor
    assert 0.05 < rel < 0.15
    # a corrupt slot (a one bit in the padding) decodes to zeros and is flagged
    bad = dict(st)
    bad["payload"] = st["payload"].copy()
    bad["payload"][S - 1] |= np.uint32(1 << 31)
    W2, s2 = oracle.decode(bad, rows, cols, n, "E8", 21)
    if _bits_used(st["payload"][:S]) < 32 * S:
        assert s2 == oracle.CORRUPT and not W2[0, :n].any()

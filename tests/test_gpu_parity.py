"""GPU path against the CPU oracle, through the C ABI (needs a B200).

Encode: tile offsets, scales, Rice parameters and payload words bit-exact.
Decode and KV decode: the oracle's own stream decoded on the GPU, each
element within 1e-5 x its tile's dequantized max-abs (plus one bf16 rounding
for bf16 outputs).  Decode-GEMV: within the fp32 accumulation bound.
Shapes span several encode chunks with a ragged last chunk.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_quantization_tile_b200 import hq, workloads
from gpu_util import (DEV, assert_recon_close, assert_streams_equal, device_stream, fetch, gemv_tolerance,
                      gpu_decode, gpu_encode, host_input)

pytestmark = pytest.mark.gpu

LATS = ["E8", "D4", "A2", "Z"]
SHAPES = {64: (37, 128), 128: (29, 256), 256: (19, 512), 512: (11, 1024), 1024: (9, 2048)}


def make_input(rows, cols, seed, dtype=torch.bfloat16):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * 0.02
    x[:, seed % cols] *= 20.0  # an outlier column
    return x.to(dtype).to(DEV)


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("tile", [64, 128, 256, 512, 1024])
@pytest.mark.parametrize("dither", [False, True])
def test_encode_bit_exact(lat, tile, dither):
    rows, cols = SHAPES[tile]
    for bps, dtype in [(4.0, torch.bfloat16), (1.5, torch.bfloat16), (7.0, torch.float32)]:
        x = make_input(rows, cols, tile + int(bps), dtype)
        s, st = gpu_encode(x, tile, lat, bps, 42, dither)
        assert st == 0
        ref = oracle.encode(host_input(x), tile, lat, bps, 42, dither)
        assert_streams_equal(fetch(s), ref)


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("tile", [64, 256, 1024])
@pytest.mark.parametrize("dither", [False, True])
def test_decode_close(lat, tile, dither):
    rows, cols = SHAPES[tile]
    x = make_input(rows, cols, 3)
    ref = oracle.encode(host_input(x), tile, lat, 4.0, 9, dither)
    w64, st = oracle.decode(ref, rows, cols, tile, lat, 9, dither)
    assert st == 0
    s = device_stream(ref)
    for dtype in (torch.bfloat16, torch.float32):
        out, gst = gpu_decode(s, rows, cols, tile, lat, 4.0, 9, dither, dtype)
        assert gst == 0
        assert_recon_close(out, w64, tile, 9, dtype == torch.bfloat16)


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("tile", [64, 128, 256, 512])
def test_decode_gemv_close(lat, tile):
    rows, cols = 45, 4 * tile
    x = make_input(rows, cols, 11)
    ref = oracle.encode(host_input(x), tile, lat, 4.0, 5)
    g = torch.Generator(device="cpu").manual_seed(2)
    xv = torch.randn(cols, generator=g).to(torch.bfloat16)
    yref = oracle.gemv(ref, rows, cols, tile, lat, 5, xv.float().numpy().astype(np.float64))
    s = device_stream(ref)
    y = torch.empty(rows, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_decode_gemv(s, rows, cols, tile, lat, 4.0, 5, xv.to(DEV), y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    tol = gemv_tolerance(ref, rows, cols, tile, lat, 5, xv.float().numpy().astype(np.float64))
    assert np.all(np.abs(y.cpu().numpy() - yref) <= tol)


def test_tiny_config_round_trip():
    """256 x 1024 fp32 N(0,1) from seed 0, tile 256, E8 at 4 bps."""
    x = workloads.tiny(DEV)
    s, st = gpu_encode(x, 256, "E8", 4.0, 0)
    assert st == 0
    ref = oracle.encode(host_input(x), 256, "E8", 4.0, 0, threads=4)
    assert_streams_equal(fetch(s), ref)
    out, gst = gpu_decode(s, 256, 1024, 256, "E8", 4.0, 0, dtype=torch.float32)
    w64, _ = oracle.decode(ref, 256, 1024, 256, "E8", 0)
    assert gst == 0
    assert_recon_close(out, w64, 256, 0, False)


def test_encode_is_deterministic_across_calls():
    x = make_input(301, 1024, 1)
    a, _ = gpu_encode(x, 256, "E8", 4.0, 3)
    b, _ = gpu_encode(x, 256, "E8", 4.0, 3)
    fa, fb = fetch(a), fetch(b)
    for key in fa:
        assert np.array_equal(fa[key], fb[key])


# ------------------------------------------------------------------ edge cases
def test_empty_inputs():
    for rows, cols in [(0, 256), (5, 0)]:
        x = torch.zeros(rows, cols, dtype=torch.bfloat16, device=DEV)
        s = hq.alloc_stream(rows, cols, 256, "E8", 4.0, DEV)
        s.tile_off.fill_(-1)
        ws = hq.alloc_workspace(rows, cols, 256, DEV)
        hq.hq_encode(x, 256, "E8", 4.0, 1, s, ws)
        y = torch.empty(rows, cols, dtype=torch.bfloat16, device=DEV)
        hq.hq_decode(s, rows, cols, 256, "E8", 4.0, 1, y)
        torch.cuda.synchronize()
        assert int(s.tile_off[0].item()) == 0


@pytest.mark.parametrize("lat", LATS)
def test_special_tiles(lat):
    """Zero, NaN, Inf, vanishing-energy and worst-case (Hadamard-row) tiles."""
    n, seed = 256, 4
    rows = 12
    x = torch.randn(rows, 2 * n, generator=torch.Generator().manual_seed(1)) * 0.02
    x[0, :n] = 0
    x[1, 5] = float("nan")
    x[2, n + 7] = float("inf")
    x[3, :n] = 0
    x[3, 9] = 2.0**-49
    x[4, :n] = 0
    x[4, 9] = 2.0**-47
    for r, row in ((5, 0), (6, 1), (7, n - 1)):
        s = oracle.signs(seed, 0, n).astype(np.float64)
        h = np.array([(-1) ** bin(row & i).count("1") for i in range(n)], np.float64)
        x[r, :n] = torch.from_numpy(s * h * 3.0)
    x[8, n:] = 1e30
    xd = x.to(torch.bfloat16).to(DEV)
    for dither in (False, True):
        s, st = gpu_encode(xd, n, lat, 6.0, seed, dither)
        assert st == hq.HQ_ST_NONFINITE
        ref = oracle.encode(host_input(xd), n, lat, 6.0, seed, dither)
        assert ref["status"] == oracle.NONFINITE
        assert_streams_equal(fetch(s), ref)
        out, gst = gpu_decode(s, rows, 2 * n, n, lat, 6.0, seed, dither, torch.float32)
        w64, _ = oracle.decode(ref, rows, 2 * n, n, lat, seed, dither)
        assert gst == 0
        assert_recon_close(out, w64, n, seed, False)


def test_single_row_and_single_tile():
    for rows, cols, tile in [(1, 256, 256), (1, 4096, 128), (1000, 64, 64)]:
        x = make_input(rows, cols, 8)
        s, _ = gpu_encode(x, tile, "E8", 4.0, 8)
        assert_streams_equal(fetch(s), oracle.encode(host_input(x), tile, "E8", 4.0, 8))


def corrupt_cases(ref):
    """(name, mutated stream, tiles expected corrupt)."""
    out = []

    def clone():
        return {k: np.array(v, copy=True) for k, v in ref.items() if k in ("payload", "off", "scale", "k")}

    c = clone(); c["k"][3] = 16; out.append(("k out of range", c, {3}))
    c = clone(); c["scale"][4] = 0x7F80; out.append(("infinite scale", c, {4}))
    c = clone(); c["scale"][5] = 0x8000 | c["scale"][5]; out.append(("negative scale", c, {5}))
    c = clone(); c["off"][7] = c["off"][8] + 1; out.append(("offsets out of order", c, {6, 7}))
    c = clone(); c["off"][10] -= 1; out.append(("tile cut short", c, {9, 10}))
    c = clone()
    last = int(c["off"][12]) - 1
    c["payload"][last] |= np.uint32(1 << 31)
    out.append(("one bit in padding or extra terminator", c, {11}))
    c = clone(); c["off"][-1] = c["off"][-1] + 100000; out.append(("end past capacity", c, {len(c["k"]) - 1}))
    return out


def test_corrupt_streams_are_contained():
    rows, cols, tile = 8, 512, 256
    x = make_input(rows, cols, 21)
    ref = oracle.encode(host_input(x), tile, "E8", 4.0, 2)
    for name, c, tiles in corrupt_cases(ref):
        w64, st = oracle.decode(c, rows, cols, tile, "E8", 2)
        if name.startswith("one bit") and st == 0:
            continue  # the flipped bit happened to be a used bit that was already set
        assert st == oracle.CORRUPT, name
        s = device_stream(c, capacity_words=ref["payload"].size)
        out, gst = gpu_decode(s, rows, cols, tile, "E8", 4.0, 2, dtype=torch.float32)
        assert gst == hq.HQ_ST_CORRUPT, name
        for t in tiles:
            r, j = divmod(t, cols // tile)
            assert np.all(out[r, j * tile:(j + 1) * tile] == 0), name
            assert np.all(w64[r, j * tile:(j + 1) * tile] == 0), name
        assert_recon_close(out, w64, tile, 2, False)


@pytest.mark.parametrize("lat", ["E8", "Z"])
def test_long_unary_codes(lat):
    """One rotated coordinate swept from small to huge over Gaussian noise:
    its Rice code's unary part runs from a few bits to hundreds, covering
    a lane whose codes fit a 64-bit window with one code of q >= 32 and
    lanes that span more than 64 bits."""
    n, seed, rows = 256, 12, 96
    rng = np.random.default_rng(5)
    s = oracle.signs(seed, 0, n).astype(np.float64)
    H = np.array([[(-1) ** bin(r & i).count("1") for i in range(n)] for r in (0, 37, 200)], np.float64)
    x = np.zeros((rows, n))
    for r in range(rows):
        amp = 0.2 * 1.06 ** r
        x[r] = s * (H[r % 3] * amp + rng.standard_normal(n) * 0.05)
    xd = torch.from_numpy(x).to(torch.float32).to(DEV)
    for bps in (2.0, 5.0):
        g, st = gpu_encode(xd, n, lat, bps, seed)
        ref = oracle.encode(host_input(xd), n, lat, bps, seed)
        assert st == 0
        assert_streams_equal(fetch(g), ref)
        out, gst = gpu_decode(device_stream(ref), rows, n, n, lat, bps, seed, dtype=torch.float32)
        w64, _ = oracle.decode(ref, rows, n, n, lat, seed)
        assert gst == 0
        assert_recon_close(out, w64, n, seed, False)


def test_checkpoint_round_trip_on_gpu(tmp_path):
    """GPU encode -> container file -> GPU decode gives the same matrix."""
    x = make_input(33, 1024, 5)
    s, st = gpu_encode(x, 256, "E8", 4.0, 11)
    assert st == 0
    path = str(tmp_path / "w.hqf")
    hq.save_stream(path, s, 33, 1024, 256, "E8", 4.0, 11)
    s2, meta = hq.load_stream(path, DEV)
    assert meta["rows"] == 33 and meta["lattice"] == "E8" and not meta["dither"]
    a, _ = gpu_decode(s, 33, 1024, 256, "E8", 4.0, 11)
    b, _ = gpu_decode(s2, 33, 1024, 256, "E8", 4.0, 11)
    assert np.array_equal(a, b)

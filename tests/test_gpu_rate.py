"""Rate accounting on the GPU (hq_stream_stats): counts by kind and the
symbol histogram of a stream equal those read from the same stream by the
oracle's unpacker, for every lattice and for fixed-rate streams."""
import numpy as np
import pytest
import torch

import oracle
from kv_quantization_tile_b200 import hq
from gpu_util import DEV, device_stream, host_input
from test_gpu_fixed_rate import device_fixed

pytestmark = pytest.mark.gpu


def _expected(ref, ntiles, n, lat, bins, fixed_slot=0):
    d = {"Z": 1, "A2": 2, "D4": 4, "E8": 8}[lat]
    C = n // d if lat in ("E8", "A2") else 0
    counts = np.zeros(8, np.int64)
    hist = np.zeros((2, bins), np.int64)
    for t in range(ntiles):
        if fixed_slot:
            k = int(oracle.unpack_k(ref["kpack"], ntiles)[t])
            words = ref["payload"][t * fixed_slot:(t + 1) * fixed_slot]
            nw = fixed_slot
        else:
            k = int(ref["k"][t])
            o0, o1 = int(ref["off"][t]), int(ref["off"][t + 1])
            words, nw = ref["payload"][o0:o1], o1 - o0
        st, _, u = oracle.unpack_tile(lat, n, k, words)
        assert st == 0
        un = int((u.astype(np.int64) >> k).sum()) + n
        counts += [1, C, n * k, un, 32 * nw - C - n * k - un, 0 if fixed_slot else 32, 16, 4 if fixed_slot else 8]
        last = (np.arange(n) % d == d - 1) if d in (4, 8) else np.zeros(n, bool)
        for row, sel in ((0, ~last), (1, last)):
            hist[row] += np.bincount(np.minimum(u[sel], bins - 1), minlength=bins)
    return counts, hist


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
def test_stream_stats_match_the_oracle(lat):
    rows, cols, tile, bins = 24, 1024, 256, 64
    g = torch.Generator(device="cpu").manual_seed(31)
    x = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16)
    ref = oracle.encode(host_input(x), tile, lat, 4.0, 42)
    s = device_stream(ref)
    counts, hist = hq.hq_stream_stats(s, rows, cols, tile, lat, 4.0, bins=bins)
    want_c, want_h = _expected(ref, rows * cols // tile, tile, lat, bins)
    assert np.array_equal(counts.cpu().numpy(), want_c)
    assert np.array_equal(hist.cpu().numpy(), want_h)
    r = hq.rate_report(counts.cpu().tolist(), hist.cpu().tolist(), tile)
    assert abs(r["payload_bits_per_coord"] * r["coords"] - 32 * int(ref["off"][-1])) < 1e-6 * r["coords"] + 1


def test_stream_stats_of_a_fixed_rate_stream():
    rows, cols, tile, bins = 16, 512, 256, 128
    g = torch.Generator(device="cpu").manual_seed(32)
    x = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16)
    S = oracle.fixed_slot_words(tile, "E8", 4.0)
    ref = oracle.encode_fixed(host_input(x), tile, "E8", S, 42)
    s = device_fixed(ref)
    counts, hist = hq.hq_stream_stats(s, rows, cols, tile, "E8", 4.0, bins=bins)
    want_c, want_h = _expected(ref, rows * cols // tile, tile, "E8", bins, fixed_slot=S)
    assert np.array_equal(counts.cpu().numpy(), want_c)
    assert np.array_equal(hist.cpu().numpy(), want_h)

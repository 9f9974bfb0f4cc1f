"""The C-ABI library on the CPU: it loads, exports every declared symbol, and
its host-only sizing and validation behave (no kernel is launched here)."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
from kv_quantization_tile_b200 import hq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LATS = ["Z", "A2", "D4", "E8"]


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hq_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 11
    lib = hq.library()
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(hq.EXPORTS) == names


def test_error_strings_and_version():
    for code in range(6):
        assert hq.hq_error_string(code)
    assert hq.hq_error_string(99) == "unknown error"
    assert hq.hq_version() >= 100


@pytest.mark.parametrize("lat", LATS)
def test_rate_constant_bit_identical_to_oracle(lat):
    for bps in [0.25, 1.0, 1.7, 2.0, 3.0, 4.0, 4.5, 5.0, 6.0, 8.0]:
        assert np.float32(hq.hq_rate_constant(lat, bps)).tobytes() == \
            np.float32(oracle.rate_constant(lat, bps)).tobytes()


def hadamard_row_tile(n, seed, j, row, amp=1.0):
    """w = s_j . h_row: after the random signs its rotation is n * amp at one
    coordinate and zero elsewhere -- the largest possible lattice symbol."""
    s = oracle.signs(seed, j, n).astype(np.float64)
    h = np.array([(-1) ** bin(row & i).count("1") for i in range(n)], np.float64)
    return (s * h * amp).astype(np.float32)


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("tile", [64, 128, 256, 512, 1024])
def test_tile_bound_holds_on_adversarial_tiles(lat, tile):
    for bps in [0.5, 2.0, 4.0, 8.0]:
        bound = hq.hq_tile_bound_words(tile, lat, bps)
        worst = 0
        for dith in (False, True):
            for row in (0, 1, tile - 1):
                w = hadamard_row_tile(tile, 3, 0, row)
                worst = max(worst, len(oracle.encode_tile(w, lat, bps, 3, 0, 5, dith)["words"]))
            rng = np.random.default_rng(tile)
            for _ in range(4):
                w = rng.standard_normal(tile).astype(np.float32)
                w[rng.integers(tile)] *= 1e4
                worst = max(worst, len(oracle.encode_tile(w, lat, bps, 3, 0, 5, dith)["words"]))
        assert worst <= bound, (lat, tile, bps, worst, bound)


def test_sizing_functions():
    assert hq.hq_max_payload_words(10, 512, 256, "E8", 4.0) == 20 * hq.hq_tile_bound_words(256, "E8", 4.0)
    assert hq.hq_max_payload_words(0, 512, 256, "E8", 4.0) == 0
    small, big = hq.hq_encode_workspace_bytes(100, 256, 256), hq.hq_encode_workspace_bytes(100000, 256, 256)
    assert small >= 256 + 8 and big > small  # a counter area plus one slot per chunk
    with pytest.raises(hq.HQError) as e:
        hq.hq_max_payload_words(10, 500, 256, "E8", 4.0)
    assert e.value.code == hq.HQ_ERR_ARG
    with pytest.raises(hq.HQError) as e:
        hq.hq_max_payload_words(1 << 30, 1 << 14, 256, "E8", 8.0)
    assert e.value.code == hq.HQ_ERR_UNSUPPORTED
    # a row count whose tile count overflows int64 is refused, not wrapped
    with pytest.raises(hq.HQError) as e:
        hq.hq_encode_workspace_bytes((1 << 62) + 1, 1024, 256)
    assert e.value.code == hq.HQ_ERR_UNSUPPORTED
    # the no-workspace encoder refuses it too, before any device call
    out = hq.hq_stream()
    assert hq.library().hq_encode_noalloc(None, hq.HQ_BF16, (1 << 62) + 1, 1024, 256, hq.HQ_E8, 4.0, 0,
                                          ctypes.byref(out), None, None) == hq.HQ_ERR_UNSUPPORTED


def _raw_encode(x, dtype, rows, cols, tile, lat, bps, stream_struct, ws=1, wsb=1 << 20):
    lib = hq.library()
    ptr = ctypes.byref(stream_struct) if stream_struct is not None else None
    return lib.hq_encode(x, dtype, rows, cols, tile, lat, bps, 0, ptr, ws, wsb, None, None)


def test_encode_and_decode_reject_bad_arguments_before_any_launch():
    s = hq.hq_stream(16, 1 << 20, 16, 16, 16)
    ARG = hq.HQ_ERR_ARG
    assert _raw_encode(16, 0, 4, 256, 256, 8, 4.0, None) == ARG            # no stream
    assert _raw_encode(16, 0, 4, 250, 256, 8, 4.0, s) == ARG               # cols % tile
    assert _raw_encode(16, 0, 4, 256, 100, 8, 4.0, s) == ARG               # tile
    assert _raw_encode(16, 0, 4, 256, 256, 3, 4.0, s) == ARG               # lattice
    assert _raw_encode(16, 0, 4, 256, 256, 8, 0.0, s) == ARG               # bps
    assert _raw_encode(16, 0, 4, 256, 256, 8, 8.5, s) == ARG
    assert _raw_encode(16, 0, 4, 256, 256, 8, float("nan"), s) == ARG
    assert _raw_encode(16, 7, 4, 256, 256, 8, 4.0, s) == ARG               # dtype
    assert _raw_encode(16, 0, -1, 256, 256, 8, 4.0, s) == ARG              # rows
    assert _raw_encode(0, 0, 4, 256, 256, 8, 4.0, s) == ARG                # x NULL
    assert _raw_encode(18, 0, 4, 256, 256, 8, 4.0, s) == ARG               # x misaligned
    small = hq.hq_stream(16, 10, 16, 16, 16)
    assert _raw_encode(16, 0, 4, 256, 256, 8, 4.0, small) == hq.HQ_ERR_CAPACITY
    assert _raw_encode(16, 0, 4, 256, 256, 8, 4.0, s, ws=0) == hq.HQ_ERR_WORKSPACE
    assert _raw_encode(16, 0, 4, 256, 256, 8, 4.0, s, wsb=8) == hq.HQ_ERR_WORKSPACE
    lib = hq.library()
    assert lib.hq_decode(None, 4, 256, 256, 8, 4.0, 0, 16, 0, None, None) == ARG
    assert lib.hq_decode(ctypes.byref(s), 4, 256, 256, 8, 4.0, 0, 0, 0, None, None) == ARG
    assert lib.hq_decode(ctypes.byref(s), 4, 256, 256, 8, 4.0, 0, 16, 5, None, None) == ARG
    assert lib.hq_decode_gemv(ctypes.byref(s), 4, 1 << 16, 256, 8, 4.0, 0, 16, 16, None, None) == \
        hq.HQ_ERR_UNSUPPORTED


def test_kv_attention_sizing_and_validation():
    for heads, tokens, d, group in [(8, 32768, 128, 4), (1, 40000, 64, 1), (3, 333, 256, 11), (2, 1, 64, 2)]:
        w = hq.hq_kv_attention_workspace_bytes(heads, tokens, d, group)
        gb = 1 if group <= 1 else 2 if group <= 2 else 4 if group <= 4 else 8
        counters = heads * -(-group // gb) * 4
        cbytes = -(-counters // 256) * 256
        per_split = heads * group * (d + 2) * 4
        assert (w - cbytes) % per_split == 0
        splits = (w - cbytes) // per_split
        assert -(-tokens // (4096 // gb)) <= splits <= tokens
    ARG = hq.HQ_ERR_ARG
    lib = hq.library()
    out = ctypes.c_uint64(0)
    assert lib.hq_kv_attention_workspace_bytes(8, 100, 96, 1, ctypes.byref(out)) == ARG
    assert lib.hq_kv_attention_workspace_bytes(8, 100, 128, 0, ctypes.byref(out)) == ARG
    assert lib.hq_kv_attention_workspace_bytes(-1, 100, 128, 1, ctypes.byref(out)) == ARG
    assert lib.hq_kv_attention_workspace_bytes(70000, 100, 128, 1, ctypes.byref(out)) == hq.HQ_ERR_UNSUPPORTED
    s = hq.hq_stream(16, 1 << 20, 16, 16, 16)
    S = ctypes.byref(s)

    def call(k=S, v=S, heads=2, tokens=10, d=128, group=1, lat=8, bk=4.0, bv=4.0, q=16, scale=0.1, o=16,
             ws=16, wsb=1 << 20):
        return lib.hq_kv_attention(k, v, heads, tokens, d, group, lat, bk, bv, 1, 2, q, scale, o, ws, wsb, None,
                                   None)

    assert call(k=None) == ARG
    assert call(v=None) == ARG
    assert call(d=100) == ARG
    assert call(group=0) == ARG
    assert call(lat=3) == ARG
    assert call(bv=9.0) == ARG
    assert call(scale=float("inf")) == ARG
    assert call(q=0) == ARG
    assert call(q=18) == ARG
    assert call(o=0) == ARG
    assert call(o=20) == ARG
    assert call(ws=0) == hq.HQ_ERR_WORKSPACE
    assert call(wsb=64) == hq.HQ_ERR_WORKSPACE
    assert call(heads=70000) == hq.HQ_ERR_UNSUPPORTED
    assert call(heads=0) == hq.HQ_OK  # nothing to do, nothing launched


def test_fixed_rate_sizing_and_validation():
    for tile in (64, 128, 256, 512, 1024):
        for lat in LATS:
            assert hq.hq_min_slot_words(tile, lat) == oracle.min_slot_words(tile, lat)
            for bps in (1.0, 2.0, 3.3, 4.0, 8.0):
                want = oracle.fixed_slot_words(tile, lat, bps)
                if want < 0:
                    with pytest.raises(hq.HQError):
                        hq.hq_fixed_slot_words(tile, lat, bps)
                else:
                    assert hq.hq_fixed_slot_words(tile, lat, bps) == want
    lib = hq.library()
    ARG = hq.HQ_ERR_ARG

    def enc(x, rows, cols, tile, lat, st, fn=lib.hq_encode_fixed):
        return fn(x, 0, rows, cols, tile, lat, 0, ctypes.byref(st) if st is not None else None, None, None)

    ok = hq.hq_stream(16, 1 << 20, 0, 16, 16, 31)
    assert enc(16, 4, 256, 256, 8, None) == ARG                                   # no stream
    assert enc(16, 4, 256, 256, 8, hq.hq_stream(16, 1 << 20, 0, 16, 16, 0)) == ARG  # slot 0
    assert enc(16, 4, 256, 256, 8, hq.hq_stream(16, 1 << 20, 0, 16, 16, 8)) == ARG  # below the minimum (9)
    assert enc(16, 4, 256, 256, 8, hq.hq_stream(16, 1 << 20, 0, 16, 16, 65)) == ARG  # above n / 4
    assert enc(16, 4, 256, 256, 8, hq.hq_stream(16, 100, 0, 16, 16, 31)) == hq.HQ_ERR_CAPACITY
    assert enc(16, 1 << 27, 256, 256, 8, hq.hq_stream(16, 1 << 40, 0, 16, 16, 64)) == hq.HQ_ERR_UNSUPPORTED
    assert enc(0, 4, 256, 256, 8, ok) == ARG                                      # x NULL
    assert enc(18, 4, 256, 256, 8, ok) == ARG                                     # x misaligned
    assert enc(16, 4, 256, 256, 3, ok) == ARG                                     # lattice
    assert enc(16, 4, 250, 256, 8, ok) == ARG                                     # cols % tile
    assert enc(16, 4, 256, 256, 8, hq.hq_stream(16, 1 << 20, 0, 0, 16, 31)) == ARG  # no scales
    # a fixed-rate stream is not a variable-rate encode target
    assert lib.hq_encode(16, 0, 4, 256, 256, 8, 4.0, 0, ctypes.byref(hq.hq_stream(16, 1 << 20, 16, 16, 16, 31)),
                         16, 1 << 20, None, None) == ARG
    # decoders check the slot and the capacity of fixed-rate streams
    assert lib.hq_decode(ctypes.byref(hq.hq_stream(16, 1 << 20, 0, 16, 16, 8)), 4, 256, 256, 8, 4.0, 0, 16, 0,
                         None, None) == ARG
    assert lib.hq_decode(ctypes.byref(hq.hq_stream(16, 100, 0, 16, 16, 31)), 4, 256, 256, 8, 4.0, 0, 16, 0,
                         None, None) == hq.HQ_ERR_CAPACITY
    # variable-rate streams still need their offsets
    assert lib.hq_decode(ctypes.byref(hq.hq_stream(16, 1 << 20, 0, 16, 16, 0)), 4, 256, 256, 8, 4.0, 0, 16, 0,
                         None, None) == ARG


def test_attention_needs_one_stream_kind():
    lib = hq.library()
    fixed = hq.hq_stream(16, 1 << 20, 0, 16, 16, 15)
    var = hq.hq_stream(16, 1 << 20, 16, 16, 16, 0)
    for k, v in ((fixed, var), (var, fixed)):
        assert lib.hq_kv_attention(hq.ctypes.byref(k), hq.ctypes.byref(v), 2, 64, 128, 1, 8, 4.0, 4.0, 1, 2, 16, 0.1,
                                   16, 16, 1 << 20, None, None) == hq.HQ_ERR_UNSUPPORTED

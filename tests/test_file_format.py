"""The packed checkpoint container (host code of the library, CPU only):
round trip of an oracle-encoded stream, detection of corruption in every
section, truncation, foreign magic or version, and argument checks."""
import numpy as np
import pytest
import torch

import oracle
from kv_quantization_tile_b200 import hq


def host_stream(ref):
    return hq.Stream(payload=torch.from_numpy(np.ascontiguousarray(ref["payload"], np.uint32).view(np.int32).copy()),
                     tile_off=torch.from_numpy(np.ascontiguousarray(ref["off"], np.uint32).view(np.int32).copy()),
                     tile_scale=torch.from_numpy(np.ascontiguousarray(ref["scale"], np.uint16).view(np.int16).copy()),
                     tile_k=torch.from_numpy(np.ascontiguousarray(ref["k"], np.uint8).copy()))


@pytest.fixture(scope="module")
def case():
    rng = np.random.default_rng(4)
    rows, cols = 12, 768
    x = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    ref = oracle.encode(x, 256, "D4", 3.5, 77, dither=True)
    data = hq.stream_to_bytes(host_stream(ref), rows, cols, 256, "D4", 3.5, 77, dither=True)
    return rows, cols, ref, data


def test_round_trip(case):
    rows, cols, ref, data = case
    s, meta = hq.stream_from_bytes(data, device="cpu")
    assert meta == {"rows": rows, "cols": cols, "tile": 256, "lattice": "D4", "bps": 3.5, "seed": 77, "dither": True,
                    "slot_words": 0}
    assert np.array_equal(s.tile_off.numpy().view(np.uint32), ref["off"])
    assert np.array_equal(s.tile_scale.numpy().view(np.uint16), ref["scale"])
    assert np.array_equal(s.tile_k.numpy(), ref["k"])
    assert np.array_equal(s.payload.numpy().view(np.uint32)[: ref["payload"].size], ref["payload"])
    w1, _ = oracle.decode(ref, rows, cols, 256, "D4", 77, dither=True)
    back = {"payload": s.payload.numpy().view(np.uint32)[: ref["payload"].size], "off": s.tile_off.numpy().view(np.uint32),
            "scale": s.tile_scale.numpy().view(np.uint16), "k": s.tile_k.numpy()}
    w2, _ = oracle.decode(back, rows, cols, 256, "D4", 77, dither=True)
    assert np.array_equal(w1, w2)
    # size: 128-byte header + the four arrays, each 8-byte aligned
    n = ref["k"].size
    a8 = lambda v: (v + 7) // 8 * 8
    assert len(data) == a8(a8(a8(128 + 4 * (n + 1)) + 2 * n) + n) + 4 * ref["payload"].size


def expect_format_error(data):
    with pytest.raises(hq.HQError) as e:
        hq.stream_from_bytes(bytes(data), device="cpu")
    assert e.value.code == hq.HQ_ERR_FORMAT


def test_corruption_anywhere_is_detected(case):
    _, _, ref, data = case
    n = ref["k"].size
    probes = [0, 5, 20, 60, 127,                      # magic, version, shape fields, checksums
              128 + 4 * 3,                            # a tile offset
              128 + 4 * (n + 1) + 3,                  # a scale
              len(data) - 4 * ref["payload"].size - 1,  # a Rice parameter (last k byte)
              len(data) - 7]                          # a payload word
    for pos in probes:
        bad = bytearray(data)
        bad[pos] ^= 0x10
        expect_format_error(bad)


def test_truncated_and_foreign(case):
    _, _, _, data = case
    expect_format_error(data[:100])
    expect_format_error(data[:-1])
    bad = bytearray(data)
    bad[:4] = b"XXXX"
    expect_format_error(bad)


def test_argument_checks():
    info = hq.hq_file_info(4, 500, 256, 8, 4.0, 0, 1, 8, 0)  # cols not a multiple of the tile
    n = hq._u64(0)
    assert hq.library().hq_file_bytes(hq.ctypes.byref(info), hq.ctypes.byref(n)) == hq.HQ_ERR_ARG
    info = hq.hq_file_info(4, 512, 256, 8, 4.0, 0, 1, 7, 0)  # ntiles != rows * cols / tile
    assert hq.library().hq_file_bytes(hq.ctypes.byref(info), hq.ctypes.byref(n)) == hq.HQ_ERR_ARG
    info = hq.hq_file_info(4, 512, 256, 8, 4.0, 2, 1, 8, 0)  # unknown flag
    assert hq.library().hq_file_bytes(hq.ctypes.byref(info), hq.ctypes.byref(n)) == hq.HQ_ERR_ARG
    info = hq.hq_file_info(4, 512, 256, 8, 4.0, 0, 1, 8, 0)
    assert hq.library().hq_file_bytes(hq.ctypes.byref(info), hq.ctypes.byref(n)) == hq.HQ_OK
    small = np.zeros(16, np.uint8)
    off = np.zeros(9, np.uint32)
    z16, z8 = np.zeros(8, np.uint16), np.zeros(8, np.uint8)
    assert hq.library().hq_file_write(hq.ctypes.byref(info), off.ctypes.data, z16.ctypes.data, z8.ctypes.data, None,
                                      small.ctypes.data, small.size) == hq.HQ_ERR_CAPACITY


def fnv1a64(data: bytes) -> int:
    h = 0xcbf29ce484222325
    for b in data:
        h = ((h ^ b) * 0x100000001b3) & 0xFFFFFFFFFFFFFFFF
    return h


def test_header_fields_and_checksums_follow_the_documented_layout(case):
    """Published FNV-1a 64 test vectors pin this Python restatement; it then
    reproduces both stored checksums, and every header field sits at its
    documented offset."""
    import struct
    assert fnv1a64(b"") == 0xcbf29ce484222325
    assert fnv1a64(b"a") == 0xaf63dc4c8601ec8c
    assert fnv1a64(b"foobar") == 0x85944171f73967e8
    rows, cols, ref, data = case
    magic, version, hbytes, flags = struct.unpack_from("<4sIII", data, 0)
    assert (magic, version, hbytes, flags) == (b"HQF1", 1, 128, 1)
    r, c, tile, lat, bps, _, seed, ntiles, words = struct.unpack_from("<qqiifIQQQ", data, 16)
    assert (r, c, tile, lat, bps, seed, ntiles, words) == (rows, cols, 256, 4, 3.5, 77, ref["k"].size,
                                                           ref["payload"].size)
    total, body, head = struct.unpack_from("<QQQ", data, 104)
    assert total == len(data)
    assert body == fnv1a64(data[128:])
    assert head == fnv1a64(data[:120] + b"\0" * 8)


# ---------------------------------------------------------------- fixed rate
def host_fixed(ref):
    return hq.Stream(payload=torch.from_numpy(np.ascontiguousarray(ref["payload"], np.uint32).view(np.int32).copy()),
                     tile_off=torch.zeros(0, dtype=torch.int32),
                     tile_scale=torch.from_numpy(np.ascontiguousarray(ref["scale"], np.uint16).view(np.int16).copy()),
                     tile_k=torch.from_numpy(np.ascontiguousarray(ref["kpack"], np.uint8).copy()),
                     slot_words=int(ref["slot"]))


@pytest.fixture(scope="module")
def fixed_case():
    rng = np.random.default_rng(9)
    rows, cols, tile = 7, 384, 128  # 21 tiles: the last k byte holds one tile
    x = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    slot = oracle.fixed_slot_words(tile, "E8", 4.0)
    ref = oracle.encode_fixed(x, tile, "E8", slot, 31, dither=True)
    data = hq.stream_to_bytes(host_fixed(ref), rows, cols, tile, "E8", 4.0, 31, dither=True)
    return rows, cols, tile, ref, data


def test_fixed_round_trip(fixed_case):
    rows, cols, tile, ref, data = fixed_case
    s, meta = hq.stream_from_bytes(data, device="cpu")
    assert meta == {"rows": rows, "cols": cols, "tile": tile, "lattice": "E8", "bps": 4.0, "seed": 31, "dither": True,
                    "slot_words": ref["slot"]}
    assert s.slot_words == ref["slot"] and s.tile_off.numel() == 0
    assert np.array_equal(s.payload.numpy().view(np.uint32), ref["payload"])
    assert np.array_equal(s.tile_scale.numpy().view(np.uint16), ref["scale"])
    assert np.array_equal(s.tile_k.numpy(), ref["kpack"])
    back = {"payload": s.payload.numpy().view(np.uint32), "scale": s.tile_scale.numpy().view(np.uint16),
            "kpack": s.tile_k.numpy(), "slot": s.slot_words}
    w1, _ = oracle.decode(ref, rows, cols, tile, "E8", 31, dither=True)
    w2, st = oracle.decode(back, rows, cols, tile, "E8", 31, dither=True)
    assert st == 0 and np.array_equal(w1, w2)
    # no offsets section: header, scales, packed k, payload (8-byte aligned sections)
    n = ref["scale"].size
    a8 = lambda v: (v + 7) // 8 * 8
    assert len(data) == a8(a8(128 + 2 * n) + (n + 1) // 2) + 4 * n * ref["slot"]


def test_fixed_corruption_is_detected(fixed_case):
    _, _, _, ref, data = fixed_case
    n = ref["scale"].size
    for pos in (8, 40, 128 + 3, 128 + 2 * n + 2, len(data) - 5):  # header, a scale, a k byte, a payload word
        bad = bytearray(data)
        bad[pos] ^= 0x04
        expect_format_error(bad)


def test_fixed_container_checks():
    lib = hq.library()
    n = hq._u64(0)
    ok = hq.hq_file_info(4, 512, 256, 8, 4.0, 2, 1, 8, 8 * 31, 31)
    assert lib.hq_file_bytes(hq.ctypes.byref(ok), hq.ctypes.byref(n)) == hq.HQ_OK
    for bad in (hq.hq_file_info(4, 512, 256, 8, 4.0, 2, 1, 8, 8 * 8, 8),      # slot below the all-zero tile
                hq.hq_file_info(4, 512, 256, 8, 4.0, 2, 1, 8, 8 * 65, 65),    # above 8 bits per coordinate
                hq.hq_file_info(4, 512, 256, 8, 4.0, 2, 1, 8, 100, 31),       # payload is not ntiles x slot
                hq.hq_file_info(4, 512, 256, 8, 4.0, 0, 1, 8, 100, 31),       # a slot on a variable-rate stream
                hq.hq_file_info(4, 512, 256, 8, 4.0, 4, 1, 8, 8 * 31, 31)):   # unknown flag
        assert lib.hq_file_bytes(hq.ctypes.byref(bad), hq.ctypes.byref(n)) == hq.HQ_ERR_ARG
    # an odd tile count whose last k byte has its unused half set: written (the
    # writer copies the arrays as given) but refused on reading
    info = hq.hq_file_info(3, 256, 256, 8, 4.0, 2, 1, 3, 3 * 31, 31)
    assert lib.hq_file_bytes(hq.ctypes.byref(info), hq.ctypes.byref(n)) == hq.HQ_OK
    buf = np.zeros(n.value, np.uint8)
    scale = np.full(3, 0x3C00, np.uint16)
    kk = np.array([0x21, 0x53], np.uint8)
    pay = np.zeros(3 * 31, np.uint32)
    assert lib.hq_file_write(hq.ctypes.byref(info), None, scale.ctypes.data, kk.ctypes.data, pay.ctypes.data,
                             buf.ctypes.data, buf.size) == hq.HQ_OK
    expect_format_error(buf.tobytes())
    kk[1] = 0x03
    assert lib.hq_file_write(hq.ctypes.byref(info), None, scale.ctypes.data, kk.ctypes.data, pay.ctypes.data,
                             buf.ctypes.data, buf.size) == hq.HQ_OK
    s, meta = hq.stream_from_bytes(buf.tobytes(), device="cpu")
    assert meta["slot_words"] == 31 and s.tile_k.numpy().tolist() == [0x21, 0x03]

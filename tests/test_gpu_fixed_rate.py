"""Fixed-rate streams (compact headers, exact rate control) on the GPU
against the CPU oracle, through the C ABI (needs a B200).

Encode: every slot word, every scale and every packed Rice parameter
bit-exact with the oracle's fixed-rate encode, for all lattices and tile
lengths, bf16 and fp32 inputs, with and without dither, on shapes whose tile
count is odd (the last byte of packed k holds one tile).  Decode, decode-GEMV,
the KV attention and the batched tensor-core product then read the oracle's
fixed-rate streams and must match the oracle within the tolerances the
variable-rate tests use.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_quantization_tile_b200 import hq
from gpu_util import (DEV, assert_attention_close, assert_recon_close, attention_tolerance, gemm_tolerance,
                      gemv_tolerance, gpu_attention, host_input)

pytestmark = pytest.mark.gpu

LATS = ["E8", "D4", "A2", "Z"]
SHAPES = {64: (37, 192), 128: (29, 384), 256: (19, 768), 512: (11, 1536), 1024: (9, 3072)}


def make_input(rows, cols, seed, dtype=torch.bfloat16, scale=0.02):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * scale
    x[:, seed % cols] *= 20.0  # an outlier column
    return x.to(dtype).to(DEV)


def gpu_encode_fixed(x, tile, lat, slot, seed, dither=False):
    rows, cols = x.shape
    s = hq.alloc_fixed_stream(rows, cols, tile, slot, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    (hq.hq_kv_encode_fixed if dither else hq.hq_encode_fixed)(x, tile, lat, seed, s, status)
    torch.cuda.synchronize()
    return s, int(status.item())


def fetch_fixed(s: hq.Stream) -> dict:
    return {"payload": s.payload[: s.words()].cpu().numpy().view(np.uint32),
            "scale": s.tile_scale.cpu().numpy().view(np.uint16), "kpack": s.tile_k.cpu().numpy(),
            "slot": s.slot_words}


def device_fixed(ref: dict) -> hq.Stream:
    pay = np.ascontiguousarray(ref["payload"], np.uint32)
    return hq.Stream(payload=torch.from_numpy(pay.view(np.int32).copy()).to(DEV) if pay.size
                     else torch.zeros(1, dtype=torch.int32, device=DEV),
                     tile_off=torch.empty(0, dtype=torch.int32, device=DEV),
                     tile_scale=torch.from_numpy(np.ascontiguousarray(ref["scale"], np.uint16).view(np.int16)).to(DEV),
                     tile_k=torch.from_numpy(np.ascontiguousarray(ref["kpack"], np.uint8)).to(DEV),
                     slot_words=int(ref["slot"]))


def assert_fixed_equal(g: dict, r: dict):
    assert np.array_equal(g["scale"], r["scale"]), \
        f"scales differ at tiles {np.nonzero(g['scale'] != r['scale'])[0][:5].tolist()}"
    assert np.array_equal(g["kpack"], r["kpack"]), "packed rice parameters differ"
    if not np.array_equal(g["payload"], r["payload"]):
        bad = np.nonzero(g["payload"] != r["payload"])[0][:5]
        raise AssertionError(f"payload differs at words {bad.tolist()} (slot {r['slot']})")


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("tile", [64, 128, 256, 512, 1024])
@pytest.mark.parametrize("dither", [False, True])
def test_fixed_encode_bit_exact(lat, tile, dither):
    rows, cols = SHAPES[tile]
    assert (rows * cols // tile) % 2 == 1
    for bps, dtype in [(4.0, torch.bfloat16), (2.5, torch.bfloat16), (6.0, torch.float32)]:
        slot = oracle.fixed_slot_words(tile, lat, bps)
        if slot < 0:
            continue
        assert slot == hq.hq_fixed_slot_words(tile, lat, bps)
        x = make_input(rows, cols, tile + int(bps), dtype)
        s, st = gpu_encode_fixed(x, tile, lat, slot, 42, dither)
        ref = oracle.encode_fixed(host_input(x), tile, lat, slot, 42, dither, threads=8)
        assert st == ref["status"] == 0
        assert_fixed_equal(fetch_fixed(s), ref)


@pytest.mark.parametrize("lat", ["E8", "A2"])
@pytest.mark.parametrize("tile", [128, 256])
def test_fixed_encode_slot_edges(lat, tile):
    """The smallest legal slot (most tiles cannot reach their closed-form
    scale: long walks up, all-zero tiles) and the largest (8 bits per
    coordinate: walks down to the bracket's bottom)."""
    rows, cols = 13, 2 * tile
    lo, hi = hq.hq_min_slot_words(tile, lat), tile // 4
    assert lo == oracle.min_slot_words(tile, lat)
    for slot in (lo, lo + 1, hi):
        for dither in (False, True):
            x = make_input(rows, cols, slot, torch.bfloat16, scale=0.5)
            s, st = gpu_encode_fixed(x, tile, lat, slot, 5, dither)
            ref = oracle.encode_fixed(host_input(x), tile, lat, slot, 5, dither)
            assert st == ref["status"] == 0
            assert_fixed_equal(fetch_fixed(s), ref)


def test_fixed_encode_zero_nonfinite_and_empty():
    tile, lat = 128, "E8"
    slot = hq.hq_fixed_slot_words(tile, lat, 4.0)
    x = make_input(6, 3 * tile, 1)
    x[1] = 0.0
    x[2, 5] = float("nan")
    x[3, 200] = float("inf")
    s, st = gpu_encode_fixed(x, tile, lat, slot, 3)
    ref = oracle.encode_fixed(host_input(x), tile, lat, slot, 3)
    assert st == ref["status"] == oracle.NONFINITE
    assert_fixed_equal(fetch_fixed(s), ref)
    # zero rows: nothing to do, no error
    e = torch.empty(0, 3 * tile, dtype=torch.bfloat16, device=DEV)
    s0, st0 = gpu_encode_fixed(e, tile, lat, slot, 3)
    assert st0 == 0


def test_fixed_rejects_bad_slots_and_kinds():
    tile, lat = 256, "E8"
    x = make_input(4, 512, 2)
    lo = hq.hq_min_slot_words(tile, lat)
    for slot in (lo - 1, tile // 4 + 1):
        s = hq.alloc_fixed_stream(4, 512, tile, slot, DEV)
        with pytest.raises(hq.HQError) as e:
            hq.hq_encode_fixed(x, tile, lat, 1, s)
        assert e.value.code == hq.HQ_ERR_ARG
    s = hq.alloc_fixed_stream(4, 512, tile, 31, DEV)
    s.payload = s.payload[:100]  # 8 tiles need 248 words
    with pytest.raises(hq.HQError) as e:
        hq.hq_encode_fixed(x, tile, lat, 1, s)
    assert e.value.code == hq.HQ_ERR_CAPACITY
    # a fixed-rate stream is not a variable-rate encode target, and vice versa
    s = hq.alloc_fixed_stream(4, 512, tile, 31, DEV)
    with pytest.raises(hq.HQError):
        hq.hq_encode(x, tile, lat, 4.0, 1, s, hq.alloc_workspace(4, 512, tile, DEV))
    v = hq.alloc_stream(4, 512, tile, lat, 4.0, DEV)
    with pytest.raises(hq.HQError):
        hq.hq_encode_fixed(x, tile, lat, 1, v)


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("tile", [64, 256, 1024])
@pytest.mark.parametrize("dither", [False, True])
def test_fixed_decode_close(lat, tile, dither):
    rows, cols = SHAPES[tile]
    slot = oracle.fixed_slot_words(tile, lat, 4.0)
    x = make_input(rows, cols, 3)
    ref = oracle.encode_fixed(host_input(x), tile, lat, slot, 9, dither)
    w64, st = oracle.decode(ref, rows, cols, tile, lat, 9, dither)
    assert st == 0
    s = device_fixed(ref)
    for dtype in (torch.bfloat16, torch.float32):
        y = torch.empty(rows, cols, dtype=dtype, device=DEV)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        (hq.hq_kv_decode if dither else hq.hq_decode)(s, rows, cols, tile, lat, 4.0, 9, y, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_recon_close(y.float().cpu().numpy(), w64, tile, 9, dtype == torch.bfloat16)


def test_fixed_decode_flags_corrupt_slots():
    tile, lat, rows, cols = 128, "E8", 8, 512
    slot = oracle.fixed_slot_words(tile, lat, 4.0)
    ref = oracle.encode_fixed(host_input(make_input(rows, cols, 4)), tile, lat, slot, 2)
    bad = dict(ref)
    bad["payload"] = ref["payload"].copy()
    victims = []
    for t in range(0, rows * cols // tile, 5):
        words = ref["payload"][t * slot:(t + 1) * slot]
        if not words[-1] >> 31:  # the slot's last bit is padding: set it
            bad["payload"][t * slot + slot - 1] |= np.uint32(1 << 31)
            victims.append(t)
    assert len(victims) >= 3
    w64, st = oracle.decode(bad, rows, cols, tile, lat, 2)
    assert st == oracle.CORRUPT
    y = torch.empty(rows, cols, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_decode(device_fixed(bad), rows, cols, tile, lat, 4.0, 2, y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == hq.HQ_ST_CORRUPT
    out = y.cpu().numpy()
    tpr = cols // tile
    for t in victims:
        r, j = divmod(t, tpr)
        assert not out[r, j * tile:(j + 1) * tile].any()
    assert_recon_close(out, w64, tile, 2, False)


@pytest.mark.parametrize("lat", LATS)
@pytest.mark.parametrize("tile", [128, 256])
def test_fixed_gemv(lat, tile):
    rows, cols = 77, 8 * tile
    slot = oracle.fixed_slot_words(tile, lat, 4.0)
    ref = oracle.encode_fixed(host_input(make_input(rows, cols, 6)), tile, lat, slot, 13)
    g = torch.Generator(device="cpu").manual_seed(1)
    xv = torch.randn(cols, generator=g).to(torch.bfloat16)
    xd = xv.float().numpy().astype(np.float64)
    y_ref = oracle.gemv(ref, rows, cols, tile, lat, 13, xd)
    y = torch.empty(rows, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_decode_gemv(device_fixed(ref), rows, cols, tile, lat, 4.0, 13, xv.to(DEV), y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    err = np.abs(y.cpu().numpy().astype(np.float64) - y_ref)
    tol = gemv_tolerance(ref, rows, cols, tile, lat, 13, xd)
    assert np.all(err <= tol), float(np.max(err / tol))


@pytest.mark.parametrize("group", [1, 4])
def test_fixed_kv_attention(group):
    heads, tokens, d, lat = 4, 300, 128, "E8"
    slot = oracle.fixed_slot_words(d, lat, 4.0)
    g = torch.Generator(device="cpu").manual_seed(group)
    kv = torch.randn(2, heads * tokens, d, generator=g).to(torch.bfloat16)
    ks = oracle.encode_fixed(host_input(kv[0]), d, lat, slot, 100, dither=True)
    vs = oracle.encode_fixed(host_input(kv[1]), d, lat, slot, 101, dither=True)
    q = torch.randn(heads * group, d, generator=g).to(torch.bfloat16)
    qd = q.float().numpy().astype(np.float64)
    scale = d ** -0.5
    out, st = gpu_attention(device_fixed(ks), device_fixed(vs), heads, tokens, d, lat, 4.0, 4.0, 100, 101,
                            q.to(DEV), scale, group)
    assert st == 0
    ref = oracle.kv_attention(ks, vs, heads, tokens, d, lat, 100, 101, qd, scale, group=group)
    tol = attention_tolerance(ks, vs, heads, tokens, d, lat, 100, 101, qd, scale, group)
    assert_attention_close(out, ref, tol)


@pytest.mark.parametrize("batch", [1, 16, 40])
def test_fixed_decode_gemm(batch):
    rows, cols, tile, lat = 200, 1024, 256, "E8"
    slot = oracle.fixed_slot_words(tile, lat, 4.0)
    ref = oracle.encode_fixed(host_input(make_input(rows, cols, 8)), tile, lat, slot, 17)
    g = torch.Generator(device="cpu").manual_seed(batch)
    X = torch.randn(batch, cols, generator=g).to(torch.bfloat16)
    Xd = X.float().numpy().astype(np.float64)
    Y = torch.empty(batch, rows, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_decode_gemm(device_fixed(ref), rows, cols, tile, lat, 4.0, 17, X.to(DEV), Y,
                      hq.alloc_gemm_workspace(rows, cols, batch, DEV), status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Y_ref = oracle.gemm(ref, rows, cols, tile, lat, 17, Xd)
    err = np.abs(Y.cpu().numpy().astype(np.float64) - Y_ref)
    tol = gemm_tolerance(ref, rows, cols, lat, 17, Xd)
    assert np.all(err <= tol), float(np.max(err / tol))


def test_fixed_round_trip_through_gpu_encode():
    """GPU encode then GPU decode equals the oracle's decode of the oracle's
    encode (the whole fixed-rate path on the device)."""
    rows, cols, tile, lat = 33, 1024, 256, "E8"
    slot = hq.hq_fixed_slot_words(tile, lat, 4.0)
    x = make_input(rows, cols, 11)
    s, st = gpu_encode_fixed(x, tile, lat, slot, 77)
    assert st == 0
    y = torch.empty(rows, cols, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_decode(s, rows, cols, tile, lat, 4.0, 77, y, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.encode_fixed(host_input(x), tile, lat, slot, 77)
    w64, _ = oracle.decode(ref, rows, cols, tile, lat, 77)
    assert_recon_close(y.cpu().numpy(), w64, tile, 77, False)
    # exact rate: slot words plus 20 bits of side information per tile
    ntiles = rows * cols // tile
    assert s.nbytes() == 4 * ntiles * slot + 2 * ntiles + (ntiles + 1) // 2


def test_fixed_checkpoint_round_trip(tmp_path):
    """GPU fixed-rate encode -> container file -> GPU decode is bit-identical
    to decoding the stream straight from the encoder."""
    rows, cols, tile, lat = 21, 768, 128, "E8"
    slot = hq.hq_fixed_slot_words(tile, lat, 4.0)
    x = make_input(rows, cols, 12)
    s, st = gpu_encode_fixed(x, tile, lat, slot, 55, dither=True)
    assert st == 0
    path = str(tmp_path / "kv.hq")
    hq.save_stream(path, s, rows, cols, tile, lat, 4.0, 55, dither=True)
    s2, meta = hq.load_stream(path, DEV)
    assert meta["slot_words"] == slot and meta["dither"]
    outs = []
    for stream in (s, s2):
        y = torch.empty(rows, cols, dtype=torch.float32, device=DEV)
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        hq.hq_kv_decode(stream, rows, cols, tile, lat, 4.0, 55, y, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        outs.append(y.cpu())
    assert torch.equal(outs[0], outs[1])

"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (needs a B200).

The GPU encodes whole matrices; the oracle re-encodes sampled tiles one by
one (tile words, scale and Rice parameter bit-exact; word count equal to the
offset difference), offsets are checked for the invariants that hold at any
size (start at 0, strictly increasing, end inside the capacity), and sampled
decoded tiles are compared with the oracle's binary64 decode of its own
words.  Decode-GEMV rows are compared with the oracle's GEMV of the same rows
encoded by the oracle.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from kv_quantization_tile_b200 import hq, workloads
from gpu_util import bf16_neighbours, DEV, gemv_tolerance, host_input

pytestmark = pytest.mark.gpu


def sample_tiles(ntiles, m, seed, tile):
    rng = np.random.default_rng(seed)
    T = 8 if tile >= 256 else (16 if tile == 128 else 32)
    fixed = {0, 1, T - 1, T, T + 1, ntiles - 2, ntiles - 1, ntiles // 2}
    return sorted({int(t) for t in rng.choice(ntiles, size=min(m, ntiles), replace=False)} | fixed)


def tile_input(x: torch.Tensor, tile: int, t: int) -> np.ndarray:
    cols = x.shape[1]
    r, j = divmod(t, cols // tile)
    seg = x[r, j * tile:(j + 1) * tile]
    return (host_input(seg.reshape(1, -1))[0].astype(np.uint32) << 16).view(np.float32)


def check_matrix(x, tile, lat, bps, seed, dither, m=64, decode=True):
    rows, cols = x.shape
    ntiles = rows * (cols // tile)
    s = hq.alloc_stream(rows, cols, tile, lat, bps, DEV)
    ws = hq.alloc_workspace(rows, cols, tile, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    (hq.hq_kv_encode if dither else hq.hq_encode)(x, tile, lat, bps, seed, s, ws, st)
    off = s.tile_off.to(torch.int64) & 0xFFFFFFFF
    d = off[1:] - off[:-1]
    assert int(off[0]) == 0
    assert bool((d > 0).all())
    assert int(off[-1]) <= s.payload.numel()
    assert int(st.item()) == 0
    tiles = sample_tiles(ntiles, m, seed + tile, tile)
    idx = torch.tensor(tiles, device=DEV)
    o0 = off[idx].cpu().numpy()
    o1 = off[idx + 1].cpu().numpy()
    sc = s.tile_scale[idx].cpu().numpy().view(np.uint16)
    kk = s.tile_k[idx].cpu().numpy()
    widx = torch.from_numpy(np.concatenate([np.arange(a, b) for a, b in zip(o0, o1)])).to(DEV)
    words = s.payload[widx].cpu().numpy().view(np.uint32)
    if decode:
        y = torch.empty(rows, cols, dtype=torch.bfloat16, device=DEV)
        (hq.hq_kv_decode if dither else hq.hq_decode)(s, rows, cols, tile, lat, bps, seed, y, st)
        assert int(st.item()) == 0
    pos = 0
    tpr = cols // tile
    for t, a, b, sci, ki in zip(tiles, o0, o1, sc, kk):
        r, j = divmod(t, tpr)
        ref = oracle.encode_tile(tile_input(x, tile, t), lat, bps, seed, j=j, t=t, dither=dither)
        nw = int(b - a)
        assert nw == len(ref["words"]), (t, nw, len(ref["words"]))
        assert np.array_equal(words[pos:pos + nw], ref["words"]), t
        assert int(sci) == ref["scale"] and int(ki) == ref["k"], t
        pos += nw
        if decode:
            stt, w64 = oracle.decode_tile(ref["words"], tile, lat, ref["scale"], ref["k"], seed, j, t, dither)
            assert stt == 0
            got = y[r, j * tile:(j + 1) * tile].float().cpu().numpy().astype(np.float64)
            # bf16_rn of the binary64 decode; where a rounding midpoint lies
            # within 1e-5 x the tile's dequantized max-abs of it, any bf16
            # value between bf16_rn(ref - tol) and bf16_rn(ref + tol)
            vh = (w64 * oracle.signs(seed, j, tile)) @ scipy.linalg.hadamard(tile)
            tol = 1e-5 * np.abs(vh).max() + 1e-30
            near = bf16_neighbours(w64)[0]
            lo, hi = bf16_neighbours(w64 - tol)[0], bf16_neighbours(w64 + tol)[0]
            assert np.all((got == near) | ((got >= lo) & (got <= hi))), t
    return s


@pytest.mark.parametrize("bps", [3.0, 4.0, 5.0])
def test_llama_layer(bps):
    for name, x in workloads.llama_layer(DEV):
        check_matrix(x, 256, "E8", bps, 42, False, m=48)
        del x
    torch.cuda.empty_cache()


def test_gemv_workload():
    w1, w2, x1, x2 = workloads.gemv_case(DEV)
    for w, xv in ((w1, x1), (w2, x2)):
        rows, cols = w.shape
        s = check_matrix(w, 256, "E8", 4.0, 42, False, m=32, decode=False)
        y = torch.empty(rows, dtype=torch.float32, device=DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        hq.hq_decode_gemv(s, rows, cols, 256, "E8", 4.0, 42, xv, y, st)
        assert int(st.item()) == 0
        yg = y.cpu().numpy()
        xh = xv.float().cpu().numpy().astype(np.float64)
        rng = np.random.default_rng(rows)
        for r in sorted(set(rng.choice(rows, 24, replace=False).tolist()) | {0, rows - 1}):
            sub = host_input(w[r:r + 1])
            ref = oracle.encode(sub, 256, "E8", 4.0, 42)
            yr = oracle.gemv(ref, 1, cols, 256, "E8", 42, xh)[0]
            tol = gemv_tolerance(ref, 1, cols, 256, "E8", 42, xh)[0]
            assert abs(yg[r] - yr) <= tol, (r, yg[r], yr, tol)


@pytest.mark.parametrize("lat", ["D4", "E8"])
@pytest.mark.parametrize("bps", [2.0, 3.0, 4.0])
def test_kv_layer(lat, bps):
    k, v = workloads.kv_layer(DEV)
    for x in (k, v):
        check_matrix(x, 128, lat, bps, 42, True, m=48)


def test_dit_stack():
    """All 72 blocks: E8 4 bps on every matrix, D4/A2/Z 4 bps on the FFN."""
    for b in range(72):
        for name, x in workloads.dit_block(b, DEV):
            check_matrix(x, 256, "E8", 4.0, 42, False, m=3, decode=(b % 12 == 0))
            if name.startswith("ffn"):
                for lat in ("D4", "A2", "Z"):
                    check_matrix(x, 256, lat, 4.0, 42, False, m=2, decode=(b % 24 == 0))
            del x
        torch.cuda.empty_cache()


def test_every_tile_of_the_llama_and_kv_layers_is_bit_exact():
    """Whole streams, not samples: the seven Llama-3.1-8B layer matrices (E8 4
    bps, tile 256, 851,968 tiles) and the dithered KV layer (K and V, tile 128,
    524,288 tiles) against the oracle's encode of the same inputs.  Counts
    tiles whose words, scale or Rice parameter differ (tie flips included):
    the bar is below 1e-6 of vectors; the count is 0."""
    import os
    from gpu_util import fetch
    threads = max(1, os.cpu_count() or 1)
    flipped, total = 0, 0
    cases = [(x, 256, False, 42) for _, x in workloads.llama_layer(DEV)]
    cases += [(x, 128, True, 42 + i) for i, x in enumerate(workloads.kv_layer(DEV))]
    for x, tile, dither, seed in cases:
        rows, cols = x.shape
        s = hq.alloc_stream(rows, cols, tile, "E8", 4.0, DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        (hq.hq_kv_encode if dither else hq.hq_encode)(x, tile, "E8", 4.0, seed, s,
                                                       hq.alloc_workspace(rows, cols, tile, DEV), st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        g = fetch(s)
        ref = oracle.encode(host_input(x), tile, "E8", 4.0, seed, dither=dither, threads=threads)
        n = g["k"].size
        bad = (g["scale"] != ref["scale"]) | (g["k"] != ref["k"])
        same_len = np.diff(g["off"].astype(np.int64)) == np.diff(ref["off"].astype(np.int64))
        bad |= ~same_len
        if not np.array_equal(g["payload"], ref["payload"]):
            # locate differing tiles by their word ranges
            diff_words = np.nonzero(g["payload"][: ref["payload"].size] != ref["payload"])[0]
            bad[np.searchsorted(ref["off"][1:].astype(np.int64), diff_words, side="right")] = True
        flipped += int(bad.sum())
        total += n
        del s, g, ref
        torch.cuda.empty_cache()
    print(f"{flipped} differing tiles of {total}")
    assert total == 851968 + 524288
    assert flipped == 0


def test_every_tile_of_one_dit_block_is_bit_exact():
    """Whole streams of one DiT block (its ten matrices, 268 M weights, E8 4
    bps, tile 256) and of its two FFN matrices with D4, A2 and Z at 4 bps,
    against the oracle's encode of the same inputs: offsets, scales, Rice
    parameters and every payload word equal."""
    import os
    from gpu_util import fetch
    threads = max(1, os.cpu_count() or 1)
    ntiles = 0
    for name, x in workloads.dit_block(0, DEV):
        rows, cols = x.shape
        lats = ["E8"] + (["D4", "A2", "Z"] if name.startswith("ffn") else [])
        xh = host_input(x)
        for lat in lats:
            s = hq.alloc_stream(rows, cols, 256, lat, 4.0, DEV)
            st = torch.zeros(1, dtype=torch.int32, device=DEV)
            hq.hq_encode(x, 256, lat, 4.0, 42, s, hq.alloc_workspace(rows, cols, 256, DEV), st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            g = fetch(s)
            ref = oracle.encode(xh, 256, lat, 4.0, 42, threads=threads)
            assert np.array_equal(g["off"], ref["off"]), (name, lat)
            assert np.array_equal(g["scale"], ref["scale"]), (name, lat)
            assert np.array_equal(g["k"], ref["k"]), (name, lat)
            assert np.array_equal(g["payload"], ref["payload"]), (name, lat)
            ntiles += g["k"].size
            del s, g, ref
        del x, xh
        torch.cuda.empty_cache()
    assert ntiles == (8 * 4096 * 16 + 2 * (16384 * 16)) + 3 * 2 * (16384 * 16)


@pytest.mark.parametrize("case", ["llama_layer", "kv_layer"])
def test_fixed_rate_full_size_sampled_tiles(case):
    """Fixed-rate streams at full size (31-word slots for the Llama layer at
    tile 256, 15-word slots for the dithered KV layer at tile 128): tiles are
    independent, so the oracle re-encodes sampled tiles alone and their
    slots, scales and packed Rice parameters must match bit for bit; sampled
    decoded tiles match the oracle's decode of its own slots."""
    if case == "llama_layer":
        mats, tile, dither = [m for _, m in workloads.llama_layer(DEV)], 256, False
    else:
        mats, tile, dither = list(workloads.kv_layer(DEV)), 128, True
    lat, seed = "E8", 42
    slot = hq.hq_fixed_slot_words(tile, lat, 4.0)
    for mi, x in enumerate(mats):
        rows, cols = x.shape
        ntiles = rows * (cols // tile)
        s = hq.alloc_fixed_stream(rows, cols, tile, slot, DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        (hq.hq_kv_encode_fixed if dither else hq.hq_encode_fixed)(x, tile, lat, seed, s, st)
        y = torch.empty(rows, cols, dtype=torch.float32, device=DEV)
        (hq.hq_kv_decode if dither else hq.hq_decode)(s, rows, cols, tile, lat, 4.0, seed, y, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        tiles = sample_tiles(ntiles, 48, 7 * mi + tile, tile)
        pay = s.payload.view(-1, slot)[torch.tensor(tiles, device=DEV)].cpu().numpy().view(np.uint32)
        sc = s.tile_scale[torch.tensor(tiles, device=DEV)].cpu().numpy().view(np.uint16)
        kp = s.tile_k.cpu().numpy()
        tpr = cols // tile
        for i, t in enumerate(tiles):
            r, j = divmod(t, tpr)
            e = oracle.encode_tile_fixed(tile_input(x, tile, t), lat, slot, seed, j=j, t=t, dither=dither)
            assert e["scale"] == sc[i], (mi, t)
            assert e["k"] == (kp[t >> 1] >> (4 * (t & 1))) & 15, (mi, t)
            assert np.array_equal(e["slot"], pay[i]), (mi, t)
            st1, ref = oracle.decode_tile(e["slot"][: e["words"]], tile, lat, e["scale"], e["k"], seed, j, t, dither)
            assert st1 == 0
            got = y[r, j * tile:(j + 1) * tile].cpu().numpy().astype(np.float64)
            scale = np.abs(scipy.linalg.hadamard(tile) @ (oracle.signs(seed, j, tile) * ref)).max()
            assert np.all(np.abs(got - ref) <= 1e-5 * scale + 1e-30), (mi, t)

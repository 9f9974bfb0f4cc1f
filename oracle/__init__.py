"""CPU oracle of the HyperQuant per-tile codec -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
under ``kv_quantization_tile_b200``) never imports it and shares no code
with it.

The arithmetic lives in ``hq_oracle.c`` (plain C, one tile at a time,
binary32 where a floating-point result decides an integer, binary64 for
reconstructions).  This module compiles it with gcc when the shared object
is missing or older than the source, and wraps it with numpy.  The only
cross-tile step of the format -- the exclusive prefix sum that turns tile
word counts into offsets -- is done here with ``numpy.cumsum``.

Method sources are cited in ``hq_oracle.c`` by page title and section.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hq_oracle.c")
_SO = os.path.join(_HERE, "libhq_oracle.so")
_CFLAGS = ["-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-Wextra"]

LATTICES = {"Z": 1, "A2": 2, "D4": 4, "E8": 8}
NONFINITE, CAPACITY, CORRUPT = 1, 2, 4

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile hq_oracle.c into libhq_oracle.so next to it (gcc)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            u64, i64, i32, f32, vp = (ctypes.c_uint64, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_float, ctypes.c_void_p)
            sig = {
                "hqo_mix64": (u64, [u64]),
                "hqo_hash": (u64, [u64, u64, u64, u64]),
                "hqo_sign": (i32, [u64, u64, ctypes.c_uint32]),
                "hqo_uniform": (f32, [u64, u64, ctypes.c_uint32]),
                "hqo_fwht_f32": (None, [vp, i32]),
                "hqo_fwht_f64": (None, [vp, i32]),
                "hqo_rate_constant": (f32, [i32, f32]),
                "hqo_sumsq": (f32, [vp, i32]),
                "hqo_tile_scale": (ctypes.c_uint16, [f32, f32, vp]),
                "hqo_nearest": (None, [i32, vp, vp, vp, vp]),
                "hqo_nearest_batch": (None, [i32, vp, i64, vp, vp, vp]),
                "hqo_dither": (None, [i32, u64, u64, ctypes.c_uint32, vp]),
                "hqo_symbols": (None, [i32, vp, vp]),
                "hqo_unsymbols": (None, [i32, vp, vp]),
                "hqo_rice_cost": (u64, [vp, i32, i32]),
                "hqo_best_k": (i32, [vp, i32]),
                "hqo_pack_tile": (i32, [i32, i32, i32, vp, vp, vp, i32]),
                "hqo_unpack_tile": (i32, [i32, i32, i32, vp, i32, vp, vp]),
                "hqo_encode_tile": (i32, [vp, i32, i32, f32, u64, u64, u64, i32, vp, vp, vp, i32,
                                          vp, vp, vp]),
                "hqo_decode_tile": (i32, [vp, i32, i32, i32, ctypes.c_uint16, i32, u64, u64, u64,
                                          i32, vp]),
                "hqo_encode_tiles": (i32, [vp, i32, i64, i64, i32, i32, f32, u64, i32, i64, i64,
                                           vp, i32, vp, vp, vp]),
                "hqo_decode_tiles": (i32, [vp, u64, vp, vp, vp, i64, i64, i32, i32, u64, i32, i64,
                                           i64, vp]),
                "hqo_gemv_rows": (i32, [vp, u64, vp, vp, vp, i64, i64, i32, i32, u64, vp, i64,
                                        i64, vp]),
                "hqo_min_slot_words": (i32, [i32, i32]),
                "hqo_fixed_slot_words": (i32, [i32, i32, f32]),
                "hqo_fixed_start_rate": (f32, [i32, i32]),
                "hqo_fixed_scale": (ctypes.c_uint16, [vp, i32, i32, ctypes.c_uint16, u64, u64, u64, i32,
                                                      vp]),
                "hqo_encode_tile_fixed": (i32, [vp, i32, i32, i32, u64, u64, u64, i32, vp, vp, vp, vp,
                                                vp]),
                "hqo_encode_tiles_fixed": (i32, [vp, i32, i64, i32, i32, i32, u64, i32, i64, i64, vp, vp,
                                                 vp, vp]),
                "hqo_decode_tiles_fixed": (i32, [vp, u64, i32, vp, vp, i64, i32, i32, u64, i32, i64, i64,
                                                 vp]),
                "hqo_act_quant_i8": (None, [vp, i32, u64, u64, vp, vp]),
                "hqo_tile_points_i8": (i32, [vp, i32, i32, i32, i32, i32, vp, vp]),
                "hqo_gemm_i8_rows": (i32, [vp, u64, vp, i32, vp, vp, i64, i32, i32, vp, vp, i64, i64, i64, vp,
                                           vp]),
                "hqo_e4m3": (ctypes.c_uint8, [f32]),
                "hqo_e4m3_value": (f32, [ctypes.c_uint8]),
                "hqo_act_quant_e4m3": (None, [vp, i32, u64, u64, vp, vp]),
                "hqo_gemm_e4m3_rows": (i32, [vp, u64, vp, i32, vp, vp, i64, i32, i32, vp, vp, i64, i64, i64, vp,
                                             vp]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _lat(lattice) -> int:
    return LATTICES[lattice] if isinstance(lattice, str) else int(lattice)


# ---------------------------------------------------------------- steps
def mix64(z: int) -> int:
    return lib().hqo_mix64(z & (2**64 - 1))


def hash64(seed: int, tag: int, a: int, b: int) -> int:
    return lib().hqo_hash(seed, tag, a, b)


def signs(seed: int, j: int, n: int) -> np.ndarray:
    L = lib()
    return np.array([L.hqo_sign(seed, j, i) for i in range(n)], dtype=np.int32)


def uniform(seed: int, t: int, i: int) -> float:
    return lib().hqo_uniform(seed, t, i)


def fwht_f32(v) -> np.ndarray:
    a = np.ascontiguousarray(v, dtype=np.float32).copy()
    lib().hqo_fwht_f32(_p(a), a.size)
    return a


def fwht_f64(v) -> np.ndarray:
    a = np.ascontiguousarray(v, dtype=np.float64).copy()
    lib().hqo_fwht_f64(_p(a), a.size)
    return a


def rate_constant(lattice, bps: float) -> float:
    return lib().hqo_rate_constant(_lat(lattice), bps)


def sumsq(w) -> float:
    a = np.ascontiguousarray(w, dtype=np.float32)
    return lib().hqo_sumsq(_p(a), a.size)


def tile_scale(S: float, c: float):
    nf = ctypes.c_int(0)
    b = lib().hqo_tile_scale(S, c, ctypes.byref(nf))
    return int(b), bool(nf.value)


def nearest(lattice, x):
    """Nearest lattice point of one vector: (coset bit, integer coords, point)."""
    d = _lat(lattice)
    xa = np.ascontiguousarray(x, dtype=np.float32)
    assert xa.size == d
    c = ctypes.c_int(0)
    z = np.zeros(d, np.int32)
    pt = np.zeros(d, np.float32)
    lib().hqo_nearest(d, _p(xa), ctypes.byref(c), _p(z), _p(pt))
    return c.value, z, pt


def nearest_batch(lattice, x):
    """Nearest points of many vectors: x[count, d] -> (c[count], z[count, d], pt[count, d])."""
    d = _lat(lattice)
    xa = np.ascontiguousarray(x, dtype=np.float32).reshape(-1, d)
    cnt = xa.shape[0]
    c = np.zeros(cnt, np.int32)
    z = np.zeros((cnt, d), np.int32)
    pt = np.zeros((cnt, d), np.float32)
    lib().hqo_nearest_batch(d, _p(xa), cnt, _p(c), _p(z), _p(pt))
    return c, z, pt


def dither(lattice, seed: int, t: int, v: int) -> np.ndarray:
    d = _lat(lattice)
    out = np.zeros(d, np.float32)
    lib().hqo_dither(d, seed, t, v, _p(out))
    return out


def symbols(lattice, z) -> np.ndarray:
    d = _lat(lattice)
    za = np.ascontiguousarray(z, dtype=np.int32)
    u = np.zeros(d, np.uint32)
    lib().hqo_symbols(d, _p(za), _p(u))
    return u


def unsymbols(lattice, u) -> np.ndarray:
    d = _lat(lattice)
    ua = np.ascontiguousarray(u, dtype=np.uint32)
    z = np.zeros(d, np.int32)
    lib().hqo_unsymbols(d, _p(ua), _p(z))
    return z


def rice_cost(u, k: int) -> int:
    ua = np.ascontiguousarray(u, dtype=np.uint32)
    return lib().hqo_rice_cost(_p(ua), ua.size, k)


def best_k(u) -> int:
    ua = np.ascontiguousarray(u, dtype=np.uint32)
    return lib().hqo_best_k(_p(ua), ua.size)


def slot_words(n: int, lattice) -> int:
    """Words that always hold one oracle tile when every symbol is < 2^15
    (the cost at k = 15 bounds the chosen k's cost)."""
    d = _lat(lattice)
    coset = n // d if d in (2, 8) else 0
    return (coset + 16 * n + 31) // 32


def pack_tile(lattice, n: int, k: int, coset, u, cap_words: int | None = None) -> np.ndarray:
    d = _lat(lattice)
    cap = cap_words or slot_words(n, d) + 64
    ca = np.ascontiguousarray(coset, dtype=np.uint8)
    ua = np.ascontiguousarray(u, dtype=np.uint32)
    w = np.zeros(cap, np.uint32)
    nw = lib().hqo_pack_tile(d, n, k, _p(ca), _p(ua), _p(w), cap)
    if nw < 0:
        raise ValueError("tile does not fit")
    return w[:nw].copy()


def unpack_tile(lattice, n: int, k: int, words):
    d = _lat(lattice)
    wa = np.ascontiguousarray(words, dtype=np.uint32)
    coset = np.zeros(max(n // d, 1), np.uint8)
    u = np.zeros(n, np.uint32)
    st = lib().hqo_unpack_tile(d, n, k, _p(wa) if wa.size else 0, wa.size, _p(coset), _p(u))
    return st, coset[: n // d], u


def encode_tile(w, lattice, bps: float, seed: int, j: int = 0, t: int = 0, dither: bool = False):
    """Encode one tile; returns a dict with scale bits, k, words, z, coset, status."""
    d = _lat(lattice)
    wa = np.ascontiguousarray(w, dtype=np.float32)
    n = wa.size
    cap = slot_words(n, d) + 64
    words = np.zeros(cap, np.uint32)
    z = np.zeros(n, np.int32)
    c = np.zeros(n // d, np.uint8)
    sc = ctypes.c_uint16(0)
    kk = ctypes.c_uint8(0)
    st = ctypes.c_int(0)
    nw = lib().hqo_encode_tile(_p(wa), n, d, bps, seed, j, t, int(dither), ctypes.byref(sc),
                               ctypes.byref(kk), _p(words), cap, _p(z), _p(c), ctypes.byref(st))
    if nw < 0:
        raise ValueError("tile does not fit")
    return {"scale": int(sc.value), "k": int(kk.value), "words": words[:nw].copy(), "z": z,
            "coset": c, "status": st.value}


def decode_tile(words, n: int, lattice, scale: int, k: int, seed: int, j: int = 0, t: int = 0,
                dither: bool = False):
    d = _lat(lattice)
    wa = np.ascontiguousarray(words, dtype=np.uint32)
    out = np.zeros(n, np.float64)
    st = lib().hqo_decode_tile(_p(wa) if wa.size else 0, wa.size, n, d, scale, k, seed, j, t,
                               int(dither), _p(out))
    return st, out


# ---------------------------------------------------------------- matrices
def _as_bits(x: np.ndarray):
    """bf16 tensors arrive as uint16 bit patterns (dtype 0); float32 as-is (1)."""
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), 0
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), 1
    raise TypeError("oracle inputs are bf16 bit patterns (uint16) or float32")


def _ranges(ntiles: int, parts: int):
    parts = max(1, min(parts, ntiles))
    edges = np.linspace(0, ntiles, parts + 1).astype(np.int64)
    return [(int(a), int(b)) for a, b in zip(edges[:-1], edges[1:]) if b > a]


def encode_tiles(x, tile: int, lattice, bps: float, seed: int, dither: bool, t0: int, t1: int):
    """Encode tiles [t0, t1) of matrix x; returns (list of word arrays, scale, k, status)."""
    xa, dt = _as_bits(x)
    rows, cols = xa.shape
    d = _lat(lattice)
    sw = slot_words(tile, d)
    nt = t1 - t0
    slots = np.zeros(max(nt, 1) * sw, np.uint32)
    nw = np.zeros(max(nt, 1), np.int32)
    sc = np.zeros(max(nt, 1), np.uint16)
    kk = np.zeros(max(nt, 1), np.uint8)
    st = lib().hqo_encode_tiles(_p(xa), dt, rows, cols, tile, d, bps, seed, int(dither), t0, t1,
                                _p(slots), sw, _p(nw), _p(sc), _p(kk))
    if st < 0:
        raise ValueError("tile does not fit its slot")
    words = [slots[i * sw: i * sw + nw[i]] for i in range(nt)]
    return words, sc[:nt], kk[:nt], st


def encode(x, tile: int, lattice, bps: float, seed: int, dither: bool = False, threads: int = 1):
    """Encode a whole matrix.  Returns dict(payload, off, scale, k, status)."""
    rows, cols = x.shape
    assert cols % tile == 0
    ntiles = rows * (cols // tile)
    words, scales, ks, status = [], [], [], 0
    ranges = _ranges(ntiles, threads * 4)
    if threads > 1 and len(ranges) > 1:
        with ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(lambda r: encode_tiles(x, tile, lattice, bps, seed, dither, *r),
                                ranges))
    else:
        parts = [encode_tiles(x, tile, lattice, bps, seed, dither, *r) for r in ranges]
    for w, s, k, st in parts:
        words += w
        scales.append(s)
        ks.append(k)
        status |= st
    counts = np.array([len(w) for w in words], dtype=np.int64)
    off = np.zeros(ntiles + 1, np.int64)
    off[1:] = np.cumsum(counts)
    payload = np.concatenate(words) if words else np.zeros(0, np.uint32)
    return {"payload": payload.astype(np.uint32), "off": off.astype(np.uint32),
            "scale": np.concatenate(scales) if scales else np.zeros(0, np.uint16),
            "k": np.concatenate(ks) if ks else np.zeros(0, np.uint8), "status": status}


def decode(stream: dict, rows: int, cols: int, tile: int, lattice, seed: int,
           dither: bool = False, threads: int = 1) -> tuple[np.ndarray, int]:
    """binary64 decode of a whole stream; returns (out[rows, cols], status).
    A fixed-rate stream (a dict with a "slot" entry) goes to decode_fixed."""
    if "slot" in stream:
        return decode_fixed(stream, rows, cols, tile, lattice, seed, dither, threads)
    d = _lat(lattice)
    ntiles = rows * (cols // tile)
    out = np.zeros((rows, cols), np.float64)
    pay = np.ascontiguousarray(stream["payload"], dtype=np.uint32)
    cap = pay.size
    if pay.size == 0:
        pay = np.zeros(1, np.uint32)
    off = np.ascontiguousarray(stream["off"], dtype=np.uint32)
    sc = np.ascontiguousarray(stream["scale"], dtype=np.uint16)
    kk = np.ascontiguousarray(stream["k"], dtype=np.uint8)
    L = lib()

    def run(r):
        return L.hqo_decode_tiles(_p(pay), cap, _p(off), _p(sc) if sc.size else 0,
                                  _p(kk) if kk.size else 0, rows, cols, tile, d, seed,
                                  int(dither), r[0], r[1], _p(out))

    ranges = _ranges(ntiles, threads * 4)
    if threads > 1 and len(ranges) > 1:
        with ThreadPoolExecutor(threads) as ex:
            sts = list(ex.map(run, ranges))
    else:
        sts = [run(r) for r in ranges]
    st = 0
    for s in sts:
        st |= s
    return out, st


def gemv(stream: dict, rows: int, cols: int, tile: int, lattice, seed: int, x,
         r0: int = 0, r1: int | None = None) -> np.ndarray:
    """y[r] = sum_c w_hat[r, c] x[c] in binary64 for rows [r0, r1)."""
    d = _lat(lattice)
    r1 = rows if r1 is None else r1
    if "slot" in stream:
        W, st = decode_fixed(stream, rows, cols, tile, lattice, seed)
        if st:
            raise ValueError("corrupt stream")
        return W[r0:r1] @ np.asarray(x, dtype=np.float64)
    if "slot" in stream:
        W, st = decode_fixed(stream, rows, cols, tile, lattice, seed)
        if st:
            raise ValueError("corrupt stream")
        return W[r0:r1] @ np.asarray(x, dtype=np.float64)
    xa = np.ascontiguousarray(x, dtype=np.float64)
    y = np.zeros(max(r1 - r0, 1), np.float64)
    pay = np.ascontiguousarray(stream["payload"], dtype=np.uint32)
    off = np.ascontiguousarray(stream["off"], dtype=np.uint32)
    sc = np.ascontiguousarray(stream["scale"], dtype=np.uint16)
    kk = np.ascontiguousarray(stream["k"], dtype=np.uint8)
    st = lib().hqo_gemv_rows(_p(pay), pay.size, _p(off), _p(sc), _p(kk), rows, cols, tile, d, seed,
                             _p(xa), r0, r1, _p(y))
    if st < 0:
        raise MemoryError
    return y[: r1 - r0]


def gemm(stream: dict, rows: int, cols: int, tile: int, lattice, seed: int, X, threads: int = 1) -> np.ndarray:
    """Batched decode + matrix product in binary64: Y = X W_hat^T with W_hat the
    stream's binary64 decode (rows x cols) and X (batch x cols) -- the plain
    definition of a layer applied to a batch of activations through the
    compressed weights ([V2] decode path beside bf16 matrix products)."""
    W, st = decode(stream, rows, cols, tile, lattice, seed, threads=threads)
    if st:
        raise ValueError("corrupt stream")
    return np.asarray(X, dtype=np.float64).reshape(-1, cols) @ W.T


def kv_attention(k_stream: dict, v_stream: dict, heads: int, tokens: int, head_dim: int, lattice,
                 seed_k: int, seed_v: int, q, scale: float, threads: int = 1, group: int = 1) -> np.ndarray:
    """Batch-1 attention over a dithered compressed KV cache, in binary64:
    K and V (rows = heads * tokens, one vector per row) are decoded with their
    dither subtracted, then for query head qh (group query heads per KV head,
    qh // group its KV head h) o = softmax(scale K_h q) V_h.  The plain
    definition of the consumer of the cache's inner products (the pages' KV
    inner products stay unbiased per vector under subtractive dither)."""
    rows = heads * tokens
    K, st_k = decode(k_stream, rows, head_dim, head_dim, lattice, seed_k, dither=True, threads=threads)
    V, st_v = decode(v_stream, rows, head_dim, head_dim, lattice, seed_v, dither=True, threads=threads)
    if st_k or st_v:
        raise ValueError("corrupt stream")
    qa = np.asarray(q, dtype=np.float64).reshape(heads * group, head_dim)
    out = np.zeros((heads * group, head_dim))
    for qh in range(heads * group):
        h = qh // group
        s = scale * (K[h * tokens:(h + 1) * tokens] @ qa[qh])
        p = np.exp(s - s.max())
        out[qh] = (p / p.sum()) @ V[h * tokens:(h + 1) * tokens]
    return out


# ---------------------------------------------------------------- fixed rate
def min_slot_words(n: int, lattice) -> int:
    """Smallest fixed-rate slot: the all-zero tile's words."""
    return lib().hqo_min_slot_words(n, _lat(lattice))


def fixed_slot_words(n: int, lattice, bps: float) -> int:
    """Slot words for a total rate of bps bits per coordinate (20 bits of
    side information per tile included); -1 below the minimum slot."""
    return lib().hqo_fixed_slot_words(n, _lat(lattice), bps)


def fixed_start_rate(n: int, slot_words: int) -> float:
    return lib().hqo_fixed_start_rate(n, slot_words)


def fixed_scale(v, lattice, c0: int, budget_bits: int, seed: int, t: int = 0, dither: bool = False):
    """The fixed-rate scale search on a rotated tile v: (bf16 bits, trials)."""
    va = np.ascontiguousarray(v, dtype=np.float32)
    tr = ctypes.c_int(0)
    sb = lib().hqo_fixed_scale(_p(va), va.size, _lat(lattice), c0, budget_bits, seed, t, int(dither),
                               ctypes.byref(tr))
    return int(sb), tr.value


def coded_bits(v, lattice, scale_bits: int, seed: int = 0, t: int = 0, dither: bool = False) -> int:
    """Coded size in bits of the rotated tile v at one scale, from the
    variable-rate encoder's own steps (quantize, best k, pack length)."""
    d = _lat(lattice)
    va = np.ascontiguousarray(v, dtype=np.float32)
    n = va.size
    inv = np.float32(1.0) / np.float32(np.uint32(scale_bits << 16).view(np.float32))
    z = np.zeros(n, np.int32)
    cos = np.zeros(n // d, np.uint8)
    for q in range(n // d):
        x = va[q * d:(q + 1) * d] * inv
        if dither:
            x = (x + globals()["dither"](d, seed, t, q)).astype(np.float32)
        cos[q], z[q * d:(q + 1) * d], _ = nearest(d, x)
    u = np.concatenate([symbols(d, z[q * d:(q + 1) * d]) for q in range(n // d)])
    k = best_k(u)
    return (n // d if d in (2, 8) else 0) + rice_cost(u, k)


def encode_tile_fixed(w, lattice, slot_words: int, seed: int, j: int = 0, t: int = 0, dither: bool = False):
    """One fixed-rate tile: dict(scale, k, slot (all slot_words words), words
    (the tile's own count), trials, status)."""
    d = _lat(lattice)
    wa = np.ascontiguousarray(w, dtype=np.float32)
    slot = np.zeros(max(slot_words, 1), np.uint32)
    sc = ctypes.c_uint16(0)
    kk = ctypes.c_uint8(0)
    tr = ctypes.c_int(0)
    st = ctypes.c_int(0)
    nw = lib().hqo_encode_tile_fixed(_p(wa), wa.size, d, slot_words, seed, j, t, int(dither), ctypes.byref(sc),
                                     ctypes.byref(kk), _p(slot), ctypes.byref(tr), ctypes.byref(st))
    if nw < 0:
        raise ValueError("slot below the minimum")
    return {"scale": int(sc.value), "k": int(kk.value), "slot": slot[:slot_words], "words": nw,
            "trials": tr.value, "status": st.value}


def pack_k(k) -> np.ndarray:
    """Rice parameters two per byte: tile t in bits 4 (t mod 2) .. +3 of byte t // 2."""
    ka = np.asarray(k, dtype=np.uint8)
    out = np.zeros((ka.size + 1) // 2, np.uint8)
    out[:] = ka[0::2] & 15
    out[: ka[1::2].size] |= (ka[1::2] & 15) << 4
    return out


def unpack_k(kpack, ntiles: int) -> np.ndarray:
    kp = np.asarray(kpack, dtype=np.uint8)
    t = np.arange(ntiles)
    return ((kp[t >> 1] >> (4 * (t & 1))) & 15).astype(np.uint8)


def _encode_tiles_fixed(x, tile, lattice, slot_words, seed, dither, t0, t1):
    xa, dt = _as_bits(x)
    nt = t1 - t0
    slots = np.zeros(max(nt, 1) * slot_words, np.uint32)
    sc = np.zeros(max(nt, 1), np.uint16)
    kk = np.zeros(max(nt, 1), np.uint8)
    tr = np.zeros(max(nt, 1), np.int32)
    st = lib().hqo_encode_tiles_fixed(_p(xa), dt, xa.shape[1], tile, _lat(lattice), slot_words, seed,
                                      int(dither), t0, t1, _p(slots), _p(sc), _p(kk), _p(tr))
    if st < 0:
        raise ValueError("slot below the minimum")
    return slots[: nt * slot_words], sc[:nt], kk[:nt], tr[:nt], st


def encode_fixed(x, tile: int, lattice, slot_words: int, seed: int, dither: bool = False,
                 threads: int = 1) -> dict:
    """Fixed-rate encode of a whole matrix.  Returns dict(payload (ntiles *
    slot words), scale, k, kpack, trials, status, slot)."""
    rows, cols = x.shape
    assert cols % tile == 0
    ntiles = rows * (cols // tile)
    ranges = _ranges(ntiles, threads * 4)
    if threads > 1 and len(ranges) > 1:
        with ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(lambda r: _encode_tiles_fixed(x, tile, lattice, slot_words, seed, dither, *r),
                                ranges))
    else:
        parts = [_encode_tiles_fixed(x, tile, lattice, slot_words, seed, dither, *r) for r in ranges]
    cat = (lambda i, dt: np.concatenate([p[i] for p in parts]) if parts else np.zeros(0, dt))
    status = 0
    for p in parts:
        status |= p[4]
    k = cat(2, np.uint8)
    return {"payload": cat(0, np.uint32), "scale": cat(1, np.uint16), "k": k, "kpack": pack_k(k),
            "trials": cat(3, np.int32), "status": status, "slot": slot_words}


def decode_fixed(stream: dict, rows: int, cols: int, tile: int, lattice, seed: int, dither: bool = False,
                 threads: int = 1) -> tuple[np.ndarray, int]:
    """binary64 decode of a fixed-rate stream; k is read from its packed form."""
    d = _lat(lattice)
    ntiles = rows * (cols // tile)
    out = np.zeros((rows, cols), np.float64)
    pay = np.ascontiguousarray(stream["payload"], dtype=np.uint32)
    cap = pay.size
    if pay.size == 0:
        pay = np.zeros(1, np.uint32)
    sc = np.ascontiguousarray(stream["scale"], dtype=np.uint16)
    kk = np.ascontiguousarray(unpack_k(stream["kpack"], ntiles))
    S = int(stream["slot"])
    L = lib()

    def run(r):
        return L.hqo_decode_tiles_fixed(_p(pay), cap, S, _p(sc) if sc.size else 0, _p(kk) if kk.size else 0,
                                        cols, tile, d, seed, int(dither), r[0], r[1], _p(out))

    ranges = _ranges(ntiles, threads * 4)
    if threads > 1 and len(ranges) > 1:
        with ThreadPoolExecutor(threads) as ex:
            sts = list(ex.map(run, ranges))
    else:
        sts = [run(r) for r in ranges]
    st = 0
    for x in sts:
        st |= x
    return out, st


# ---------------------------------------------------------------- int8 product
def act_quant_i8(X, tile: int, seed: int):
    """Rotated activations quantized per (batch row, column tile): returns
    (Q int8 [batch, cols], S float32 [batch, cols // tile])."""
    xa, dt = _as_bits(np.atleast_2d(X))
    batch, cols = xa.shape
    xf = (xa.astype(np.uint32) << 16).view(np.float32) if dt == 0 else xa.astype(np.float32)
    xf = np.ascontiguousarray(xf)
    tpr = cols // tile
    Q = np.zeros((batch, cols), np.int8)
    S = np.zeros((batch, tpr), np.float32)
    L = lib()
    q = np.zeros(tile, np.int8)
    sc = ctypes.c_float(0)
    for b in range(batch):
        for j in range(tpr):
            seg = np.ascontiguousarray(xf[b, j * tile:(j + 1) * tile])
            L.hqo_act_quant_i8(_p(seg), tile, seed, j, _p(q), ctypes.byref(sc))
            Q[b, j * tile:(j + 1) * tile] = q
            S[b, j] = sc.value
    return Q, S


def tile_points_i8(words, n: int, lattice, k: int, exact: bool = True):
    """(status, doubled lattice coordinates as int8 saturated to +-127, saturated count)."""
    wa = np.ascontiguousarray(words, dtype=np.uint32)
    a = np.zeros(n, np.int8)
    sat = ctypes.c_int(0)
    st = lib().hqo_tile_points_i8(_p(wa) if wa.size else 0, wa.size, n, _lat(lattice), k, int(exact), _p(a),
                                  ctypes.byref(sat))
    return st, a, sat.value


def gemm_i8(stream: dict, rows: int, cols: int, tile: int, lattice, seed: int, X, threads: int = 1,
            r0: int = 0, r1: int | None = None):
    """The integer tensor-core product in binary64 (see hq_oracle.c) for
    weight rows [r0, r1): returns (Y [batch, r1 - r0], status, saturated
    coordinates)."""
    Q, S = act_quant_i8(X, tile, seed)
    return _lowbit_product("hqo_gemm_i8_rows", Q, S, stream, rows, cols, tile, lattice, threads, r0, r1)


def e4m3(x) -> np.ndarray:
    """OCP FP8 E4M3 bits of binary32 values (round to nearest even, saturating)."""
    xa = np.asarray(x, np.float32).ravel()
    L = lib()
    return np.array([L.hqo_e4m3(float(v)) for v in xa], np.uint8).reshape(np.shape(x))


def e4m3_value(b) -> np.ndarray:
    ba = np.asarray(b, np.uint8).ravel()
    L = lib()
    return np.array([L.hqo_e4m3_value(int(v)) for v in ba], np.float32).reshape(np.shape(b))


def act_quant_e4m3(X, tile: int, seed: int):
    """Rotated activations scaled per (batch row, column tile) to +-448 and
    rounded to E4M3: (Q bits uint8 [batch, cols], S float32 [batch, cols // tile])."""
    xa, dt = _as_bits(np.atleast_2d(X))
    batch, cols = xa.shape
    xf = np.ascontiguousarray((xa.astype(np.uint32) << 16).view(np.float32) if dt == 0 else xa.astype(np.float32))
    tpr = cols // tile
    Q = np.zeros((batch, cols), np.uint8)
    S = np.zeros((batch, tpr), np.float32)
    L = lib()
    q = np.zeros(tile, np.uint8)
    sc = ctypes.c_float(0)
    for b in range(batch):
        for j in range(tpr):
            seg = np.ascontiguousarray(xf[b, j * tile:(j + 1) * tile])
            L.hqo_act_quant_e4m3(_p(seg), tile, seed, j, _p(q), ctypes.byref(sc))
            Q[b, j * tile:(j + 1) * tile] = q
            S[b, j] = sc.value
    return Q, S


def gemm_e4m3(stream: dict, rows: int, cols: int, tile: int, lattice, seed: int, X, threads: int = 1,
              r0: int = 0, r1: int | None = None):
    """The fp8 (E4M3) tensor-core product in binary64 (see hq_oracle.c)."""
    Q, S = act_quant_e4m3(X, tile, seed)
    return _lowbit_product("hqo_gemm_e4m3_rows", Q, S, stream, rows, cols, tile, lattice, threads, r0, r1)


def _lowbit_product(fn_name, Q, S, stream, rows, cols, tile, lattice, threads, r0, r1):
    r1 = rows if r1 is None else r1
    batch = Q.shape[0]
    pay = np.ascontiguousarray(stream["payload"], dtype=np.uint32)
    cap = pay.size
    if pay.size == 0:
        pay = np.zeros(1, np.uint32)
    ntiles = rows * (cols // tile)
    if "slot" in stream:
        off, slot, kk = None, int(stream["slot"]), np.ascontiguousarray(unpack_k(stream["kpack"], ntiles))
    else:
        off, slot, kk = np.ascontiguousarray(stream["off"], np.uint32), 0, np.ascontiguousarray(stream["k"], np.uint8)
    sc = np.ascontiguousarray(stream["scale"], dtype=np.uint16)
    L = lib()

    def run(rg):
        r0, r1 = rg
        Y = np.zeros((batch, r1 - r0), np.float64)
        sat = ctypes.c_int(0)
        st = getattr(L, fn_name)(_p(pay), cap, _p(off) if off is not None else 0, slot, _p(sc), _p(kk), cols, tile,
                                 _lat(lattice), _p(Q), _p(S), batch, r0, r1, _p(Y), ctypes.byref(sat))
        return r0, r1, Y, st, sat.value

    ranges = [(a + r0, b + r0) for a, b in _ranges(r1 - r0, threads * 4)]
    if threads > 1 and len(ranges) > 1:
        with ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(run, ranges))
    else:
        parts = [run(rg) for rg in ranges]
    Y = np.zeros((batch, r1 - r0), np.float64)
    st = sat = 0
    for a, b, y, s_, n_ in parts:
        Y[:, a - r0:b - r0] = y
        st |= s_
        sat += n_
    return Y, st, sat

"""Helpers shared by the GPU parity tests: moving tensors between the CUDA
library and the oracle, and the tolerances the tests use."""
from __future__ import annotations

import math

import numpy as np
import scipy.linalg
import torch

import oracle
from kv_quantization_tile_b200 import hq

DEV = "cuda"


def host_input(x: torch.Tensor) -> np.ndarray:
    """Oracle input: bf16 as uint16 bit patterns, fp32 as float32."""
    x = x.contiguous().cpu()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view(np.uint16)
    return x.numpy().astype(np.float32)


def tile_values(xh: np.ndarray, tile: int, t: int) -> np.ndarray:
    rows, cols = xh.shape
    r, j = divmod(t, cols // tile)
    seg = xh[r, j * tile:(j + 1) * tile]
    if seg.dtype == np.uint16:
        return (seg.astype(np.uint32) << 16).view(np.float32)
    return seg.astype(np.float32)


def gpu_encode(x: torch.Tensor, tile, lat, bps, seed, dither=False):
    rows, cols = x.shape
    s = hq.alloc_stream(rows, cols, tile, lat, bps, x.device)
    ws = hq.alloc_workspace(rows, cols, tile, x.device)
    status = torch.zeros(1, dtype=torch.int32, device=x.device)
    (hq.hq_kv_encode if dither else hq.hq_encode)(x, tile, lat, bps, seed, s, ws, status)
    torch.cuda.synchronize()
    return s, int(status.item())


def fetch(s: hq.Stream) -> dict:
    off = s.tile_off.cpu().numpy().view(np.uint32)
    nw = int(off[-1])
    return {"payload": s.payload[:nw].cpu().numpy().view(np.uint32), "off": off,
            "scale": s.tile_scale.cpu().numpy().view(np.uint16), "k": s.tile_k.cpu().numpy()}


def device_stream(ref: dict, device=DEV, capacity_words=None) -> hq.Stream:
    pay = np.ascontiguousarray(ref["payload"], np.uint32)
    cap = capacity_words if capacity_words is not None else max(pay.size, 1)
    p = torch.zeros(cap, dtype=torch.int32)
    p[: pay.size] = torch.from_numpy(pay.view(np.int32))
    return hq.Stream(payload=p.to(device),
                     tile_off=torch.from_numpy(np.ascontiguousarray(ref["off"], np.uint32).view(np.int32)).to(device),
                     tile_scale=torch.from_numpy(np.ascontiguousarray(ref["scale"], np.uint16).view(np.int16)).to(device),
                     tile_k=torch.from_numpy(np.ascontiguousarray(ref["k"], np.uint8)).to(device))


def gpu_decode(s: hq.Stream, rows, cols, tile, lat, bps, seed, dither=False, dtype=torch.bfloat16):
    y = torch.empty(rows, cols, dtype=dtype, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    (hq.hq_kv_decode if dither else hq.hq_decode)(s, rows, cols, tile, lat, bps, seed, y, status)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), int(status.item())


def assert_streams_equal(g: dict, r: dict, tiles=None):
    assert np.array_equal(g["off"], r["off"]), "offsets differ"
    assert np.array_equal(g["scale"], r["scale"]), "scales differ"
    assert np.array_equal(g["k"], r["k"]), "rice parameters differ"
    if not np.array_equal(g["payload"], r["payload"]):
        bad = np.nonzero(g["payload"] != r["payload"])[0][:5]
        raise AssertionError(f"payload differs at words {bad.tolist()}")


def rotated(ref64: np.ndarray, tile: int, seed: int) -> np.ndarray:
    """v_hat = H (s_j . w_hat) per tile (inverts w_hat = s_j . H v_hat / n)."""
    rows, cols = ref64.shape
    tpr = cols // tile
    H = scipy.linalg.hadamard(tile).astype(np.float64)
    S = np.stack([oracle.signs(seed, j, tile) for j in range(tpr)]).astype(np.float64)
    return (ref64.reshape(rows, tpr, tile) * S[None]) @ H


def recon_tolerance(ref64: np.ndarray, tile: int, seed: int) -> np.ndarray:
    """Per element: 1e-5 x the tile's dequantized max-abs (Delta max|y - delta|),
    the bound on the binary32 decode's distance from the binary64 one."""
    rows, cols = ref64.shape
    vh = rotated(ref64, tile, seed)
    scale = np.abs(vh).max(axis=2, keepdims=True)
    return np.broadcast_to(1e-5 * scale, vh.shape).reshape(rows, cols).copy() + 1e-30


def bf16_neighbours(x: np.ndarray):
    """For binary64 x: the nearest bf16 value (ties to even), the two bf16
    values around x, and x's distance from their midpoint (bf16 keeps 8
    significant bits)."""
    m, e = np.frexp(x)                      # x = m 2^e, 1/2 <= |m| < 1
    a = m * 256.0
    lo, hi = np.floor(a), np.floor(a) + 1.0
    near = np.ldexp(np.rint(a), e - 8)       # rint: ties to even
    mid_dist = np.abs(a - (lo + 0.5)) * np.ldexp(1.0, e - 8)
    return near, np.ldexp(lo, e - 8), np.ldexp(hi, e - 8), mid_dist


def assert_recon_close(out: np.ndarray, ref64: np.ndarray, tile: int, seed: int, bf16_out: bool) -> int:
    """fp32 outputs: within recon_tolerance of the binary64 decode.  bf16
    outputs: equal to the binary64 decode rounded to bf16 (nearest, ties to
    even), except where a bf16 rounding midpoint lies within recon_tolerance
    of that value -- there the binary32 decode may round to any bf16 value
    between bf16_rn(ref - tol) and bf16_rn(ref + tol) (rounding is monotone):
    one of the two neighbours at a midpoint, or a small value left by
    binary32 cancellation where the exact result is near zero.  Returns the
    number of such exceptions; those away from zero (|ref| >= tol) must stay
    below 1e-2 of the elements."""
    tol = recon_tolerance(ref64, tile, seed)
    o = out.astype(np.float64)
    if not bf16_out:
        err = np.abs(o - ref64)
        if not np.all(err <= tol):
            i = np.unravel_index(np.argmax(err / tol), err.shape)
            raise AssertionError(f"reconstruction off at {i}: {out[i]} vs {ref64[i]} (tol {tol[i]})")
        return 0
    near = bf16_neighbours(ref64)[0]
    lo = bf16_neighbours(ref64 - tol)[0]
    hi = bf16_neighbours(ref64 + tol)[0]
    exact = o == near
    ok = exact | ((o >= lo) & (o <= hi))
    if not np.all(ok):
        i = np.unravel_index(np.argmax(~ok), o.shape)
        raise AssertionError(f"bf16 reconstruction at {i}: {out[i]}, want bf16_rn({ref64[i]}) = {near[i]}")
    # near zero (|ref| < tol) the binary32 rounding residue of a cancelling
    # sum is itself a representable value: counted apart, not limited
    near_zero = np.abs(ref64) < tol
    n_mid = int(np.sum(~exact & ~near_zero))
    # a wrong rounding (truncation, or rounding from a value off by more than
    # tol) already fails the interval test away from midpoints; the count
    # guards against a systematic bias at them.  Small A2 tiles reach 0.3 %:
    # their points put many outputs exactly on a bf16 midpoint in real
    # arithmetic, which binary32 and binary64 residues of the sqrt(3) terms
    # push to either side.
    assert n_mid <= 1e-2 * o.size + 1, f"{n_mid} of {o.size} outputs round across a midpoint"
    return n_mid + int(np.sum(~exact & near_zero))


def gemv_tolerance(ref: dict, rows, cols, tile, lat, seed, x: np.ndarray) -> np.ndarray:
    """fp32 error bound of sum_j (Delta_j / n) <y_j, H(s_j . x_j)>: every term
    is at most |y_i| ||x_j||_1 Delta_j / n; per row the rounding count is
    below 2 log2(n) + 16 + tiles per row."""
    w64, _ = oracle.decode(ref, rows, cols, tile, lat, seed)
    vh = np.abs(rotated(w64, tile, seed)).sum(axis=2)           # Delta_j ||y_j||_1
    xl1 = np.abs(x.reshape(cols // tile, tile)).sum(axis=1)      # ||x_j||_1
    B = (vh * xl1[None]).sum(axis=1) / tile
    K = 2 * math.log2(tile) + 16 + cols // tile
    return 2.0**-24 * K * B + 1e-30


def attention_tolerance(ks: dict, vs: dict, heads, tokens, d, lat, seed_k, seed_v, q: np.ndarray,
                        scale: float, group: int = 1) -> np.ndarray:
    """Per output element, an fp32 error bound of the GPU attention against
    the binary64 oracle, derived from the kernel's arithmetic (u = 2^-24,
    g(m) = m u / (1 - m u)):
      score s_t = scale (Delta_t / n) <y_t - delta_t, H(s_K . q)>, with
        |ds_t| <= |scale| / n (g(n+2) sum_i |z_ti||q~_i| + g(log2 n) ||q||_1 ||z_t||_1) + 3 u |s_t|
        (z_t = Delta_t (y_t - delta_t) the rotated vector, q~ its query);
      softmax weights then carry a relative error of at most
        eta = max_t |ds_t| + u (2 max_t |s_t - m| + 16)   (exp, shifts, merge),
        moving a convex combination by <= 2 e/(1-e) max_t |v_hat_ti|, e = expm1(eta);
      the rotated accumulation sum_t w_t z_t (any order, at most
        tokens + 48 + log2 n roundings deep), the division by the weight sum
        and the final transform add (2 g(M) + g(log2 n + 1)) (1/n) sum_i sum_t w_t |z_ti|."""
    u = 2.0**-24

    def g(m):
        return m * u / (1 - m * u)

    rows = heads * tokens
    K, _ = oracle.decode(ks, rows, d, d, lat, seed_k, dither=True, threads=8)
    V, _ = oracle.decode(vs, rows, d, d, lat, seed_v, dither=True, threads=8)
    H = scipy.linalg.hadamard(d).astype(np.float64)
    sk = oracle.signs(seed_k, 0, d).astype(np.float64)
    sv = oracle.signs(seed_v, 0, d).astype(np.float64)
    ZK = np.abs((K * sk) @ H)
    ZV = np.abs((V * sv) @ H)
    L = math.log2(d)
    M = tokens + 48 + L
    qa = np.asarray(q, np.float64).reshape(heads * group, d)
    tol = np.zeros((heads * group, d))
    for qh in range(heads * group):
        h = qh // group
        sl = slice(h * tokens, (h + 1) * tokens)
        qv = qa[qh]
        qt = np.abs(H @ (sk * qv))
        s = scale * (K[sl] @ qv)
        ds = abs(scale) / d * (g(d + 2) * (ZK[sl] @ qt) + g(L) * np.abs(qv).sum() * ZK[sl].sum(axis=1)) \
            + 3 * u * np.abs(s)
        m = s.max()
        eta = ds.max() + u * (2 * np.abs(s - m).max() + 16)
        e = math.expm1(eta)
        p = np.exp(s - m)
        w = p / p.sum()
        err_w = 2 * e / (1 - e) * np.abs(V[sl]).max(axis=0)
        A = (w @ ZV[sl]).sum() / d
        tol[qh] = err_w + (2 * g(M) + g(L + 1)) * A * (1 + 2 * e)
    return tol + 2.0**-100


def gpu_attention(ks: hq.Stream, vs: hq.Stream, heads, tokens, d, lat, bps_k, bps_v, seed_k, seed_v,
                  q: torch.Tensor, scale: float, group: int = 1):
    """Run hq_kv_attention; returns (out as float64 numpy, device status)."""
    out = torch.full((heads * group, d), float("nan"), dtype=torch.float32, device=DEV)
    ws = hq.alloc_attention_workspace(heads, tokens, d, group, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_kv_attention(ks, vs, heads, tokens, d, lat, bps_k, bps_v, seed_k, seed_v, q, scale, out, ws,
                       group=group, status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), int(status.item())


def assert_attention_close(out: np.ndarray, ref: np.ndarray, tol: np.ndarray):
    err = np.abs(out - ref)
    if not np.all(err <= tol):
        i = np.unravel_index(np.argmax(err / tol), err.shape)
        raise AssertionError(f"attention off at {i}: {out[i]} vs {ref[i]} (tol {tol[i]}, "
                             f"{int((err > tol).sum())} elements out)")


def gemm_tolerance(ref: dict, rows, cols, lat, seed, X: np.ndarray, tile: int = 256) -> np.ndarray:
    """Per output element, an error bound of the tensor-core batched product
    against the binary64 oracle.  Each product term A_ri B_bi uses
    A = bf16(Delta y) and B = bf16(x~) with x~ = H(s . x) from an fp32 transform
    (error <= g(log2 n) ||x_j||_1 per element): |A B - z x~| <= (2u + u^2)
    |z||x~| + (1 + u) |z| g(log2 n) ||x_j||_1 with u = 2^-8 (bf16); the fp32
    accumulation over every term (tensor-core adds bounded with 2^-23 per
    add, cols + 64 deep) adds (cols + 64) 2^-23 sum |z||x~|; all over n."""
    u, u32 = 2.0**-8, 2.0**-23
    tpr = cols // tile
    W, _ = oracle.decode(ref, rows, cols, tile, lat, seed, threads=8)
    H = scipy.linalg.hadamard(tile).astype(np.float64)
    S = np.stack([oracle.signs(seed, j, tile) for j in range(tpr)]).astype(np.float64)
    Z = np.abs((W.reshape(rows, tpr, tile) * S[None]) @ H)                    # |Delta y|
    Xa = np.asarray(X, np.float64).reshape(-1, tpr, tile)
    Xt = np.abs((Xa * S[None]) @ H)                                           # |x~|
    xl1 = np.abs(Xa).sum(axis=2)                                              # ||x_bj||_1
    dots = Xt.reshape(Xt.shape[0], -1) @ Z.reshape(rows, -1).T
    rot = xl1 @ Z.sum(axis=2).T
    L = math.log2(tile)
    g = L * 2.0**-24 / (1 - L * 2.0**-24)
    return ((2 * u + u * u + (cols + 64) * u32) * dots + (1 + u) * g * rot) / tile + 1e-30

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


def recon_tolerance(ref64: np.ndarray, tile: int, seed: int, bf16_out: bool) -> np.ndarray:
    """Per element: 1e-5 x the tile's dequantized max-abs (Delta max|y - delta|),
    plus one bf16 rounding of the reference for bf16 outputs."""
    rows, cols = ref64.shape
    vh = rotated(ref64, tile, seed)
    scale = np.abs(vh).max(axis=2, keepdims=True)
    tol = np.broadcast_to(1e-5 * scale, vh.shape).reshape(rows, cols).copy()
    if bf16_out:
        tol += np.abs(ref64) * 2.0**-8
    return tol + 1e-30


def assert_recon_close(out: np.ndarray, ref64: np.ndarray, tile: int, seed: int, bf16_out: bool):
    tol = recon_tolerance(ref64, tile, seed, bf16_out)
    err = np.abs(out.astype(np.float64) - ref64)
    if not np.all(err <= tol):
        i = np.unravel_index(np.argmax(err / tol), err.shape)
        raise AssertionError(f"reconstruction off at {i}: {out[i]} vs {ref64[i]} (tol {tol[i]})")


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

"""Thin ctypes binding of the C ABI in ``include/hq.h`` (``libhq.so``).

Names and argument order follow the C functions; this module only marshals
torch tensors to device pointers and the current CUDA stream to a
``cudaStream_t``.  Every step of the codec runs in the library's kernels.
There is no fallback: if the library is missing, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with "
                      "`python -c 'import __graft_entry__ as g; g.build()'`")

HQ_Z, HQ_A2, HQ_D4, HQ_E8 = 1, 2, 4, 8
HQ_BF16, HQ_F32 = 0, 1
HQ_OK, HQ_ERR_ARG, HQ_ERR_UNSUPPORTED, HQ_ERR_CAPACITY, HQ_ERR_WORKSPACE, HQ_ERR_CUDA, HQ_ERR_FORMAT = range(7)
HQ_ST_NONFINITE, HQ_ST_CAPACITY, HQ_ST_CORRUPT, HQ_ST_TIMEOUT, HQ_ST_RANGE = 1, 2, 4, 8, 16
LATTICES = {"Z": HQ_Z, "A2": HQ_A2, "D4": HQ_D4, "E8": HQ_E8}

EXPORTS = ["hq_error_string", "hq_version", "hq_rate_constant", "hq_tile_bound_words",
           "hq_max_payload_words", "hq_encode_workspace_bytes", "hq_encode", "hq_kv_encode",
           "hq_decode", "hq_kv_decode", "hq_decode_gemv", "hq_encode_noalloc", "hq_test_encode_stalled",
           "hq_kv_attention_workspace_bytes", "hq_kv_attention", "hq_decode_gemm_workspace_bytes",
           "hq_decode_gemm", "hq_file_bytes", "hq_file_write", "hq_file_read", "hq_test_gemm_stalled",
           "hq_min_slot_words", "hq_fixed_slot_words", "hq_encode_fixed", "hq_kv_encode_fixed",
           "hq_decode_gemm_int8_workspace_bytes", "hq_decode_gemm_int8", "hq_decode_gemm_fp8",
           "hq_stream_stats"]


class hq_file_info(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("tile", ctypes.c_int32),
                ("lattice", ctypes.c_int32), ("bps", ctypes.c_float), ("flags", ctypes.c_uint32),
                ("seed", ctypes.c_uint64), ("ntiles", ctypes.c_uint64), ("payload_words", ctypes.c_uint64),
                ("slot_words", ctypes.c_uint32)]


class hq_stream(ctypes.Structure):
    _fields_ = [("payload", ctypes.c_void_p), ("payload_capacity_words", ctypes.c_uint64),
                ("tile_off", ctypes.c_void_p), ("tile_scale", ctypes.c_void_p),
                ("tile_k", ctypes.c_void_p), ("slot_words", ctypes.c_uint32)]


_lib = ctypes.CDLL(_LIB_PATH)
_i64, _u64, _i32, _f32, _vp = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
_SIGS = {
    "hq_error_string": (ctypes.c_char_p, [_i32]),
    "hq_version": (_i32, []),
    "hq_rate_constant": (_i32, [_i32, _f32, ctypes.POINTER(_f32)]),
    "hq_tile_bound_words": (_i32, [_i32, _i32, _f32, ctypes.POINTER(ctypes.c_uint32)]),
    "hq_max_payload_words": (_i32, [_i64, _i64, _i32, _i32, _f32, ctypes.POINTER(_u64)]),
    "hq_encode_workspace_bytes": (_i32, [_i64, _i64, _i32, ctypes.POINTER(_u64)]),
    "hq_encode": (_i32, [_vp, _i32, _i64, _i64, _i32, _i32, _f32, _u64, ctypes.POINTER(hq_stream),
                         _vp, _u64, _vp, _vp]),
    "hq_kv_encode": (_i32, [_vp, _i32, _i64, _i64, _i32, _i32, _f32, _u64, ctypes.POINTER(hq_stream),
                            _vp, _u64, _vp, _vp]),
    "hq_decode": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _u64, _vp, _i32,
                         _vp, _vp]),
    "hq_kv_decode": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _u64, _vp, _i32,
                            _vp, _vp]),
    "hq_decode_gemv": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _u64, _vp, _vp,
                              _vp, _vp]),
    "hq_stream_stats": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _vp, _vp, _i32,
                               _vp, _vp]),
    "hq_encode_noalloc": (_i32, [_vp, _i32, _i64, _i64, _i32, _i32, _f32, _u64, ctypes.POINTER(hq_stream),
                                 _vp, _vp]),
    "hq_test_encode_stalled": (_i32, [_vp, _i32, _i64, _i64, _i32, _i32, _f32, _u64, ctypes.POINTER(hq_stream),
                                      _vp, _u64, _vp, _vp, ctypes.c_uint32]),
    "hq_kv_attention_workspace_bytes": (_i32, [_i64, _i64, _i32, _i32, ctypes.POINTER(_u64)]),
    "hq_decode_gemm_workspace_bytes": (_i32, [_i64, _i64, _i64, ctypes.POINTER(_u64)]),
    "hq_test_gemm_stalled": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _u64, _vp, _i64, _vp,
                                    _vp, _u64, _vp, _vp, _i64]),
    "hq_file_bytes": (_i32, [ctypes.POINTER(hq_file_info), ctypes.POINTER(_u64)]),
    "hq_file_write": (_i32, [ctypes.POINTER(hq_file_info), _vp, _vp, _vp, _vp, _vp, _u64]),
    "hq_file_read": (_i32, [_vp, _u64, ctypes.POINTER(hq_file_info), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                            ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    "hq_min_slot_words": (_i32, [_i32, _i32, ctypes.POINTER(ctypes.c_uint32)]),
    "hq_fixed_slot_words": (_i32, [_i32, _i32, _f32, ctypes.POINTER(ctypes.c_uint32)]),
    "hq_encode_fixed": (_i32, [_vp, _i32, _i64, _i64, _i32, _i32, _u64, ctypes.POINTER(hq_stream), _vp, _vp]),
    "hq_kv_encode_fixed": (_i32, [_vp, _i32, _i64, _i64, _i32, _i32, _u64, ctypes.POINTER(hq_stream), _vp, _vp]),
    "hq_decode_gemm_int8_workspace_bytes": (_i32, [_i64, _i64, _i64, ctypes.POINTER(_u64)]),
    "hq_decode_gemm_int8": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _u64, _vp, _i64, _vp, _vp,
                                   _u64, _vp, _vp]),
    "hq_decode_gemm_fp8": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _u64, _vp, _i64, _vp, _vp,
                                  _u64, _vp, _vp]),
    "hq_decode_gemm": (_i32, [ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32, _f32, _u64, _vp, _i64, _vp, _vp,
                              _u64, _vp, _vp]),
    "hq_kv_attention": (_i32, [ctypes.POINTER(hq_stream), ctypes.POINTER(hq_stream), _i64, _i64, _i32, _i32,
                               _i32, _f32, _f32, _u64, _u64, _vp, _f32, _vp, _vp, _u64, _vp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype, _fn.argtypes = _res, _args


class HQError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {hq_error_string(code)} (code {code})")
        self.code = code


def library():
    return _lib


def library_path() -> str:
    return _LIB_PATH


def _check(code: int, where: str):
    if code != HQ_OK:
        raise HQError(code, where)


def _lat(lattice) -> int:
    return LATTICES[lattice] if isinstance(lattice, str) else int(lattice)


def _ptr(t) -> int:
    if t is None:
        return 0
    return t.data_ptr()


def _stream_handle(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HQ_BF16
    if t.dtype == torch.float32:
        return HQ_F32
    raise TypeError("bf16 or fp32 tensors only")


# ----------------------------------------------------------------- sizing
def hq_error_string(code: int) -> str:
    return _lib.hq_error_string(code).decode()


def hq_version() -> int:
    return _lib.hq_version()


def hq_rate_constant(lattice, bps: float) -> float:
    out = _f32(0)
    _check(_lib.hq_rate_constant(_lat(lattice), bps, ctypes.byref(out)), "hq_rate_constant")
    return out.value


def hq_tile_bound_words(tile: int, lattice, bps: float) -> int:
    out = ctypes.c_uint32(0)
    _check(_lib.hq_tile_bound_words(tile, _lat(lattice), bps, ctypes.byref(out)), "hq_tile_bound_words")
    return out.value


def hq_max_payload_words(rows: int, cols: int, tile: int, lattice, bps: float) -> int:
    out = _u64(0)
    _check(_lib.hq_max_payload_words(rows, cols, tile, _lat(lattice), bps, ctypes.byref(out)),
           "hq_max_payload_words")
    return out.value


def hq_encode_workspace_bytes(rows: int, cols: int, tile: int) -> int:
    out = _u64(0)
    _check(_lib.hq_encode_workspace_bytes(rows, cols, tile, ctypes.byref(out)), "hq_encode_workspace_bytes")
    return out.value


# ----------------------------------------------------------------- streams
@dataclass
class Stream:
    """Device buffers of one compressed matrix (all owned by torch).
    slot_words > 0 marks a fixed-rate stream: tile t in payload words
    [t S, t S + S), no offsets (tile_off empty), k packed two per byte."""
    payload: torch.Tensor      # int32 words (bit patterns of uint32)
    tile_off: torch.Tensor     # int32, ntiles + 1 (uint32 offsets); empty for fixed rate
    tile_scale: torch.Tensor   # int16, ntiles (bf16 bits of Delta)
    tile_k: torch.Tensor       # uint8, ntiles (fixed rate: (ntiles + 1) // 2 packed bytes)
    slot_words: int = 0

    def struct(self) -> hq_stream:
        return hq_stream(_ptr(self.payload), self.payload.numel(),
                         _ptr(self.tile_off) if self.tile_off.numel() else 0,
                         _ptr(self.tile_scale) if self.tile_scale.numel() else 0,
                         _ptr(self.tile_k) if self.tile_k.numel() else 0, self.slot_words)

    def words(self) -> int:
        """Payload words actually used (variable rate: reads tile_off[-1] and synchronises)."""
        if self.slot_words:
            return self.tile_scale.numel() * self.slot_words
        return int(self.tile_off[-1].item()) & 0xFFFFFFFF

    def nbytes(self) -> int:
        """Compressed bytes: used payload words plus the per-tile headers
        (fixed rate: bf16 Delta and a 4-bit k per tile, rounded to bytes)."""
        if self.slot_words:
            return 4 * self.words() + 2 * self.tile_scale.numel() + self.tile_k.numel()
        return 4 * self.words() + 4 * self.tile_off.numel() + 2 * self.tile_scale.numel() + self.tile_k.numel()


def alloc_stream(rows: int, cols: int, tile: int, lattice, bps: float, device="cuda",
                 capacity_words: int | None = None) -> Stream:
    ntiles = rows * (cols // tile)
    cap = capacity_words if capacity_words is not None else hq_max_payload_words(rows, cols, tile, lattice, bps)
    return Stream(payload=torch.empty(max(cap, 1), dtype=torch.int32, device=device),
                  tile_off=torch.empty(ntiles + 1, dtype=torch.int32, device=device),
                  tile_scale=torch.empty(ntiles, dtype=torch.int16, device=device),
                  tile_k=torch.empty(ntiles, dtype=torch.uint8, device=device))


def hq_min_slot_words(tile: int, lattice) -> int:
    out = ctypes.c_uint32(0)
    _check(_lib.hq_min_slot_words(tile, _lat(lattice), ctypes.byref(out)), "hq_min_slot_words")
    return out.value


def hq_fixed_slot_words(tile: int, lattice, bps: float) -> int:
    out = ctypes.c_uint32(0)
    _check(_lib.hq_fixed_slot_words(tile, _lat(lattice), bps, ctypes.byref(out)), "hq_fixed_slot_words")
    return out.value


def alloc_fixed_stream(rows: int, cols: int, tile: int, slot_words: int, device="cuda") -> Stream:
    """Buffers of a fixed-rate stream with slots of slot_words words."""
    ntiles = rows * (cols // tile)
    return Stream(payload=torch.empty(max(ntiles * slot_words, 1), dtype=torch.int32, device=device),
                  tile_off=torch.empty(0, dtype=torch.int32, device=device),
                  tile_scale=torch.empty(ntiles, dtype=torch.int16, device=device),
                  tile_k=torch.empty((ntiles + 1) // 2, dtype=torch.uint8, device=device),
                  slot_words=slot_words)


def alloc_workspace(rows: int, cols: int, tile: int, device="cuda") -> torch.Tensor:
    return torch.empty(hq_encode_workspace_bytes(rows, cols, tile), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------- codec
def _encode(fn, x: torch.Tensor, tile: int, lattice, bps: float, seed: int, out: Stream,
            workspace: torch.Tensor, status: torch.Tensor | None, stream):
    assert x.is_contiguous() and x.dim() == 2
    rows, cols = x.shape
    s = out.struct()
    code = fn(_ptr(x), _dtype_code(x), rows, cols, tile, _lat(lattice), bps, seed, ctypes.byref(s),
              _ptr(workspace), workspace.numel(), _stream_handle(stream), _ptr(status))
    _check(code, fn.__name__)
    return out


def hq_encode(x, tile, lattice, bps, seed, out: Stream, workspace, status=None, stream=None) -> Stream:
    return _encode(_lib.hq_encode, x, tile, lattice, bps, seed, out, workspace, status, stream)


def hq_kv_encode(x, tile, lattice, bps, seed, out: Stream, workspace, status=None, stream=None) -> Stream:
    return _encode(_lib.hq_kv_encode, x, tile, lattice, bps, seed, out, workspace, status, stream)


def _encode_fixed(fn, x: torch.Tensor, tile: int, lattice, seed: int, out: Stream, status, stream):
    assert x.is_contiguous() and x.dim() == 2
    rows, cols = x.shape
    s = out.struct()
    _check(fn(_ptr(x), _dtype_code(x), rows, cols, tile, _lat(lattice), seed, ctypes.byref(s),
              _stream_handle(stream), _ptr(status)), fn.__name__)
    return out


def hq_encode_fixed(x, tile, lattice, seed, out: Stream, status=None, stream=None) -> Stream:
    """Fixed-rate encode into out (from alloc_fixed_stream): every tile fits
    its slot, with Delta searched per tile."""
    return _encode_fixed(_lib.hq_encode_fixed, x, tile, lattice, seed, out, status, stream)


def hq_kv_encode_fixed(x, tile, lattice, seed, out: Stream, status=None, stream=None) -> Stream:
    return _encode_fixed(_lib.hq_kv_encode_fixed, x, tile, lattice, seed, out, status, stream)


def _decode(fn, s: Stream, rows: int, cols: int, tile: int, lattice, bps: float, seed: int,
            y: torch.Tensor, status, stream):
    assert y.is_contiguous() and tuple(y.shape) == (rows, cols)
    st = s.struct()
    _check(fn(ctypes.byref(st), rows, cols, tile, _lat(lattice), bps, seed, _ptr(y), _dtype_code(y),
              _stream_handle(stream), _ptr(status)), fn.__name__)
    return y


def hq_decode(s: Stream, rows, cols, tile, lattice, bps, seed, y, status=None, stream=None):
    return _decode(_lib.hq_decode, s, rows, cols, tile, lattice, bps, seed, y, status, stream)


def hq_kv_decode(s: Stream, rows, cols, tile, lattice, bps, seed, y, status=None, stream=None):
    return _decode(_lib.hq_kv_decode, s, rows, cols, tile, lattice, bps, seed, y, status, stream)


def hq_decode_gemv(s: Stream, rows, cols, tile, lattice, bps, seed, x, y, status=None, stream=None):
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.numel() == cols
    assert y.dtype == torch.float32 and y.is_contiguous() and y.numel() == rows
    st = s.struct()
    _check(_lib.hq_decode_gemv(ctypes.byref(st), rows, cols, tile, _lat(lattice), bps, seed, _ptr(x), _ptr(y),
                               _stream_handle(stream), _ptr(status)), "hq_decode_gemv")
    return y


STATS_KEYS = ("tiles", "coset", "low", "unary", "padding", "offset_header", "scale_header", "k_header")


def hq_stream_stats(s: Stream, rows, cols, tile, lattice, bps, bins=1024, status=None, stream=None):
    """Bits by kind and the symbol histogram of a stream (device tensors:
    counts int64[8] in STATS_KEYS order, hist int64[2][bins])."""
    dev = s.payload.device
    counts = torch.empty(8, dtype=torch.int64, device=dev)
    hist = torch.empty(2, bins, dtype=torch.int64, device=dev)
    st = s.struct()
    _check(_lib.hq_stream_stats(ctypes.byref(st), rows, cols, tile, _lat(lattice), bps, _ptr(counts), _ptr(hist),
                                bins, _stream_handle(stream), _ptr(status)), "hq_stream_stats")
    return counts, hist


def _entropy_bits(counts) -> float:
    total = sum(counts)
    return -sum(c / total * math.log2(c / total) for c in counts if c) if total else 0.0


def rate_report(counts, hist, tile: int) -> dict:
    """Itemized rate of a stream from hq_stream_stats (host lists or tensors):
    bits per coordinate by kind, the empirical entropy of the symbols per
    coordinate (stripped last coordinates counted apart), and the Rice code's
    excess over it (low-part + unary bits minus that entropy)."""
    c = [int(v) for v in counts]
    h = [[int(v) for v in row] for row in hist]
    coords = c[0] * tile
    if coords == 0:
        return {"coords": 0}
    n0, n1 = sum(h[0]), sum(h[1])
    sym_entropy = (_entropy_bits(h[0]) * n0 + _entropy_bits(h[1]) * n1) / coords
    per = {k: c[i] / coords for i, k in enumerate(STATS_KEYS) if i > 0}
    rice = per["low"] + per["unary"]
    return {"coords": coords,
            "bits_per_coord": {k: round(v, 4) for k, v in per.items()},
            "payload_bits_per_coord": round(per["coset"] + rice + per["padding"], 4),
            "total_bits_per_coord": round(sum(per.values()), 4),
            "rice_bits_per_coord": round(rice, 4),
            "symbol_entropy_bits_per_coord": round(sym_entropy, 4),
            "rice_gap_bits_per_coord": round(rice - sym_entropy, 4),
            "symbols_clipped_to_last_bin": h[0][-1] + h[1][-1]}


def hq_decode_gemm_workspace_bytes(rows: int, cols: int, batch: int) -> int:
    out = _u64(0)
    _check(_lib.hq_decode_gemm_workspace_bytes(rows, cols, batch, ctypes.byref(out)), "hq_decode_gemm_workspace_bytes")
    return out.value


def alloc_gemm_workspace(rows: int, cols: int, batch: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(hq_decode_gemm_workspace_bytes(rows, cols, batch), 16), dtype=torch.uint8, device=device)


def hq_decode_gemm(s: Stream, rows, cols, tile, lattice, bps, seed, x, y, workspace, status=None, stream=None):
    """Y = X W_hat^T for bf16 activations x [batch, cols] through the stream of
    W (rows x cols, tile 256); y is fp32 [batch, rows]."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == cols
    batch = x.shape[0]
    assert y.dtype == torch.float32 and y.is_contiguous() and y.numel() == batch * rows
    st = s.struct()
    _check(_lib.hq_decode_gemm(ctypes.byref(st), rows, cols, tile, _lat(lattice), bps, seed, _ptr(x), batch, _ptr(y),
                               _ptr(workspace), workspace.numel(), _stream_handle(stream), _ptr(status)),
           "hq_decode_gemm")
    return y


def hq_decode_gemm_int8_workspace_bytes(rows: int, cols: int, batch: int) -> int:
    out = _u64(0)
    _check(_lib.hq_decode_gemm_int8_workspace_bytes(rows, cols, batch, ctypes.byref(out)),
           "hq_decode_gemm_int8_workspace_bytes")
    return out.value


def alloc_gemm_int8_workspace(rows: int, cols: int, batch: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(hq_decode_gemm_int8_workspace_bytes(rows, cols, batch), 16), dtype=torch.uint8,
                       device=device)


def hq_decode_gemm_int8(s: Stream, rows, cols, tile, lattice, bps, seed, x, y, workspace, status=None, stream=None):
    """Y = X W_hat^T on the integer tensor cores: A = 2y in int8, the rotated
    activations quantized to int8 per (row, column tile); y is fp32 [batch, rows]."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == cols
    batch = x.shape[0]
    assert y.dtype == torch.float32 and y.is_contiguous() and y.numel() == batch * rows
    st = s.struct()
    _check(_lib.hq_decode_gemm_int8(ctypes.byref(st), rows, cols, tile, _lat(lattice), bps, seed, _ptr(x), batch,
                                    _ptr(y), _ptr(workspace), workspace.numel(), _stream_handle(stream),
                                    _ptr(status)), "hq_decode_gemm_int8")
    return y


def hq_decode_gemm_fp8(s: Stream, rows, cols, tile, lattice, bps, seed, x, y, workspace, status=None, stream=None):
    """Y = X W_hat^T on the fp8 tensor cores: A = e4m3(2y), the rotated
    activations in E4M3 per (row, column tile); workspace from
    alloc_gemm_int8_workspace; y is fp32 [batch, rows]."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2 and x.shape[1] == cols
    batch = x.shape[0]
    assert y.dtype == torch.float32 and y.is_contiguous() and y.numel() == batch * rows
    st = s.struct()
    _check(_lib.hq_decode_gemm_fp8(ctypes.byref(st), rows, cols, tile, _lat(lattice), bps, seed, _ptr(x), batch,
                                   _ptr(y), _ptr(workspace), workspace.numel(), _stream_handle(stream),
                                   _ptr(status)), "hq_decode_gemm_fp8")
    return y


def hq_test_gemm_stalled(s: Stream, rows, cols, tile, lattice, bps, seed, x, y, workspace, stalled_tile: int,
                         status=None, stream=None):
    """hq_decode_gemm with one column tile's tensor-core work withheld (a
    failure-detection test hook): the bounded wait runs out and HQ_ST_TIMEOUT
    is raised."""
    st = s.struct()
    _check(_lib.hq_test_gemm_stalled(ctypes.byref(st), rows, cols, tile, _lat(lattice), bps, seed, _ptr(x), x.shape[0],
                                     _ptr(y), _ptr(workspace), workspace.numel(), _stream_handle(stream), _ptr(status),
                                     stalled_tile), "hq_test_gemm_stalled")
    return y


def hq_kv_attention_workspace_bytes(heads: int, tokens: int, head_dim: int, group: int = 1) -> int:
    out = _u64(0)
    _check(_lib.hq_kv_attention_workspace_bytes(heads, tokens, head_dim, group, ctypes.byref(out)),
           "hq_kv_attention_workspace_bytes")
    return out.value


def alloc_attention_workspace(heads: int, tokens: int, head_dim: int, group: int = 1,
                              device="cuda") -> torch.Tensor:
    return torch.empty(hq_kv_attention_workspace_bytes(heads, tokens, head_dim, group), dtype=torch.uint8,
                       device=device)


def hq_kv_attention(k: Stream, v: Stream, heads: int, tokens: int, head_dim: int, lattice, bps_k: float,
                    bps_v: float, seed_k: int, seed_v: int, q, scale: float, out, workspace, group: int = 1,
                    status=None, stream=None):
    """Batch-1 attention of q (bf16 [heads * group, head_dim]) over the KV
    streams written by hq_kv_encode; out is fp32 [heads * group, head_dim]."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.numel() == heads * group * head_dim
    assert out.dtype == torch.float32 and out.is_contiguous() and out.numel() == heads * group * head_dim
    ks, vs = k.struct(), v.struct()
    _check(_lib.hq_kv_attention(ctypes.byref(ks), ctypes.byref(vs), heads, tokens, head_dim, group,
                                _lat(lattice), bps_k, bps_v, seed_k, seed_v, _ptr(q), scale, _ptr(out),
                                _ptr(workspace), workspace.numel(), _stream_handle(stream), _ptr(status)),
           "hq_kv_attention")
    return out


def hq_encode_noalloc(x, tile, lattice, bps, seed, out: Stream, status=None, stream=None) -> Stream:
    """hq_encode without a workspace, for callers that cannot allocate device
    memory: the library keeps a fixed scratch array on each GPU instead (see
    include/hq.h for its size limit and the rule that overlapping calls on
    one GPU must be serialised)."""
    assert x.is_contiguous() and x.dim() == 2
    rows, cols = x.shape
    s = out.struct()
    _check(_lib.hq_encode_noalloc(_ptr(x), _dtype_code(x), rows, cols, tile, _lat(lattice), bps, seed,
                                  ctypes.byref(s), _stream_handle(stream), _ptr(status)), "hq_encode_noalloc")
    return out


# ----------------------------------------------------------------- files
def stream_to_bytes(s: Stream, rows: int, cols: int, tile: int, lattice, bps: float, seed: int,
                    dither: bool = False) -> bytes:
    """The checkpoint container of a stream (its arrays are copied to the host)."""
    scale = s.tile_scale.cpu().numpy().view(np.uint16)
    kk = s.tile_k.cpu().numpy()
    ntiles = rows * (cols // tile)
    if s.slot_words:
        off = None
        words = ntiles * s.slot_words
        flags = 2
    else:
        off = s.tile_off.cpu().numpy().view(np.uint32)
        words = int(off[-1])
        flags = 0
    pay = s.payload[:words].cpu().numpy().view(np.uint32)
    info = hq_file_info(rows, cols, tile, _lat(lattice), bps, flags | (1 if dither else 0), seed, ntiles, words,
                        s.slot_words)
    n = _u64(0)
    _check(_lib.hq_file_bytes(ctypes.byref(info), ctypes.byref(n)), "hq_file_bytes")
    buf = np.zeros(n.value, dtype=np.uint8)
    _check(_lib.hq_file_write(ctypes.byref(info), off.ctypes.data if off is not None else None,
                              scale.ctypes.data if scale.size else None,
                              kk.ctypes.data if kk.size else None, pay.ctypes.data if pay.size else None,
                              buf.ctypes.data, buf.size), "hq_file_write")
    return buf.tobytes()


def stream_from_bytes(data: bytes, device="cuda") -> tuple[Stream, dict]:
    """Check a container and return (device Stream, meta) with meta holding
    rows, cols, tile, lattice, bps, seed and dither."""
    buf = np.frombuffer(data, dtype=np.uint8)
    info = hq_file_info()
    ptrs = [_vp() for _ in range(4)]
    _check(_lib.hq_file_read(buf.ctypes.data, buf.size, ctypes.byref(info), *[ctypes.byref(p) for p in ptrs]),
           "hq_file_read")
    base = buf.ctypes.data
    n, words = int(info.ntiles), int(info.payload_words)

    def view(p, dtype, count):
        start = (p.value or base) - base
        return np.frombuffer(data, dtype=dtype, count=count, offset=start).copy()

    fixed = bool(info.flags & 2)
    off = np.zeros(0, np.uint32) if fixed else view(ptrs[0], np.uint32, n + 1)
    scale = view(ptrs[1], np.uint16, n)
    kk = view(ptrs[2], np.uint8, (n + 1) // 2 if fixed else n)
    pay = view(ptrs[3], np.uint32, words)
    pay_t = torch.zeros(max(words, 1), dtype=torch.int32)
    pay_t[:words] = torch.from_numpy(pay.view(np.int32))
    stream = Stream(payload=pay_t.to(device), tile_off=torch.from_numpy(off.view(np.int32)).to(device),
                    tile_scale=torch.from_numpy(scale.view(np.int16)).to(device),
                    tile_k=torch.from_numpy(kk).to(device), slot_words=int(info.slot_words))
    names = {v: k for k, v in LATTICES.items()}
    meta = {"rows": int(info.rows), "cols": int(info.cols), "tile": int(info.tile), "lattice": names[info.lattice],
            "bps": float(info.bps), "seed": int(info.seed), "dither": bool(info.flags & 1),
            "slot_words": int(info.slot_words)}
    return stream, meta


def save_stream(path: str, s: Stream, rows, cols, tile, lattice, bps, seed, dither=False) -> None:
    with open(path, "wb") as f:
        f.write(stream_to_bytes(s, rows, cols, tile, lattice, bps, seed, dither))


def load_stream(path: str, device="cuda") -> tuple[Stream, dict]:
    with open(path, "rb") as f:
        return stream_from_bytes(f.read(), device)

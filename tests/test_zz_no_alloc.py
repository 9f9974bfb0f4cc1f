"""hq_encode_noalloc -- the encoder for callers that cannot allocate device
memory (engines with their own pre-reserved pools, plug-ins inside another
framework's allocator, paths where cudaMalloc may not run).  Its scratch is a
fixed array inside the library, so it takes no workspace.

Called through the C ABI, its stream must equal hq_encode's bit for bit, on
two calls in a row (the second must not see what the first left in the
shared scratch).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from kv_quantization_tile_b200 import hq

pytestmark = pytest.mark.gpu
DEV = "cuda"


def stream_arrays(s: hq.Stream):
    off = s.tile_off.cpu().numpy().view(np.uint32)
    return (off, s.payload[: int(off[-1])].cpu().numpy(), s.tile_scale.cpu().numpy(), s.tile_k.cpu().numpy())


def encode_with_workspace(x, tile, lat, bps, seed):
    rows, cols = x.shape
    s = hq.alloc_stream(rows, cols, tile, lat, bps, DEV)
    hq.hq_encode(x, tile, lat, bps, seed, s, hq.alloc_workspace(rows, cols, tile, DEV))
    return s


def encode_without_workspace(x, tile, lat, bps, seed, status):
    """Raw C-ABI call (no Python wrapper logic in between)."""
    rows, cols = x.shape
    s = hq.alloc_stream(rows, cols, tile, lat, bps, DEV)
    st = s.struct()
    code = hq.library().hq_encode_noalloc(
        x.data_ptr(), hq.HQ_BF16, rows, cols, tile, hq.LATTICES[lat], bps, seed, ctypes.byref(st),
        torch.cuda.current_stream().cuda_stream, status.data_ptr())
    assert code == hq.HQ_OK, hq.hq_error_string(code)
    return s


def test_noalloc_encode_matches_hq_encode_on_two_calls_in_a_row():
    g = torch.Generator(device="cpu").manual_seed(123)
    cases = [(torch.randn(517, 4096, generator=g) * 0.02, 256, "E8", 4.0, 42),
             (torch.randn(3000, 128, generator=g), 128, "D4", 3.0, 7)]
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for xh, tile, lat, bps, seed in cases:
        x = xh.to(torch.bfloat16).to(DEV)
        ref = stream_arrays(encode_with_workspace(x, tile, lat, bps, seed))
        got = stream_arrays(encode_without_workspace(x, tile, lat, bps, seed, status))
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for a, b in zip(ref, got):
            assert np.array_equal(a, b)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    limit = 256 + 8 * 65536  # bytes of the library's fixed scratch array
    rows, cols = 1024, 2048
    while hq.hq_encode_workspace_bytes(rows, cols, 256) <= limit:
        rows *= 2
    s = hq.hq_stream(16, 1 << 40, 16, 16, 16)
    code = hq.library().hq_encode_noalloc(16, hq.HQ_BF16, rows, cols, 256, hq.HQ_E8, 4.0, 0,
                                          ctypes.byref(s), None, None)
    assert code == hq.HQ_ERR_UNSUPPORTED

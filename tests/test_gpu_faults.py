"""Failure detection on the GPU without a fault, trap or hang.

The encoder's only wait between thread blocks is the look-back on earlier
chunks' prefix slots, bounded by 0.5 s.  A testing hook makes one chunk
never publish its slot (a flag nothing sets): the next chunk's wait must run
out, the call must return with HQ_ST_TIMEOUT in the device status, and the
device must stay usable -- a normal encode right after is bit-exact.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from kv_quantization_tile_b200 import hq
from gpu_util import DEV, assert_streams_equal, fetch, host_input

pytestmark = pytest.mark.gpu


def test_stalled_prefix_slot_times_out_and_device_stays_usable():
    g = torch.Generator(device="cpu").manual_seed(3)
    rows, cols, tile = 400, 1024, 256  # several encode chunks
    x = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    s = hq.alloc_stream(rows, cols, tile, "E8", 4.0, DEV)
    ws = hq.alloc_workspace(rows, cols, tile, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    st = s.struct()
    t0 = time.time()
    code = hq.library().hq_test_encode_stalled(
        x.data_ptr(), hq.HQ_BF16, rows, cols, tile, hq.HQ_E8, 4.0, 42, ctypes.byref(st), ws.data_ptr(),
        ws.numel(), torch.cuda.current_stream().cuda_stream, status.data_ptr(), 0)
    assert code == hq.HQ_OK
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert int(status.item()) & hq.HQ_ST_TIMEOUT
    assert elapsed < 10.0  # bounded: one or a few 0.5 s waits
    # the context is still usable: a normal encode is bit-exact with the oracle
    status.zero_()
    hq.hq_encode(x, tile, "E8", 4.0, 42, s, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert_streams_equal(fetch(s), oracle.encode(host_input(x), tile, "E8", 4.0, 42))


def test_stalled_tensor_core_tile_times_out_and_device_stays_usable():
    """The batched product waits (bounded) on an mbarrier for each column
    tile's tensor-core products.  A testing hook withholds one tile's
    products and commit: the blocks that wait for it give up after 0.5 s,
    raise HQ_ST_TIMEOUT, free their tensor memory and return; a normal call
    right after matches the oracle."""
    from gpu_util import device_stream, gemm_tolerance
    g = torch.Generator(device="cpu").manual_seed(5)
    rows, cols = 256, 1024
    w = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16)
    ref = oracle.encode(host_input(w), 256, "E8", 4.0, 9)
    s = device_stream(ref)
    x = torch.randn(16, cols, generator=g).to(torch.bfloat16).to(DEV)
    y = torch.empty(16, rows, dtype=torch.float32, device=DEV)
    ws = hq.alloc_gemm_workspace(rows, cols, 16, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.time()
    hq.hq_test_gemm_stalled(s, rows, cols, 256, "E8", 4.0, 9, x, y, ws, 1, status)
    torch.cuda.synchronize()
    assert int(status.item()) & hq.HQ_ST_TIMEOUT
    assert time.time() - t0 < 10.0
    status.zero_()
    hq.hq_decode_gemm(s, rows, cols, 256, "E8", 4.0, 9, x, y, ws, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    X = x.float().cpu().numpy().astype(np.float64)
    want = oracle.gemm(ref, rows, cols, 256, "E8", 9, X)
    assert np.all(np.abs(y.cpu().numpy() - want) <= gemm_tolerance(ref, rows, cols, "E8", 9, X))

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

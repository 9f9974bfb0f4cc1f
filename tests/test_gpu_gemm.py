"""Batched decode + matrix product on the tensor cores (needs a B200):
Y = X W_hat^T through hq_decode_gemm against the binary64 oracle, each output
element within gpu_util.gemm_tolerance (bf16 operands, fp32 accumulation).
Shapes cover ragged row blocks, batches below, at and across the block's
batch rows, split column tiles, every lattice, and the full Llama gate."""
import numpy as np
import pytest
import torch

import oracle
from kv_quantization_tile_b200 import hq, workloads
from gpu_util import DEV, device_stream, fetch, gemm_tolerance, gpu_encode, host_input

pytestmark = pytest.mark.gpu


def weights(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, cols, generator=g) * 0.02
    w[:, seed % cols] *= 15.0
    return w.to(torch.bfloat16)


def acts(batch, cols, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(batch, cols, generator=g).to(torch.bfloat16)


def run_gemm(s, rows, cols, lat, bps, seed, x):
    y = torch.full((x.shape[0], rows), float("nan"), dtype=torch.float32, device=DEV)
    ws = hq.alloc_gemm_workspace(rows, cols, x.shape[0], DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_decode_gemm(s, rows, cols, 256, lat, bps, seed, x.to(DEV), y, ws, st)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), int(st.item())


def check(ref, rows, cols, lat, bps, seed, x, s=None):
    s = s if s is not None else device_stream(ref)
    out, st = run_gemm(s, rows, cols, lat, bps, seed, x)
    assert st == 0
    X = x.float().numpy().astype(np.float64)
    want = oracle.gemm(ref, rows, cols, 256, lat, seed, X, threads=8)
    tol = gemm_tolerance(ref, rows, cols, lat, seed, X)
    err = np.abs(out - want)
    if not np.all(err <= tol):
        i = np.unravel_index(np.argmax(err / tol), err.shape)
        raise AssertionError(f"y{i}: {out[i]} vs {want[i]} (tol {tol[i]}, {int((err > tol).sum())} out)")
    return out, want


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("batch", [1, 5, 16, 17, 40, 64, 100])
def test_gemm_matches_oracle(lat, batch):
    rows, cols = 200, 1280
    w = weights(rows, cols, 3)
    ref = oracle.encode(host_input(w), 256, lat, 4.0, 7)
    check(ref, rows, cols, lat, 4.0, 7, acts(batch, cols, batch))


@pytest.mark.parametrize("rows,cols,batch", [(128, 256, 3), (1, 512, 9), (333, 256, 70), (129, 4096, 33),
                                            (200, 512, 200), (130, 768, 300)])
def test_gemm_shapes(rows, cols, batch):
    w = weights(rows, cols, rows)
    ref = oracle.encode(host_input(w), 256, "E8", 4.0, 5)
    check(ref, rows, cols, "E8", 4.0, 5, acts(batch, cols, 1))


def test_gemm_rates():
    rows, cols = 150, 768
    w = weights(rows, cols, 8)
    for bps in (1.5, 6.0, 8.0):
        ref = oracle.encode(host_input(w), 256, "E8", bps, 2)
        check(ref, rows, cols, "E8", bps, 2, acts(24, cols, 4))


def test_gemm_batch_one_agrees_with_gemv():
    rows, cols = 300, 1024
    w = weights(rows, cols, 4)
    ref = oracle.encode(host_input(w), 256, "E8", 4.0, 1)
    x = acts(1, cols, 6)
    out, want = check(ref, rows, cols, "E8", 4.0, 1, x)
    g = oracle.gemv(ref, rows, cols, 256, "E8", 1, x.float().numpy()[0].astype(np.float64))
    assert np.allclose(want[0], g, rtol=1e-12, atol=1e-12)


def test_gemm_empty_and_corrupt():
    rows, cols = 64, 512
    w = weights(rows, cols, 9)
    ref = oracle.encode(host_input(w), 256, "E8", 4.0, 3)
    s = device_stream(ref)
    y = torch.zeros(0, rows, dtype=torch.float32, device=DEV)
    ws = torch.empty(16, dtype=torch.uint8, device=DEV)
    hq.hq_decode_gemm(s, rows, cols, 256, "E8", 4.0, 3, torch.zeros(0, cols, dtype=torch.bfloat16, device=DEV), y, ws)
    bad = {k: np.array(v, copy=True) for k, v in ref.items() if k in ("payload", "off", "scale", "k")}
    bad["k"][5] = 16
    out, st = run_gemm(device_stream(bad), rows, cols, "E8", 4.0, 3, acts(8, cols, 2))
    assert st == hq.HQ_ST_CORRUPT
    assert np.all(np.isfinite(out))


def test_gemm_repeatable():
    rows, cols = 256, 2048
    ref = oracle.encode(host_input(weights(rows, cols, 1)), 256, "E8", 4.0, 4)
    s = device_stream(ref)
    x = acts(48, cols, 3)
    a, _ = run_gemm(s, rows, cols, "E8", 4.0, 4, x)
    b, _ = run_gemm(s, rows, cols, "E8", 4.0, 4, x)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("batch", [16, 64])
def test_gemm_full_size_gate(batch):
    """The Llama-3.1-8B gate projection (14336 x 4096), GPU-encoded, against
    the oracle on the whole output."""
    w1, _, _, _ = workloads.gemv_case(DEV)
    rows, cols = w1.shape
    s, st = gpu_encode(w1, 256, "E8", 4.0, 42)
    assert st == 0
    check(fetch(s), rows, cols, "E8", 4.0, 42, acts(batch, cols, 11), s=s)

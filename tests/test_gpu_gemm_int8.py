"""Integer tensor-core product (hq_decode_gemm_int8) against the CPU oracle
(needs a B200).

The quantized activations Q and their scales, read back from the workspace,
are bit-exact with the oracle's (the binary32 rotation and the int8
rounding are decided identically).  Y is compared with the oracle's binary64
product within the fp32 bound of the epilogue: every column tile's term
Delta s / (2 n) (A . q) -- the int32 sum is exact -- takes two roundings,
and the sum over column tiles (and split-K partials) one per add:
|Y_gpu - Y_ref| <= (tiles per row + 8) 2^-24 sum_j |term_j|.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from kv_quantization_tile_b200 import hq, workloads
from gpu_util import DEV, host_input

pytestmark = pytest.mark.gpu
N = 256


def make(rows, cols, seed, scale=0.02):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(rows, cols, generator=g) * scale
    w[:, seed % cols] *= 20.0
    return w.to(torch.bfloat16).to(DEV)


def term_sums(ref, rows, cols, lat, seed, X):
    """sum_j |Delta s / (2 n) (A . q)| per (b, r), from the decoded, rotated weights."""
    W, _ = oracle.decode(ref, rows, cols, N, lat, seed, threads=8)
    tpr = cols // N
    H = scipy.linalg.hadamard(N).astype(np.float64)
    S = np.stack([oracle.signs(seed, j, N) for j in range(tpr)]).astype(np.float64)
    Z = (W.reshape(rows, tpr, N) * S[None]) @ H                          # Delta y per tile
    Q, SX = oracle.act_quant_i8(X, N, seed)
    Xq = Q.reshape(-1, tpr, N).astype(np.float64) * SX[:, :, None]       # s q per tile
    T = np.einsum("btk,rtk->brt", Xq, Z) / N
    return np.abs(T).sum(axis=2)


def run_gpu(s, rows, cols, lat, seed, X, bps=4.0):
    batch = X.shape[0]
    y = torch.full((batch, rows), float("nan"), dtype=torch.float32, device=DEV)
    ws = hq.alloc_gemm_int8_workspace(rows, cols, batch, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    hq.hq_decode_gemm_int8(s, rows, cols, N, lat, bps, seed, X, y, ws, st)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), int(st.item()), ws


def check(s, ref, rows, cols, lat, seed, X, bps=4.0, want_status=0):
    Xh = host_input(X)
    y, st, ws = run_gpu(s, rows, cols, lat, seed, X, bps)
    assert st == want_status
    Y, ost, sat = oracle.gemm_i8(ref, rows, cols, N, lat, seed, Xh, threads=8)
    assert (ost == 0) and ((sat > 0) == bool(want_status & hq.HQ_ST_RANGE))
    tol = (cols // N + 8) * 2.0**-24 * term_sums(ref, rows, cols, lat, seed, Xh) + 1e-30
    err = np.abs(y - Y)
    assert np.all(err <= tol), float(np.max(err / tol))
    # the quantized activations and their scales, read back from the workspace
    batch = X.shape[0]
    Q, SX = oracle.act_quant_i8(Xh, N, seed)
    wsn = ws.cpu().numpy()
    q = wsn[: batch * cols].view(np.int8).reshape(batch, cols)
    assert np.array_equal(q, Q)
    nb = 16 if batch <= 16 else 32 if batch <= 32 else 64
    pad = (batch + nb - 1) // nb * nb
    so = (pad * cols + 255) // 256 * 256
    sx = wsn[so: so + pad * (cols // N) * 4].view(np.float32).reshape(pad, cols // N)[:batch]
    assert np.array_equal(sx, SX)


@pytest.mark.parametrize("lat", ["E8", "D4", "Z"])
@pytest.mark.parametrize("batch", [1, 16, 37, 100])
def test_int8_product(lat, batch):
    rows, cols, seed = 203, 1024, 5
    w = make(rows, cols, 3)
    ref = oracle.encode(host_input(w), N, lat, 4.0, seed, threads=8)
    from gpu_util import device_stream
    g = torch.Generator().manual_seed(batch)
    X = torch.randn(batch, cols, generator=g).to(torch.bfloat16).to(DEV)
    check(device_stream(ref), ref, rows, cols, lat, seed, X)


def test_int8_product_on_a_fixed_rate_stream():
    rows, cols, seed, lat = 130, 1536, 8, "E8"
    w = make(rows, cols, 9)
    slot = hq.hq_fixed_slot_words(N, lat, 4.0)
    ref = oracle.encode_fixed(host_input(w), N, lat, slot, seed)
    s = hq.Stream(payload=torch.from_numpy(ref["payload"].view(np.int32).copy()).to(DEV),
                  tile_off=torch.empty(0, dtype=torch.int32, device=DEV),
                  tile_scale=torch.from_numpy(ref["scale"].view(np.int16).copy()).to(DEV),
                  tile_k=torch.from_numpy(ref["kpack"].copy()).to(DEV), slot_words=slot)
    X = torch.randn(24, cols, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).to(DEV)
    check(s, ref, rows, cols, lat, seed, X)


def test_int8_saturation_is_flagged_and_matches_the_oracle():
    rows, cols, seed, lat = 64, 512, 4, "Z"
    w = make(rows, cols, 1, scale=1.0)
    ref = oracle.encode(host_input(w), N, lat, 8.0, seed)  # 8 bps: |2y| far above 127
    from gpu_util import device_stream
    X = torch.randn(16, cols, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).to(DEV)
    check(device_stream(ref), ref, rows, cols, lat, seed, X, bps=8.0, want_status=hq.HQ_ST_RANGE)


def test_int8_refuses_a2_and_handles_empty():
    rows, cols = 32, 512
    s = hq.alloc_stream(rows, cols, N, "A2", 4.0, DEV)
    X = torch.zeros(4, cols, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(4, rows, dtype=torch.float32, device=DEV)
    with pytest.raises(hq.HQError) as e:
        hq.hq_decode_gemm_int8(s, rows, cols, N, "A2", 4.0, 1, X, y, hq.alloc_gemm_int8_workspace(rows, cols, 4, DEV))
    assert e.value.code == hq.HQ_ERR_UNSUPPORTED
    # zero activations: zero output
    w = make(rows, cols, 2)
    s = hq.alloc_stream(rows, cols, N, "E8", 4.0, DEV)
    hq.hq_encode(w, N, "E8", 4.0, 1, s, hq.alloc_workspace(rows, cols, N, DEV))
    out, st, _ = run_gpu(s, rows, cols, "E8", 1, X)
    assert st == 0 and not out.any()


def test_int8_full_size_gate_sampled_rows():
    """The Llama gate projection (14336 x 4096) at batch 16 in the launch
    configuration the benchmark times; rows sampled across the matrix
    against the oracle's product of the same rows."""
    lat, seed = "E8", 42
    w = dict(workloads.llama_layer(DEV, names=["gate"]))["gate"]
    rows, cols = w.shape
    s = hq.alloc_stream(rows, cols, N, lat, 4.0, DEV)
    hq.hq_encode(w, N, lat, 4.0, seed, s, hq.alloc_workspace(rows, cols, N, DEV))
    X = torch.randn(16, cols, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16).to(DEV)
    y, st, _ = run_gpu(s, rows, cols, lat, seed, X)
    assert st == 0
    off = s.tile_off.cpu().numpy().view(np.uint32)
    ref = {"payload": s.payload[: int(off[-1])].cpu().numpy().view(np.uint32), "off": off,
           "scale": s.tile_scale.cpu().numpy().view(np.uint16), "k": s.tile_k.cpu().numpy()}
    Xh = host_input(X)
    for r0 in (0, 127, 7000, rows - 9):
        Y, ost, sat = oracle.gemm_i8(ref, rows, cols, N, lat, seed, Xh, r0=r0, r1=r0 + 9)
        assert ost == 0 and sat == 0
        scale = np.abs(Y).max()
        assert np.allclose(y[:, r0:r0 + 9], Y, rtol=0, atol=(cols // N + 8) * 2.0**-24 * 40 * scale + 1e-30)

"""8-bit tensor-core products (hq_decode_gemm_int8, and hq_decode_gemm_fp8
with E4M3 operands) against the CPU oracle (needs a B200).

The quantized activations Q and their scales, read back from the workspace,
are bit-exact with the oracle's (the binary32 rotation and the int8
rounding are decided identically).  Y is compared with the oracle's binary64
product within the fp32 bound of the epilogue: every column tile's term
Delta s / (2 n) (A . q) -- the int32 sum is exact -- takes two roundings,
and the sum over column tiles (and split-K partials) one per add:
|Y_gpu - Y_ref| <= (tiles per row + 8) 2^-24 sum_j |term_j|.  The fp8
variant's in-tile sums of E4M3 products are formed by the tensor cores in an
undocumented internal precision: its bound adds 2^-16 of the element-wise
absolute sums (a layout or format error is orders of magnitude above it).
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


FMTS = {"int8": (oracle.act_quant_i8, oracle.gemm_i8, "hq_decode_gemm_int8"),
        "fp8": (oracle.act_quant_e4m3, oracle.gemm_e4m3, "hq_decode_gemm_fp8")}


def term_sums(ref, rows, cols, lat, seed, X, fmt):
    """Per (b, r): sum_j |Delta s / (2 n) (A . q)| and the element-wise sum
    sum_j sum_i |Delta s / (2 n) A_i q_i|, from the decoded, rotated weights
    (E4M3 rounds A by at most 2^-4 relative: a 1.07 margin covers it)."""
    W, _ = oracle.decode(ref, rows, cols, N, lat, seed, threads=8)
    tpr = cols // N
    H = scipy.linalg.hadamard(N).astype(np.float64)
    S = np.stack([oracle.signs(seed, j, N) for j in range(tpr)]).astype(np.float64)
    Z = (W.reshape(rows, tpr, N) * S[None]) @ H                          # Delta y per tile
    Q, SX = FMTS[fmt][0](X, N, seed)
    qv = oracle.e4m3_value(Q).astype(np.float64) if fmt == "fp8" else Q.astype(np.float64)
    Xq = qv.reshape(-1, tpr, N) * SX[:, :, None]                         # s q per tile
    T = np.einsum("btk,rtk->brt", Xq, Z) / N
    Tabs = np.einsum("btk,rtk->brt", np.abs(Xq), np.abs(Z)) / N
    m = 1.07 if fmt == "fp8" else 1.0
    return m * np.abs(T).sum(axis=2), m * Tabs.sum(axis=2)


def run_gpu(s, rows, cols, lat, seed, X, bps=4.0, fmt="int8"):
    batch = X.shape[0]
    y = torch.full((batch, rows), float("nan"), dtype=torch.float32, device=DEV)
    ws = hq.alloc_gemm_int8_workspace(rows, cols, batch, DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    getattr(hq, FMTS[fmt][2])(s, rows, cols, N, lat, bps, seed, X, y, ws, st)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64), int(st.item()), ws


def check(s, ref, rows, cols, lat, seed, X, bps=4.0, want_status=0, fmt="int8"):
    Xh = host_input(X)
    y, st, ws = run_gpu(s, rows, cols, lat, seed, X, bps, fmt)
    assert st == want_status
    Y, ost, sat = FMTS[fmt][1](ref, rows, cols, N, lat, seed, Xh, threads=8)
    assert (ost == 0) and ((sat > 0) == bool(want_status & hq.HQ_ST_RANGE))
    tsum, tabs = term_sums(ref, rows, cols, lat, seed, Xh, fmt)
    tol = (cols // N + 8) * 2.0**-24 * tsum + 1e-30
    if fmt == "fp8":  # the tensor cores' internal accumulation of E4M3 products
        tol = tol + 2.0**-16 * tabs
    err = np.abs(y - Y)
    assert np.all(err <= tol), float(np.max(err / tol))
    # the quantized activations and their scales, read back from the workspace
    batch = X.shape[0]
    Q, SX = FMTS[fmt][0](Xh, N, seed)
    wsn = ws.cpu().numpy()
    q = wsn[: batch * cols].view(Q.dtype).reshape(batch, cols)
    assert np.array_equal(q, Q)
    nb = 16 if batch <= 16 else 32 if batch <= 32 else 64 if batch <= 64 else 128
    pad = (batch + nb - 1) // nb * nb
    so = (pad * cols + 255) // 256 * 256
    sx = wsn[so: so + pad * (cols // N) * 4].view(np.float32).reshape(pad, cols // N)[:batch]
    assert np.array_equal(sx, SX)


@pytest.mark.parametrize("lat", ["E8", "D4", "Z"])
@pytest.mark.parametrize("batch", [1, 16, 37, 100, 150])
@pytest.mark.parametrize("fmt", ["int8", "fp8"])
def test_int8_product(lat, batch, fmt):
    rows, cols, seed = 203, 1024, 5
    w = make(rows, cols, 3)
    ref = oracle.encode(host_input(w), N, lat, 4.0, seed, threads=8)
    from gpu_util import device_stream
    g = torch.Generator().manual_seed(batch)
    X = torch.randn(batch, cols, generator=g).to(torch.bfloat16).to(DEV)
    check(device_stream(ref), ref, rows, cols, lat, seed, X, fmt=fmt)


@pytest.mark.parametrize("fmt", ["int8", "fp8"])
def test_int8_product_on_a_fixed_rate_stream(fmt):
    rows, cols, seed, lat = 130, 1536, 8, "E8"
    w = make(rows, cols, 9)
    slot = hq.hq_fixed_slot_words(N, lat, 4.0)
    ref = oracle.encode_fixed(host_input(w), N, lat, slot, seed)
    s = hq.Stream(payload=torch.from_numpy(ref["payload"].view(np.int32).copy()).to(DEV),
                  tile_off=torch.empty(0, dtype=torch.int32, device=DEV),
                  tile_scale=torch.from_numpy(ref["scale"].view(np.int16).copy()).to(DEV),
                  tile_k=torch.from_numpy(ref["kpack"].copy()).to(DEV), slot_words=slot)
    X = torch.randn(24, cols, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).to(DEV)
    check(s, ref, rows, cols, lat, seed, X, fmt=fmt)


@pytest.mark.parametrize("fmt", ["int8", "fp8"])
def test_int8_saturation_is_flagged_and_matches_the_oracle(fmt):
    rows, cols, seed, lat = 64, 512, 4, "Z"
    w = make(rows, cols, 1, scale=1.0)
    ref = oracle.encode(host_input(w), N, lat, 8.0, seed)  # 8 bps: |2y| far above 127 (and 448)
    from gpu_util import device_stream
    X = torch.randn(16, cols, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).to(DEV)
    check(device_stream(ref), ref, rows, cols, lat, seed, X, bps=8.0, want_status=hq.HQ_ST_RANGE, fmt=fmt)


def test_int8_refuses_a2_and_handles_empty():
    rows, cols = 32, 512
    s = hq.alloc_stream(rows, cols, N, "A2", 4.0, DEV)
    X = torch.zeros(4, cols, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(4, rows, dtype=torch.float32, device=DEV)
    for fn in (hq.hq_decode_gemm_int8, hq.hq_decode_gemm_fp8):
        with pytest.raises(hq.HQError) as e:
            fn(s, rows, cols, N, "A2", 4.0, 1, X, y, hq.alloc_gemm_int8_workspace(rows, cols, 4, DEV))
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

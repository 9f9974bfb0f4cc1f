"""Batch-1 attention over the dithered compressed KV cache (needs a B200):
the CUDA kernel through the C ABI against the binary64 oracle
(softmax(scale K_hat q) V_hat per query head, K_hat and V_hat the oracle's own
dithered decode), each output element within the fp32 bound derived in
gpu_util.attention_tolerance.  Streams come from the oracle's encoder, so the
attention kernel is checked on its own; one case runs the GPU encoder first.
Shapes cover several token splits with a ragged last split, grouped queries
that fill and do not fill a block, and more splits than one merge pass."""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_quantization_tile_b200 import hq, workloads
from gpu_util import (DEV, assert_attention_close, attention_tolerance, device_stream, fetch, gpu_attention,
                      gpu_encode, host_input)

pytestmark = pytest.mark.gpu


def kv_case(heads, tokens, d, seed):
    """K with a per-channel spread (as in key caches), V plain Gaussian, both
    bf16 bit patterns; queries drawn by the caller."""
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((heads, tokens, d)) * np.exp2(rng.uniform(-2, 3, (heads, 1, d)))
    V = rng.standard_normal((heads, tokens, d))
    to_bf16 = lambda a: host_input(torch.from_numpy(a.reshape(heads * tokens, d)).to(torch.bfloat16))
    return to_bf16(K), to_bf16(V)


def queries(heads, group, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(heads * group, d, generator=g).to(torch.bfloat16)


def run_case(heads, tokens, d, lat, bps_k, bps_v, group, seed=0, scale=None):
    Kh, Vh = kv_case(heads, tokens, d, seed)
    sk, sv = 100 + seed, 200 + seed
    ks = oracle.encode(Kh, d, lat, bps_k, sk, dither=True, threads=8)
    vs = oracle.encode(Vh, d, lat, bps_v, sv, dither=True, threads=8)
    q = queries(heads, group, d, seed)
    scale = 1 / math.sqrt(d) if scale is None else scale
    qf = q.float().numpy().astype(np.float64)
    ref = oracle.kv_attention(ks, vs, heads, tokens, d, lat, sk, sv, qf, scale, threads=8, group=group)
    out, st = gpu_attention(device_stream(ks), device_stream(vs), heads, tokens, d, lat, bps_k, bps_v, sk, sv,
                            q.to(DEV), scale, group)
    assert st == 0
    tol = attention_tolerance(ks, vs, heads, tokens, d, lat, sk, sv, qf, scale, group)
    assert_attention_close(out, ref, tol)
    return out, ref, tol


@pytest.mark.parametrize("lat", ["E8", "D4", "A2", "Z"])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("group", [1, 4])
def test_attention_matches_oracle(lat, d, group):
    run_case(2, 701, d, lat, 4.0, 3.0, group, seed=d + group)


@pytest.mark.parametrize("group", [2, 3, 8, 11])
def test_grouped_query_shapes(group):
    """Query chunks that fill a block, leave it ragged, and span two blocks."""
    run_case(3, 333, 128, "E8", 4.0, 4.0, group, seed=group)


def test_more_splits_than_one_merge_pass():
    """One head, one query, 40000 tokens: more than 256 token splits, so the
    merge of the last block runs over several chunks of split factors."""
    out, ref, tol = run_case(1, 40000, 64, "E8", 4.0, 4.0, 1, seed=7)
    assert out.shape == (1, 64)


def test_single_token_returns_its_value_vector():
    heads, d = 3, 128
    Kh, Vh = kv_case(heads, 1, d, 5)
    ks = oracle.encode(Kh, d, "E8", 4.0, 1, dither=True)
    vs = oracle.encode(Vh, d, "E8", 4.0, 2, dither=True)
    V, _ = oracle.decode(vs, heads, d, d, "E8", 2, dither=True)
    q = queries(heads, 2, d, 5)
    out, st = gpu_attention(device_stream(ks), device_stream(vs), heads, 1, d, "E8", 4.0, 4.0, 1, 2, q.to(DEV),
                            0.1, group=2)
    assert st == 0
    ref = np.repeat(V, 2, axis=0)
    assert np.all(np.abs(out - ref) <= 1e-5 * np.abs(ref).max(axis=1, keepdims=True))


def test_zero_tokens_and_zero_heads():
    d = 128
    empty = hq.alloc_stream(0, d, d, "E8", 4.0, DEV)
    empty.tile_off.zero_()
    q = torch.zeros(2 * 4 * d, dtype=torch.bfloat16, device=DEV)
    out = torch.full((2 * 4, d), 7.0, device=DEV)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    hq.hq_kv_attention(empty, empty, 2, 0, d, "E8", 4.0, 4.0, 1, 2, q, 0.1, out, ws, group=4)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    hq.hq_kv_attention(empty, empty, 0, 0, d, "E8", 4.0, 4.0, 1, 2, q[:0], 0.1, out[:0], ws, group=4)


def test_zero_vectors_and_extreme_scale():
    """All-zero cached keys score 0 exactly; a large negative scale makes the
    softmax nearly one-hot on the most negative score."""
    heads, tokens, d = 2, 300, 64
    Kh, Vh = kv_case(heads, tokens, d, 9)
    Kh[::7] = 0  # zero rows (bf16 +0 bit patterns)
    sk, sv = 3, 4
    ks = oracle.encode(Kh, d, "D4", 5.0, sk, dither=True)
    vs = oracle.encode(Vh, d, "D4", 5.0, sv, dither=True)
    assert np.all(ks["scale"][::7] == 0)
    q = queries(heads, 1, d, 9)
    qf = q.float().numpy().astype(np.float64)
    for scale in (0.125, -3.0):
        ref = oracle.kv_attention(ks, vs, heads, tokens, d, "D4", sk, sv, qf, scale)
        out, st = gpu_attention(device_stream(ks), device_stream(vs), heads, tokens, d, "D4", 5.0, 5.0, sk, sv,
                                q.to(DEV), scale)
        assert st == 0
        assert_attention_close(out, ref, attention_tolerance(ks, vs, heads, tokens, d, "D4", sk, sv, qf, scale))


def test_end_to_end_from_gpu_encoder():
    """GPU KV encode (bit-exact against the oracle's) feeding GPU attention."""
    heads, tokens, d, group = 4, 1500, 128, 4
    k, v = workloads.kv_layer("cpu", tokens=tokens)
    k, v = k[: heads * tokens].to(DEV), v[: heads * tokens].to(DEV)
    gk, st1 = gpu_encode(k, d, "E8", 4.0, 11, dither=True)
    gv, st2 = gpu_encode(v, d, "E8", 4.0, 12, dither=True)
    assert st1 == 0 and st2 == 0
    fk, fv = fetch(gk), fetch(gv)
    q = queries(heads, group, d, 1)
    qf = q.float().numpy().astype(np.float64)
    scale = 1 / math.sqrt(d)
    ref = oracle.kv_attention(fk, fv, heads, tokens, d, "E8", 11, 12, qf, scale, threads=8, group=group)
    out, st = gpu_attention(gk, gv, heads, tokens, d, "E8", 4.0, 4.0, 11, 12, q.to(DEV), scale, group)
    assert st == 0
    assert_attention_close(out, ref, attention_tolerance(fk, fv, heads, tokens, d, "E8", 11, 12, qf, scale, group))


def test_corrupt_tile_is_flagged():
    heads, tokens, d = 1, 200, 128
    Kh, Vh = kv_case(heads, tokens, d, 2)
    ks = oracle.encode(Kh, d, "E8", 4.0, 1, dither=True)
    vs = oracle.encode(Vh, d, "E8", 4.0, 2, dither=True)
    bad = {k: np.array(val, copy=True) for k, val in vs.items() if k in ("payload", "off", "scale", "k")}
    bad["k"][17] = 16
    q = queries(heads, 1, d, 2)
    out, st = gpu_attention(device_stream(ks), device_stream(bad), heads, tokens, d, "E8", 4.0, 4.0, 1, 2,
                            q.to(DEV), 0.1)
    assert st == hq.HQ_ST_CORRUPT
    assert np.all(np.isfinite(out))


def test_repeat_calls_are_bitwise_identical():
    heads, tokens, d, group = 2, 5000, 128, 4
    Kh, Vh = kv_case(heads, tokens, d, 4)
    ks = device_stream(oracle.encode(Kh, d, "E8", 4.0, 1, dither=True, threads=8))
    vs = device_stream(oracle.encode(Vh, d, "E8", 4.0, 2, dither=True, threads=8))
    q = queries(heads, group, d, 4).to(DEV)
    a, _ = gpu_attention(ks, vs, heads, tokens, d, "E8", 4.0, 4.0, 1, 2, q, 0.09, group)
    b, _ = gpu_attention(ks, vs, heads, tokens, d, "E8", 4.0, 4.0, 1, 2, q, 0.09, group)
    assert np.array_equal(a, b)


def test_full_size_llama_kv_layer():
    """The Llama-3.1-8B decode step's cache: 8 KV heads x 32768 tokens x 128,
    4 query heads per KV head, E8 at 4 bps, in the launch configuration the
    benchmark times; the whole output against the oracle."""
    heads, tokens, d, group = workloads.KV_HEADS, workloads.KV_TOKENS, workloads.KV_HEAD_DIM, 4
    k, v = workloads.kv_layer(DEV)
    gk, st1 = gpu_encode(k, d, "E8", 4.0, 31, dither=True)
    gv, st2 = gpu_encode(v, d, "E8", 4.0, 32, dither=True)
    assert st1 == 0 and st2 == 0
    fk, fv = fetch(gk), fetch(gv)
    q = queries(heads, group, d, 3)
    qf = q.float().numpy().astype(np.float64)
    scale = 1 / math.sqrt(d)
    out, st = gpu_attention(gk, gv, heads, tokens, d, "E8", 4.0, 4.0, 31, 32, q.to(DEV), scale, group)
    assert st == 0
    ref = oracle.kv_attention(fk, fv, heads, tokens, d, "E8", 31, 32, qf, scale, threads=16, group=group)
    assert_attention_close(out, ref, attention_tolerance(fk, fv, heads, tokens, d, "E8", 31, 32, qf, scale, group))

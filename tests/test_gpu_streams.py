"""The library enqueues everything on the caller's stream (needs a B200):
encode + decode + GEMV captured in a CUDA graph and replayed give the eager
results bit for bit, and calls on two streams at once, each with its own
workspace and outputs, give the same results as one after the other."""
import numpy as np
import pytest
import torch

from kv_quantization_tile_b200 import hq, workloads
from gpu_util import DEV, fetch

pytestmark = pytest.mark.gpu


def inputs(seed, rows=384, cols=2048):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16).to(DEV)


def test_graph_capture_and_replay():
    x = inputs(1)
    rows, cols = x.shape
    xv = torch.randn(cols, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).to(DEV)
    s = hq.alloc_stream(rows, cols, 256, "E8", 4.0, DEV)
    ws = hq.alloc_workspace(rows, cols, 256, DEV)
    y = torch.empty(rows, cols, dtype=torch.bfloat16, device=DEV)
    gy = torch.empty(rows, dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)

    def step():
        hq.hq_encode(x, 256, "E8", 4.0, 3, s, ws, st)
        hq.hq_decode(s, rows, cols, 256, "E8", 4.0, 3, y, st)
        hq.hq_decode_gemv(s, rows, cols, 256, "E8", 4.0, 3, xv, gy, st)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # eager, on the stream the graph will use
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = (fetch(s), y.clone(), gy.clone())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        s.payload.zero_(); y.zero_(); gy.zero_()
        graph.replay()
        torch.cuda.synchronize()
        got = fetch(s)
        for key in ("off", "scale", "k", "payload"):
            assert np.array_equal(got[key], eager[0][key]), key
        assert torch.equal(y, eager[1]) and torch.equal(gy, eager[2])
    assert int(st.item()) == 0


def test_two_streams_at_once():
    xs = [inputs(10 + i) for i in range(2)]
    rows, cols = xs[0].shape
    res = []
    for x in xs:  # one after the other
        s = hq.alloc_stream(rows, cols, 256, "D4", 3.0, DEV)
        hq.hq_encode(x, 256, "D4", 3.0, 5, s, hq.alloc_workspace(rows, cols, 256, DEV))
        torch.cuda.synchronize()
        res.append(fetch(s))
    streams = [torch.cuda.Stream() for _ in xs]
    outs = [hq.alloc_stream(rows, cols, 256, "D4", 3.0, DEV) for _ in xs]
    wss = [hq.alloc_workspace(rows, cols, 256, DEV) for _ in xs]
    for _ in range(3):
        for x, s, w, stm in zip(xs, outs, wss, streams):
            stm.wait_stream(torch.cuda.current_stream())
            hq.hq_encode(x, 256, "D4", 3.0, 5, s, w, stream=stm)
        torch.cuda.synchronize()
        for s, r in zip(outs, res):
            g = fetch(s)
            for key in ("off", "scale", "k", "payload"):
                assert np.array_equal(g[key], r[key]), key


def test_fixed_rate_graph_capture_and_replay():
    """Fixed-rate KV encode + attention over the fixed-rate streams, captured
    in a CUDA graph: replays reproduce the eager results bit for bit."""
    heads, tokens, d, lat, group = 2, 640, 128, "E8", 4
    g = torch.Generator().manual_seed(4)
    k = torch.randn(heads * tokens, d, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(heads * tokens, d, generator=g).to(torch.bfloat16).to(DEV)
    q = torch.randn(heads * group, d, generator=g).to(torch.bfloat16).to(DEV)
    slot = hq.hq_fixed_slot_words(d, lat, 4.0)
    ks = hq.alloc_fixed_stream(heads * tokens, d, d, slot, DEV)
    vs = hq.alloc_fixed_stream(heads * tokens, d, d, slot, DEV)
    ws = hq.alloc_attention_workspace(heads, tokens, d, group, DEV)
    out = torch.empty(heads * group, d, dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)

    def step():
        hq.hq_kv_encode_fixed(k, d, lat, 7, ks, st)
        hq.hq_kv_encode_fixed(v, d, lat, 8, vs, st)
        hq.hq_kv_attention(ks, vs, heads, tokens, d, lat, 4.0, 4.0, 7, 8, q, 0.1, out, ws, group=group, status=st)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = (ks.payload.clone(), ks.tile_k.clone(), vs.payload.clone(), out.clone())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        ks.payload.zero_(); vs.payload.zero_(); ks.tile_k.zero_(); out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(ks.payload, eager[0]) and torch.equal(ks.tile_k, eager[1])
        assert torch.equal(vs.payload, eager[2]) and torch.equal(out, eager[3])
    assert int(st.item()) == 0

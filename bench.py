#!/usr/bin/env python
"""Benchmark of the B200 HyperQuant codec.

A step is one pass of the codec over one Llama-3.1-8B-shaped decoder layer
(seven bf16 matrices, 218,103,808 weights, N(0, 0.02^2) with 0.1 % outlier
columns x20): E8 lattice at 4 bits per coordinate, tile 256 -- encode all
seven, then decode all seven back to bf16.  `value` is bf16 GB/s of encode
input plus decode output over the whole job (all ranks), with the inputs
resident in HBM.  Each rank encodes its own layer (independent problems: weak
scaling, no collective on the data path).

Also reported: per-kernel roofline of the dominant kernel (algorithmic bytes
/ CUDA-event time on the launching stream), the end-to-end figure through the
C ABI from pinned host buffers, every workload (the tiny fp32 matrix; the
Llama layer at 3, 4 and 5 bps; the dithered KV layer with D4 and E8 at 2, 3
and 4 bps; the whole 72-block DiT stack as one job plus D4/A2/Z passes over
its FFN matrices) with the itemized rate and Rice gap of each stream, the
batch-1 decode-GEMV, batched product, attention and fixed-rate paths, the
CPU oracle timed on a bounded sample on all cores and on one thread, and SM
clocks sampled during the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "E8 4-bps encode/decode GB/s of bf16 in/out and % of B200 HBM roofline"
TILE, LAT, BPS, SEED = 256, "E8", 4.0, 42


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-extras", action="store_true", help="skip GEMV/KV/e2e/CPU legs")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--only", default=None, help="comma-separated matrix names (profiling cases)")
    p.add_argument("--leg", default=None, choices=["gemv", "gemm", "configs", "dit", "kv_attention", "fixed", "profile"],
                   help="run one side leg alone on cuda:0 and print its JSON (profiling cases)")
    p.add_argument("--group", type=int, default=4, help="query heads per KV head for --leg kv_attention")
    p.add_argument("--batch", type=int, default=None, help="one batch size for --leg gemm")
    return p.parse_args()


LAYER_ELEMENTS = 218103808  # q, k, v, o, gate, up, down


def layer_config(world: int = 1) -> dict:
    return {"workload": "llama3.1-8b-layer: 7 bf16 matrices (q,k,v,o 4096/1024x4096, gate/up 14336x4096, "
                        "down 4096x14336), E8 4 bps tile 256, encode + decode",
            "elements_per_rank": LAYER_ELEMENTS, "tile": TILE, "lattice": LAT, "bps": BPS,
            "l2": "no flush: each step streams 436 MB in + 436 MB out per rank (> 126 MB L2)",
            "parallelism": f"replicas x{world} (independent layers, no data-path collective)"}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class Clocks:
    """SM clock and clock-event reasons of one GPU, sampled every 10 ms during
    the timed region through NVML (read-only queries); nvidia-smi if NVML is
    unavailable."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, device):
        self.device, self.samples, self.stop_flag, self.thread = device, [], False, None
        self.max_mhz, self.handle, self.nvml = None, None, None

    def _open(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            self.handle = pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)
        self.nvml = pynvml
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)

    def _loop(self):
        pn = self.nvml
        get_reasons = getattr(pn, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pn.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag:
            try:
                self.samples.append((pn.nvmlDeviceGetClockInfo(self.handle, pn.NVML_CLOCK_SM),
                                     get_reasons(self.handle)))
            except Exception:
                pass
            time.sleep(0.01)

    def start(self):
        try:
            self._open()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None

    def stop(self):
        if self.thread:
            self.stop_flag = True
            self.thread.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "samples": 0, "reasons": [], "source": "none"}
        reasons = set()
        for _, bits in self.samples:
            for name, const in self.REASONS.items():
                mask = getattr(self.nvml, const, None) or getattr(self.nvml, const.replace("Event", "Throttle"), 0)
                if bits & mask:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(reasons), "source": "nvml, 10 ms"}


# ------------------------------------------------------------------ oracle leg
def _oracle_sample():
    """The gate matrix of the Llama layer as uint16 bf16 bits, and the built oracle."""
    import numpy as np
    import torch

    import oracle
    from kv_quantization_tile_b200 import workloads

    gate = workloads.outlier_weight(14336, 4096, 1004, 1104, "cpu")
    oracle.build()
    return oracle, gate.view(torch.int16).numpy().view(np.uint16)


def _oracle_rows(oracle, bits, r0: int, rows: int, threads: int) -> None:
    blk = bits[r0: r0 + rows]
    s = oracle.encode(blk, TILE, LAT, BPS, SEED, threads=threads)
    oracle.decode(s, blk.shape[0], blk.shape[1], TILE, LAT, SEED, threads=threads)


def _oracle_timed(oracle, bits, seconds: float, threads: int):
    """Encode + decode of whole rows of the gate matrix, blocks of 8 rows per
    thread, until `seconds` of wall time have passed: (rows, seconds)."""
    done, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds and done < bits.shape[0]:
        n = min(8 * threads, bits.shape[0] - done)
        _oracle_rows(oracle, bits, done, n, threads)
        done += n
    return done, time.perf_counter() - t0


def cpu_baseline(seconds: float):
    """The CPU oracle (as it stands) on a bounded sample of the gate matrix,
    timed on all host cores (one thread per core over disjoint row blocks)
    and on one thread."""
    oracle, bits = _oracle_sample()
    cores = len(os.sched_getaffinity(0))
    rows, el = _oracle_timed(oracle, bits, seconds, cores)
    rows1, el1 = _oracle_timed(oracle, bits, max(1.0, seconds / 3), 1)
    cols = bits.shape[1]
    return {"value": round(4 * rows * cols / el / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"encode+decode of the first {rows} rows x {cols} of the gate matrix "
                      f"({rows * cols} weights, E8 4 bps, tile 256) in {el:.1f} s on {cores} threads",
            "single_thread": {"value": round(4 * rows1 * cols / el1 / 1e9, 5), "unit": "GB/s", "cores": 1,
                              "sample": f"first {rows1} rows x {cols} of the gate matrix in {el1:.1f} s"}}


def run_reference(args):
    """The oracle as the reference arm: every step encodes and decodes the same
    bounded sample of the Llama layer's gate matrix (a fixed number of whole
    rows, sized so that warm-up plus timed steps take about a minute), on all
    host cores; ms_per_step is the measured wall time of a step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    oracle, bits = _oracle_sample()
    cores = len(os.sched_getaffinity(0))
    cols = bits.shape[1]
    # calibrate the rows a step can take in its share of the minute
    rows_c, el_c = _oracle_timed(oracle, bits, 1.0, cores)
    per = max(0.25, min(args.cpu_seconds, 60.0 / max(1, args.steps + args.warmup)))
    rows = max(cores, min(bits.shape[0], int(rows_c / el_c * per) // cores * cores))
    for _ in range(args.warmup):
        _oracle_rows(oracle, bits, 0, rows, cores)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _oracle_rows(oracle, bits, 0, rows, cores)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    v = round(4 * rows * cols / (ms * 1e-3) / 1e9, 4)
    sample = (f"each step: encode+decode of the first {rows} rows x {cols} of the gate matrix "
              f"({rows * cols} weights, E8 4 bps, tile 256) on {cores} threads")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(layer_config(1), sample=sample, elements_per_step=rows * cols),
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


# ------------------------------------------------------------------ GPU leg
KERNEL_HEADERS = ("hq_device.cuh", "hq_fast.cuh", "hq_parse.cuh", "hq_internal.h")


def kernel_source_sha(kernel_file: str) -> str:
    """sha256 over a kernel's .cu file and the shared device headers."""
    h = hashlib.sha256()
    for f in (kernel_file,) + KERNEL_HEADERS:
        h.update(open(os.path.join(ROOT, "kv_quantization_tile_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def traffic_record(kernel_file: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (kernel file + shared headers, sha256
    recorded beside it)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))
        r = rec.get(kernel_file)
        if r and r.get("source_sha256") == kernel_source_sha(kernel_file):
            return r
    except Exception:
        pass
    return None


def run_ours(args):
    import torch
    import torch.distributed as dist

    from kv_quantization_tile_b200 import hq, workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    stream = torch.cuda.current_stream()
    mats = workloads.llama_layer(dev, names=args.only.split(",") if args.only else None)
    n_elem = sum(m.numel() for _, m in mats)
    ctx = []
    for name, x in mats:
        r, c = x.shape
        ctx.append({"name": name, "x": x, "shape": (r, c), "s": hq.alloc_stream(r, c, TILE, LAT, BPS, dev),
                    "ws": hq.alloc_workspace(r, c, TILE, dev),
                    "y": torch.empty(r, c, dtype=torch.bfloat16, device=dev)})
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def encode(m):
        hq.hq_encode(m["x"], TILE, LAT, BPS, SEED, m["s"], m["ws"], status)

    def decode(m):
        r, c = m["shape"]
        hq.hq_decode(m["s"], r, c, TILE, LAT, BPS, SEED, m["y"], status)

    def step(ev=None):
        for i, m in enumerate(ctx):
            if ev: ev["enc"][i][0].record(stream)
            encode(m)
            if ev: ev["enc"][i][1].record(stream)
        for i, m in enumerate(ctx):
            if ev: ev["dec"][i][0].record(stream)
            decode(m)
            if ev: ev["dec"][i][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, f"device status {int(status.item())}"
    comp_bytes = [m["s"].nbytes() for m in ctx]
    payload_words = sum(m["s"].words() for m in ctx)

    def E():
        return torch.cuda.Event(enable_timing=True)

    evs = [{"enc": [(E(), E()) for _ in ctx], "dec": [(E(), E()) for _ in ctx]} for _ in range(args.steps)]
    clocks = Clocks(dev)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = E(), E()
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms_local = t_start.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(ms_local)

    enc_ms = [sum(e[i][0].elapsed_time(e[i][1]) for e in (ev["enc"] for ev in evs)) / args.steps
              for i in range(len(ctx))]
    dec_ms = [sum(e[i][0].elapsed_time(e[i][1]) for e in (ev["dec"] for ev in evs)) / args.steps
              for i in range(len(ctx))]
    enc_bytes = [2 * m["x"].numel() + cb for m, cb in zip(ctx, comp_bytes)]
    dec_bytes = enc_bytes
    peak, peak_kind = peaks()
    enc_gbs = sum(enc_bytes) / sum(enc_ms) / 1e6
    dec_gbs = sum(dec_bytes) / sum(dec_ms) / 1e6
    dominant = "encode" if sum(enc_ms) >= sum(dec_ms) else "decode"
    dom_gbs = enc_gbs if dominant == "encode" else dec_gbs
    kfile = "hq_encode.cu" if dominant == "encode" else "hq_decode.cu"
    tr = traffic_record(kfile)
    value = world * 4 * n_elem / (ms * 1e-3) / 1e9

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(layer_config(world), elements_per_rank=n_elem),
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": round(dom_gbs, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(dom_gbs / peak, 4),
                     "traffic": tr["dram_bytes_per_launch"] if tr else None,
                     "traffic_launch": tr["launch"] if tr else None,
                     "alg_bytes_launch": tr["alg_bytes"] if tr else None},
        "ops": {"encode": {"ms_per_step": round(sum(enc_ms), 4), "alg_gbs": round(enc_gbs, 1),
                           "bf16_gbs": round(2 * n_elem / sum(enc_ms) / 1e6, 1), "frac": round(enc_gbs / peak, 4)},
                "decode": {"ms_per_step": round(sum(dec_ms), 4), "alg_gbs": round(dec_gbs, 1),
                           "bf16_gbs": round(2 * n_elem / sum(dec_ms) / 1e6, 1), "frac": round(dec_gbs / peak, 4)},
                "bits_per_weight_payload": round(32 * payload_words / n_elem, 4),
                "bits_per_weight_total": round(8 * sum(comp_bytes) / n_elem, 4),
                "per_matrix_ms": {m["name"]: [round(a, 4), round(b, 4)] for m, a, b in zip(ctx, enc_ms, dec_ms)}},
        "gpu_launches": 2 * len(ctx) * args.steps,
        "clocks": clk,
    }

    if not args.no_extras:
        out["e2e"] = e2e_leg(args, ctx, dev, stream, status, n_elem, world, max_over_ranks, barrier)
        if rank == 0:
            out["configs"] = configs_leg(dev, peak, [m["x"] for m in ctx])
            del ctx
            out["configs"]["dit_stack"] = dit_leg(dev, peak)
            out["paths"] = {"gemv": gemv_leg(dev, peak), "gemm": gemm_leg(dev, peak),
                            "kv_attention": attention_leg(dev, peak), "fixed_rate": fixed_leg(dev, peak)}
            out["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()


def e2e_leg(args, ctx, dev, stream, status, n_elem, world, max_over_ranks, barrier):
    """Same work through the C ABI from pinned host memory: per matrix, H2D of
    its input, encode, decode, D2H of the decoded matrix, all timed.  As a user
    would drive the API, copies run on their own streams: the input of one
    matrix crosses PCIe while another is encoded and a third is read back
    (per-matrix events order the reuse of every buffer across steps)."""
    import torch

    from kv_quantization_tile_b200 import hq

    # a small matrix first and last: the pipeline fills and drains quickly
    order = {"k": 0, "q": 1, "gate": 2, "up": 3, "down": 4, "o": 5, "v": 6}
    ctx = sorted(ctx, key=lambda m: order.get(m["name"], 3))
    host_in = [m["x"].cpu().pin_memory() for m in ctx]
    host_out = [torch.empty(m["shape"], dtype=torch.bfloat16).pin_memory() for m in ctx]
    dev_in = [torch.empty_like(m["x"]) for m in ctx]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    n = len(ctx)
    loaded = [torch.cuda.Event() for _ in range(n)]   # input m on the device
    encoded = [torch.cuda.Event() for _ in range(n)]  # input m consumed
    decoded = [torch.cuda.Event() for _ in range(n)]  # output m ready
    read = [torch.cuda.Event() for _ in range(n)]     # output m copied out
    for e in encoded + read:
        e.record(stream)

    def step():
        for i, (m, hi, di) in enumerate(zip(ctx, host_in, dev_in)):
            s_in.wait_event(encoded[i])
            with torch.cuda.stream(s_in):
                di.copy_(hi, non_blocking=True)
            loaded[i].record(s_in)
        for i, (m, di, ho) in enumerate(zip(ctx, dev_in, host_out)):
            r, c = m["shape"]
            stream.wait_event(loaded[i])
            stream.wait_event(read[i])
            with torch.cuda.stream(stream):
                hq.hq_encode(di, TILE, LAT, BPS, SEED, m["s"], m["ws"], status, stream=stream)
                encoded[i].record(stream)
                hq.hq_decode(m["s"], r, c, TILE, LAT, BPS, SEED, m["y"], status, stream=stream)
                decoded[i].record(stream)
            s_out.wait_event(decoded[i])
            with torch.cuda.stream(s_out):
                ho.copy_(m["y"], non_blocking=True)
            read[i].record(s_out)
        stream.wait_stream(s_out)

    steps = max(3, min(args.steps, 5))
    step()
    torch.cuda.synchronize()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_stream(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps)
    nbytes = 2 * n_elem
    return {"value": round(world * 4 * n_elem / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(ms, 3), "steps": steps, "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
            "overlap": "H2D, compute and D2H on three streams, pipelined across the seven matrices"}


def flush_l2(buf):
    buf.zero_()


def time_launches(fn, flush, reps=20):
    import torch
    ts = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def codec_pass(mats, tile, lat, bps, dev, peak, kv=False, reps=5, flush=None, seed=SEED, stats=True):
    """One job over `mats`: encode every matrix, then decode every matrix back
    to its own dtype (into one scratch output per shape), timed as two CUDA-event
    intervals on the current stream; median over `reps` jobs after one warm-up.
    Reports time, bytes, GB/s (algorithmic: input + stream bytes) and, when
    `stats`, the itemized rate of the streams (rate accounting kernel)."""
    import torch

    from kv_quantization_tile_b200 import hq

    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ws, out, streams = {}, {}, []
    for x in mats:
        r, c = x.shape
        if (r, c) not in ws:
            ws[(r, c)] = hq.alloc_workspace(r, c, tile, dev)
        if (r, c, x.dtype) not in out:
            out[(r, c, x.dtype)] = torch.empty_like(x)
        streams.append(hq.alloc_stream(r, c, tile, lat, bps, dev))
    enc_fn = hq.hq_kv_encode if kv else hq.hq_encode
    dec_fn = hq.hq_kv_decode if kv else hq.hq_decode

    def enc():
        for x, s in zip(mats, streams):
            enc_fn(x, tile, lat, bps, seed, s, ws[tuple(x.shape)], st)

    def dec():
        for x, s in zip(mats, streams):
            r, c = x.shape
            dec_fn(s, r, c, tile, lat, bps, seed, out[(r, c, x.dtype)], st)

    enc(); dec()
    torch.cuda.synchronize()
    assert int(st.item()) == 0, f"device status {int(st.item())}"
    flush = flush or (lambda: None)
    te = time_launches(enc, flush, reps=reps)
    td = time_launches(dec, flush, reps=reps)
    n = sum(x.numel() for x in mats)
    nin = sum(x.numel() * x.element_size() for x in mats)
    cb = sum(s.nbytes() for s in streams)
    alg = nin + cb
    res = {"matrices": len(mats), "weights": n, "input_bytes": nin, "stream_bytes": cb,
           "bits_per_weight_total": round(8 * cb / n, 4),
           "encode_ms": round(te, 4), "decode_ms": round(td, 4),
           "encode_alg_gbs": round(alg / te / 1e6, 1), "decode_alg_gbs": round(alg / td / 1e6, 1),
           "encode_frac": round(alg / te / 1e6 / peak, 4), "decode_frac": round(alg / td / 1e6 / peak, 4),
           "job_gbs": round(2 * nin / (te + td) / 1e6, 1)}
    if stats:
        tot_c = tot_h = None
        for x, s in zip(mats, streams):
            c, h = hq.hq_stream_stats(s, x.shape[0], x.shape[1], tile, lat, bps, status=st)
            tot_c = c if tot_c is None else tot_c + c
            tot_h = h if tot_h is None else tot_h + h
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        res["rate"] = hq.rate_report(tot_c.cpu().tolist(), tot_h.cpu().tolist(), tile)
    del streams, ws, out
    return res


def configs_leg(dev, peak, llama_mats):
    """Every workload: the tiny fp32 matrix, the Llama layer at 3, 4 and 5 bps,
    the KV layer (dithered, tile 128) for D4 and E8 at 2, 3 and 4 bps, each with
    its itemized rate and Rice gap."""
    import torch

    from kv_quantization_tile_b200 import workloads

    flushbuf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    res = {"tiny_fp32": dict(codec_pass([workloads.tiny(dev)], TILE, LAT, BPS, dev, peak, reps=20,
                                        flush=lambda: flush_l2(flushbuf)),
                             note="256 x 1024 fp32 (1 MB) E8 4 bps tile 256; L2 flushed before each timed job")}
    res["llama_layer"] = {f"E8_{b:g}bps": codec_pass(llama_mats, TILE, LAT, float(b), dev, peak)
                          for b in (3, 4, 5)}
    k, v = workloads.kv_layer(dev)
    res["kv_layer"] = {f"{lat}_{b:g}bps": codec_pass([k, v], 128, lat, float(b), dev, peak, kv=True, reps=10)
                       for lat in ("E8", "D4") for b in (2, 3, 4)}
    del k, v, flushbuf
    return res


def dit_leg(dev, peak, reps=3):
    """The 72-block video-DiT weight stack (720 bf16 matrices, 19.3 G weights,
    38.6 GB), all resident in HBM; one job = encode all 720 matrices at E8 4 bps
    tile 256, then decode all 720 (median of `reps` jobs).  Then the 144 FFN
    matrices alone with D4, A2 and Z at 4 bps."""
    import torch

    from kv_quantization_tile_b200 import workloads

    mats, ffn = [], []
    for b in range(workloads.DIT_BLOCKS):
        for name, x in workloads.dit_block(b, dev):
            mats.append(x)
            if name.startswith("ffn"):
                ffn.append(x)
    res = {"blocks": workloads.DIT_BLOCKS, "E8_4bps": codec_pass(mats, TILE, "E8", BPS, dev, peak, reps=reps)}
    for lat in ("D4", "A2", "Z"):
        res[f"ffn_{lat}_4bps"] = codec_pass(ffn, TILE, lat, BPS, dev, peak, reps=reps)
    del mats, ffn
    torch.cuda.empty_cache()
    return res


def gemv_leg(dev, peak):
    """Batch-1 decode-GEMV on 14336x4096 and 4096x14336 E8 4-bps streams vs the
    bf16 GEMV (cuBLAS) on the uncompressed matrices; L2 flushed before each."""
    import torch

    from kv_quantization_tile_b200 import hq, workloads

    w1, w2, x1, x2 = workloads.gemv_case(dev)
    flushbuf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    res = {}
    for name, w, x in (("14336x4096", w1, x1), ("4096x14336", w2, x2)):
        r, c = w.shape
        s = hq.alloc_stream(r, c, TILE, LAT, BPS, dev)
        ws = hq.alloc_workspace(r, c, TILE, dev)
        hq.hq_encode(w, TILE, LAT, BPS, SEED, s, ws)
        y = torch.empty(r, dtype=torch.float32, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        for _ in range(3):
            hq.hq_decode_gemv(s, r, c, TILE, LAT, BPS, SEED, x, y, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        ms = time_launches(lambda: hq.hq_decode_gemv(s, r, c, TILE, LAT, BPS, SEED, x, y, st),
                           lambda: flush_l2(flushbuf))
        xm = x.view(-1, 1)
        ms_bf16 = time_launches(lambda: torch.matmul(w, xm), lambda: flush_l2(flushbuf))
        nb = s.nbytes() + 2 * c + 4 * r
        res[name] = {"us": round(ms * 1e3, 2), "alg_gbs": round(nb / ms / 1e6, 1), "frac": round(nb / ms / 1e6 / peak, 4),
                     "compressed_bytes": s.nbytes(), "bf16_gemv_us": round(ms_bf16 * 1e3, 2),
                     "speedup_vs_bf16": round(ms_bf16 / ms, 3)}
        del s, ws
    return res


def gemm_leg(dev, peak, batches=(1, 16, 64, 256)):
    """Batched decode + matrix product on the tensor cores for the Llama gate
    projection (14336 x 4096, E8 4 bps): Y = X W_hat^T for X of `batch` bf16
    rows, against cuBLAS bf16 (torch.matmul) on the uncompressed weights and
    against decoding to bf16 first.  L2 flushed before each timed launch."""
    import torch

    from kv_quantization_tile_b200 import hq, workloads

    w1, _, _, _ = workloads.gemv_case(dev)
    r, c = w1.shape
    s = hq.alloc_stream(r, c, TILE, LAT, BPS, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    hq.hq_encode(w1, TILE, LAT, BPS, SEED, s, hq.alloc_workspace(r, c, TILE, dev), st)
    flushbuf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    wd = torch.empty_like(w1)
    res = {"matrix": f"{r}x{c}", "compressed_bytes": s.nbytes()}
    for batch in batches:
        g = torch.Generator(device=dev).manual_seed(6000 + batch)
        x = torch.randn(batch, c, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(batch, r, dtype=torch.float32, device=dev)
        ws = hq.alloc_gemm_workspace(r, c, batch, dev)
        ws8 = hq.alloc_gemm_int8_workspace(r, c, batch, dev)
        y8 = torch.empty(batch, r, dtype=torch.float32, device=dev)

        def ours():
            hq.hq_decode_gemm(s, r, c, TILE, LAT, BPS, SEED, x, y, ws, st)

        def ours_int8():
            hq.hq_decode_gemm_int8(s, r, c, TILE, LAT, BPS, SEED, x, y8, ws8, st)

        yf8 = torch.empty(batch, r, dtype=torch.float32, device=dev)

        def ours_fp8():
            hq.hq_decode_gemm_fp8(s, r, c, TILE, LAT, BPS, SEED, x, yf8, ws8, st)

        def dense():
            torch.matmul(x, w1.t())

        def decode_then_dense():
            hq.hq_decode(s, r, c, TILE, LAT, BPS, SEED, wd, st)
            torch.matmul(x, wd.t())

        for _ in range(3):
            ours(); ours_int8(); ours_fp8(); dense(); decode_then_dense()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        ref = (x.float() @ wd.float().t())  # the bf16 decode's product, for the int8 path's error
        rel8 = float((y8 - ref).norm() / ref.norm())
        relf8 = float((yf8 - ref).norm() / ref.norm())
        tf8 = time_launches(ours_fp8, lambda: flush_l2(flushbuf))
        rel16 = float((y - ref).norm() / ref.norm())
        t8 = time_launches(ours_int8, lambda: flush_l2(flushbuf))
        t = time_launches(ours, lambda: flush_l2(flushbuf))
        td = time_launches(dense, lambda: flush_l2(flushbuf))
        tdd = time_launches(decode_then_dense, lambda: flush_l2(flushbuf))
        flops = 2.0 * batch * r * c
        res[f"batch{batch}"] = {"us": round(t * 1e3, 2), "tflops": round(flops / t / 1e9, 2),
                                "weights_per_us": round(r * c / t / 1e3, 1),
                                "bf16_cublas_us": round(td * 1e3, 2), "decode_then_cublas_us": round(tdd * 1e3, 2),
                                "int8_us": round(t8 * 1e3, 2), "int8_rel_err": round(rel8, 5),
                                "fp8_us": round(tf8 * 1e3, 2), "fp8_rel_err": round(relf8, 5),
                                "bf16_rel_err": round(rel16, 5)}
    return res


def attention_leg(dev, peak, group=4):
    """Batch-1 decode attention of one Llama-3.1-8B layer: 32 query heads over
    the 8 x 32768 x 128 K and V caches (4 query heads per KV head), straight
    from the E8 4-bps dithered streams, against (a) torch's bf16 SDPA on the
    uncompressed cache and (b) decoding the streams to bf16 and then SDPA.
    L2 flushed before each timed launch (the streams fit in L2)."""
    import torch
    import torch.nn.functional as F

    from kv_quantization_tile_b200 import hq, workloads

    k, v = workloads.kv_layer(dev)
    heads, tokens, d = workloads.KV_HEADS, workloads.KV_TOKENS, workloads.KV_HEAD_DIM
    streams = []
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for x, seed in ((k, SEED), (v, SEED + 1)):
        s = hq.alloc_stream(heads * tokens, d, d, LAT, BPS, dev)
        hq.hq_kv_encode(x, d, LAT, BPS, seed, s, hq.alloc_workspace(heads * tokens, d, d, dev), st)
        streams.append(s)
    ks, vs = streams
    g = torch.Generator(device=dev).manual_seed(5000)
    q = torch.randn(heads * group, d, generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty(heads * group, d, dtype=torch.float32, device=dev)
    ws = hq.alloc_attention_workspace(heads, tokens, d, group, dev)
    scale = 1.0 / math.sqrt(d)

    def ours():
        hq.hq_kv_attention(ks, vs, heads, tokens, d, LAT, BPS, BPS, SEED, SEED + 1, q, scale, out, ws, group=group,
                           status=st)

    kb, vb = k.view(1, heads, tokens, d), v.view(1, heads, tokens, d)
    q4 = q.view(1, heads * group, 1, d)

    def sdpa(kk=kb, vv=vb):
        return F.scaled_dot_product_attention(q4, kk, vv, scale=scale, enable_gqa=True)

    kd, vd = torch.empty_like(k), torch.empty_like(v)

    def decode_then_sdpa():
        hq.hq_kv_decode(ks, heads * tokens, d, d, LAT, BPS, SEED, kd, st)
        hq.hq_kv_decode(vs, heads * tokens, d, d, LAT, BPS, SEED + 1, vd, st)
        sdpa(kd.view(1, heads, tokens, d), vd.view(1, heads, tokens, d))

    flushbuf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(3):
        ours(); sdpa(); decode_then_sdpa()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    t = time_launches(ours, lambda: flush_l2(flushbuf))
    t_sdpa = time_launches(sdpa, lambda: flush_l2(flushbuf))
    t_dec = time_launches(decode_then_sdpa, lambda: flush_l2(flushbuf))
    nb = ks.nbytes() + vs.nbytes() + 2 * q.numel() + 4 * out.numel()
    return {"config": {"kv_heads": heads, "tokens": tokens, "head_dim": d, "query_heads": heads * group,
                       "lattice": LAT, "bps": BPS},
            "us": round(t * 1e3, 2), "alg_gbs": round(nb / t / 1e6, 1), "frac": round(nb / t / 1e6 / peak, 4),
            "compressed_bytes": nb, "bf16_sdpa_us": round(t_sdpa * 1e3, 2),
            "decode_then_sdpa_us": round(t_dec * 1e3, 2), "speedup_vs_bf16_sdpa": round(t_sdpa / t, 3)}


def fixed_leg(dev, peak):
    """Fixed-rate streams at 4 bits per weight in total (side information
    included): the seven Llama-3.1-8B layer matrices (tile 256, E8, slot 31)
    and one KV layer's K and V with dither (tile 128, E8, slot 15); encode
    (with its per-tile scale search) and decode timed with CUDA events,
    inputs far larger than L2; plus the batch-1 decode-GEMV on the fixed
    14336x4096 stream.  The reconstruction error is reported beside the
    variable-rate stream's at its nominal 4 bps."""
    import torch

    from kv_quantization_tile_b200 import hq, workloads

    res = {}
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    flushbuf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def run(mats, tile, dither, tag):
        slot = hq.hq_fixed_slot_words(tile, LAT, BPS)
        ctx = []
        for x in mats:
            r, c = x.shape
            ctx.append((x, hq.alloc_fixed_stream(r, c, tile, slot, dev), torch.empty_like(x)))
        enc_fn = hq.hq_kv_encode_fixed if dither else hq.hq_encode_fixed
        dec_fn = hq.hq_kv_decode if dither else hq.hq_decode

        def enc():
            for x, s, _ in ctx:
                enc_fn(x, tile, LAT, SEED, s, st)

        def dec():
            for x, s, y in ctx:
                dec_fn(s, x.shape[0], x.shape[1], tile, LAT, BPS, SEED, y, st)

        for _ in range(3):
            enc(); dec()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        n = sum(x.numel() for x, _, _ in ctx)
        cb = sum(s.nbytes() for _, s, _ in ctx)
        te = time_launches(enc, lambda: flush_l2(flushbuf), reps=5)
        td = time_launches(dec, lambda: flush_l2(flushbuf), reps=5)
        num = sum(float(((y.float() - x.float()) ** 2).sum()) for x, _, y in ctx)
        den = sum(float((x.float() ** 2).sum()) for x, _, _ in ctx)
        # the variable-rate stream of the same inputs at its nominal rate, for comparison
        vnum, vbytes = 0.0, 0
        for x, _, y in ctx:
            r, c = x.shape
            v = hq.alloc_stream(r, c, tile, LAT, BPS, dev)
            (hq.hq_kv_encode if dither else hq.hq_encode)(x, tile, LAT, BPS, SEED, v, hq.alloc_workspace(r, c, tile, dev), st)
            dec_fn(v, r, c, tile, LAT, BPS, SEED, y, st)
            vnum += float(((y.float() - x.float()) ** 2).sum())
            vbytes += v.nbytes()
            del v
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        res[tag] = {"slot_words": slot, "tile": tile, "bits_per_value_total": round(8 * cb / n, 4),
                    "encode_ms": round(te, 4), "decode_ms": round(td, 4),
                    "encode_alg_gbs": round((2 * n + cb) / te / 1e6, 1),
                    "decode_alg_gbs": round((2 * n + cb) / td / 1e6, 1),
                    "encode_frac": round((2 * n + cb) / te / 1e6 / peak, 4),
                    "decode_frac": round((2 * n + cb) / td / 1e6 / peak, 4),
                    "rel_rmse": round(math.sqrt(num / den), 5),
                    "variable_rate": {"bits_per_value_total": round(8 * vbytes / n, 4),
                                      "rel_rmse": round(math.sqrt(vnum / den), 5)}}
        return ctx

    ctx = run([m for _, m in workloads.llama_layer(dev)], TILE, False, "llama_layer_e8")
    del ctx
    k, v = workloads.kv_layer(dev)
    ctx = run([k, v], 128, True, "kv_layer_e8")
    # attention of 32 query heads (4 per KV head) over the fixed-rate K and V streams
    group, heads = 4, workloads.KV_HEADS
    tokens = k.shape[0] // heads
    q = torch.randn(heads * group, 128, generator=torch.Generator(device=dev).manual_seed(5), device=dev).to(torch.bfloat16)
    out = torch.empty(heads * group, 128, dtype=torch.float32, device=dev)
    aws = hq.alloc_attention_workspace(heads, tokens, 128, group, dev)
    (_, ksf, _), (_, vsf, _) = ctx

    def attend():
        hq.hq_kv_attention(ksf, vsf, heads, tokens, 128, LAT, BPS, BPS, SEED, SEED, q, 128 ** -0.5, out, aws,
                           group=group, status=st)

    for _ in range(3):
        attend()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    t = time_launches(attend, lambda: flush_l2(flushbuf))
    nb = ksf.nbytes() + vsf.nbytes()
    res["kv_attention_group4"] = {"us": round(t * 1e3, 2), "alg_gbs": round(nb / t / 1e6, 1),
                                  "frac": round(nb / t / 1e6 / peak, 4), "compressed_bytes": nb}
    del ctx, k, v, ksf, vsf
    w1, _, x1, _ = workloads.gemv_case(dev)
    r, c = w1.shape
    slot = hq.hq_fixed_slot_words(TILE, LAT, BPS)
    s = hq.alloc_fixed_stream(r, c, TILE, slot, dev)
    hq.hq_encode_fixed(w1, TILE, LAT, SEED, s, st)
    y = torch.empty(r, dtype=torch.float32, device=dev)
    for _ in range(3):
        hq.hq_decode_gemv(s, r, c, TILE, LAT, BPS, SEED, x1, y, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ms = time_launches(lambda: hq.hq_decode_gemv(s, r, c, TILE, LAT, BPS, SEED, x1, y, st), lambda: flush_l2(flushbuf))
    nb = s.nbytes() + 2 * c + 4 * r
    res["gemv_14336x4096"] = {"us": round(ms * 1e3, 2), "alg_gbs": round(nb / ms / 1e6, 1),
                              "frac": round(nb / ms / 1e6 / peak, 4), "compressed_bytes": nb - 2 * c - 4 * r}
    return res


def profile_leg(dev):
    """One cold launch each of the decode-GEMV (14336 x 4096, E8 4 bps), the
    fixed-rate encode of the Llama gate matrix (31-word slots) and the KV
    attention of 32 query heads over the 8 x 32768 x 128 E8 4-bps K and V
    streams: the launches the path profiles capture."""
    import torch

    from kv_quantization_tile_b200 import hq, workloads

    st = torch.zeros(1, dtype=torch.int32, device=dev)
    w1, _, x1, _ = workloads.gemv_case(dev)
    r, c = w1.shape
    s = hq.alloc_stream(r, c, TILE, LAT, BPS, dev)
    hq.hq_encode(w1, TILE, LAT, BPS, SEED, s, hq.alloc_workspace(r, c, TILE, dev), st)
    y = torch.empty(r, dtype=torch.float32, device=dev)
    hq.hq_decode_gemv(s, r, c, TILE, LAT, BPS, SEED, x1, y, st)
    gate = workloads.llama_layer(dev, names=["gate"])[0][1]
    slot = hq.hq_fixed_slot_words(TILE, LAT, BPS)
    fs = hq.alloc_fixed_stream(gate.shape[0], gate.shape[1], TILE, slot, dev)
    hq.hq_encode_fixed(gate, TILE, LAT, SEED, fs, st)
    k, v = workloads.kv_layer(dev)
    heads, tokens, d = workloads.KV_HEADS, workloads.KV_TOKENS, workloads.KV_HEAD_DIM
    streams = []
    for x, seed in ((k, SEED), (v, SEED + 1)):
        sx = hq.alloc_stream(heads * tokens, d, d, LAT, BPS, dev)
        hq.hq_kv_encode(x, d, LAT, BPS, seed, sx, hq.alloc_workspace(heads * tokens, d, d, dev), st)
        streams.append(sx)
    q = torch.randn(4 * heads, d, generator=torch.Generator(device=dev).manual_seed(5000), device=dev).to(torch.bfloat16)
    out = torch.empty(4 * heads, d, dtype=torch.float32, device=dev)
    aws = hq.alloc_attention_workspace(heads, tokens, d, 4, dev)
    hq.hq_kv_attention(streams[0], streams[1], heads, tokens, d, LAT, BPS, BPS, SEED, SEED + 1, q, 1.0 / math.sqrt(d),
                       out, aws, group=4, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return {"launches": ["gemv_kernel 14336x4096", "encode_fixed_kernel gate", "kv_attention_kernel 32 query heads"]}


def run_leg(args):
    peak, _ = peaks()
    if args.leg == "gemv":
        res = gemv_leg("cuda", peak)
    elif args.leg == "gemm":
        res = gemm_leg("cuda", peak, batches=(args.batch,) if args.batch else (1, 16, 64, 256))
    elif args.leg == "configs":
        from kv_quantization_tile_b200 import workloads
        res = configs_leg("cuda", peak, [m for _, m in workloads.llama_layer("cuda")])
    elif args.leg == "dit":
        res = dit_leg("cuda", peak)
    elif args.leg == "profile":
        res = profile_leg("cuda")
    elif args.leg == "fixed":
        res = fixed_leg("cuda", peak)
    else:
        res = attention_leg("cuda", peak, group=args.group)
    print(json.dumps({"leg": args.leg, **res}))


def main():
    args = parse()
    if args.leg:
        run_leg(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

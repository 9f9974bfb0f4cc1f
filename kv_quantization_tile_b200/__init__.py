"""B200-native HyperQuant per-tile codec.

The codec (random-sign Walsh-Hadamard rotation per tile, per-tile scale,
nearest point of E8/D4/A2/Z, lossless strip, Rice code with a per-tile
parameter; decode, fused batch-1 decode-GEMV and the dithered KV variant)
runs in hand-written sm_100a CUDA kernels behind the C ABI declared in
``include/hq.h``.  ``kv_quantization_tile_b200.hq`` is a thin ctypes binding
with the same names; torch supplies device memory and streams only.
"""

"""Seeded synthetic inputs with the shapes and value distributions of the
codec's workloads.  No codec arithmetic lives here: this module only draws
tensors, so the CUDA path and the CPU oracle can be fed identical bytes.

Workloads (stand-ins for the pages' Llama-3.1-8B, LTX-2 and KV-cache
experiments, whose weights and data are not available; only shapes and
distributions are taken):

* ``tiny``       one 256 x 1024 fp32 matrix, N(0, 1), seed 0.
* ``llama_layer`` one Llama-3.1-8B-shaped decoder layer in bf16: q/o 4096 x
  4096, k/v 1024 x 4096, gate/up 14336 x 4096, down 4096 x 14336, entries
  N(0, 0.02^2) with 0.1 % of input columns scaled x20 (outlier channels).
* ``gemv_case``  14336 x 4096 and 4096 x 14336 bf16 N(0, 0.02^2) plus a bf16
  N(0, 1) vector for batch-1 decode-GEMV.
* ``kv_layer``   K and V, 8 heads x 32768 tokens x 128 bf16; V ~ N(0, 1),
  K ~ N(0, 1) times per-(head, channel) scales 2^U(-2, 3) (log-uniform in
  [0.25, 8]); laid out as (heads * tokens) rows of 128.
* ``dit_block``  block b of a 72-block video-DiT weight stack (19.3 G
  parameters): 8 attention matrices 4096 x 4096 (self and cross q/k/v/o),
  FFN up 16384 x 4096 and down 4096 x 16384, N(0, 0.02^2) with 0.1 %
  outlier columns x20.

Every tensor is drawn with ``torch.randn`` from a ``torch.Generator`` on
the requested device seeded as documented, so it is reproducible per device
type.  Row-major [rows, cols] = [out features, in features].
"""
from __future__ import annotations

import torch

LLAMA_LAYER = [("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
               ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336)]
DIT_BLOCK = ([(f"{kind}_{p}", 4096, 4096) for kind in ("self", "cross") for p in "qkvo"]
             + [("ffn_up", 16384, 4096), ("ffn_down", 4096, 16384)])
DIT_BLOCKS = 72
KV_HEADS, KV_TOKENS, KV_HEAD_DIM = 8, 32768, 128


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(rows: int, cols: int, std: float, seed: int, device="cpu",
           dtype=torch.bfloat16) -> torch.Tensor:
    x = torch.randn(rows, cols, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def outlier_weight(rows: int, cols: int, seed: int, outlier_seed: int, device="cpu",
                   std: float = 0.02, frac: float = 0.001, factor: float = 20.0) -> torch.Tensor:
    """N(0, std^2) with round(frac * cols) input columns scaled by `factor`
    before the bf16 rounding; the columns come from randperm(cols)."""
    x = torch.randn(rows, cols, generator=_gen(seed, device), device=device, dtype=torch.float32)
    x.mul_(std)
    n_out = round(frac * cols)
    if n_out:
        cols_idx = torch.randperm(cols, generator=_gen(outlier_seed, device), device=device)[:n_out]
        x[:, cols_idx] *= factor
    return x.to(torch.bfloat16)


def tiny(device="cpu") -> torch.Tensor:
    return normal(256, 1024, 1.0, 0, device, dtype=torch.float32)


def llama_layer(device="cpu", names=None):
    """[(name, bf16 tensor)] for the seven matrices, seeds 1000+m / 1100+m."""
    out = []
    for m, (name, r, c) in enumerate(LLAMA_LAYER):
        if names is None or name in names:
            out.append((name, outlier_weight(r, c, 1000 + m, 1100 + m, device)))
    return out


def gemv_case(device="cpu"):
    """(W1 14336x4096, W2 4096x14336, x1 len 4096, x2 len 14336), all bf16."""
    w1 = normal(14336, 4096, 0.02, 2000, device)
    w2 = normal(4096, 14336, 0.02, 2001, device)
    x = torch.randn(4096 + 14336, generator=_gen(2002, device), device=device).to(torch.bfloat16)
    return w1, w2, x[:4096].clone(), x[4096:].clone()


def kv_layer(device="cpu", tokens: int = KV_TOKENS):
    """(K, V) as [heads * tokens, 128] bf16."""
    k = torch.randn(KV_HEADS, tokens, KV_HEAD_DIM, generator=_gen(3000, device), device=device)
    v = torch.randn(KV_HEADS, tokens, KV_HEAD_DIM, generator=_gen(3001, device), device=device)
    u = torch.rand(KV_HEADS, 1, KV_HEAD_DIM, generator=_gen(3002, device), device=device)
    k.mul_(torch.exp2(u * 5.0 - 2.0))
    return (k.reshape(-1, KV_HEAD_DIM).to(torch.bfloat16),
            v.reshape(-1, KV_HEAD_DIM).to(torch.bfloat16))


def dit_block(b: int, device="cpu", names=None):
    """[(name, bf16 tensor)] for block b, seeds 4000 + 16 b + m (outliers +8)."""
    out = []
    for m, (name, r, c) in enumerate(DIT_BLOCK):
        if names is None or name in names:
            out.append((name, outlier_weight(r, c, 4000 + 16 * b + m, 4000 + 16 * b + m + 8,
                                             device)))
    return out

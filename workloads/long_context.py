"""Long block-external caches drawn on the device (the long-context sweep).

FlashBlock's pages report that the gap between dense and cached block-external
attention grows with context (100k to 800k tokens). Generating such caches with
the numpy generator would take minutes, so this module draws them on the GPU
with a seeded torch generator, in the dllm workload's distributions: K and V
~ N(0, 1) rounded to bf16, K channels scaled per (kv head, channel) by
LogNormal(0, 0.5). It computes nothing of the method: draw, scale, round, lay
out contiguously (token t of the single sequence is row t).
"""

from __future__ import annotations

import torch

_CHUNK = 1 << 16  # tokens drawn per call (bounds the float32 temporary)


def long_prefix(n_tokens: int, n_heads_kv: int = 32, head_dim: int = 128, seed: int = 2000,
                device="cuda"):
    """(k, v, k_scale): bf16 [n_tokens, n_heads_kv, head_dim] on `device`, seeded."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    k_scale = torch.empty(n_heads_kv, head_dim, device=device).log_normal_(0.0, 0.5, generator=g)
    k = torch.empty(n_tokens, n_heads_kv, head_dim, dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    for t0 in range(0, n_tokens, _CHUNK):
        t1 = min(n_tokens, t0 + _CHUNK)
        x = torch.randn(t1 - t0, n_heads_kv, head_dim, generator=g, device=device)
        k[t0:t1] = (x * k_scale).to(torch.bfloat16)
        torch.randn(t1 - t0, n_heads_kv, head_dim, generator=g, device=device, out=x)
        v[t0:t1] = x.to(torch.bfloat16)
    return k, v, k_scale

"""Seeded synthetic KV caches (inputs only; none of the method's arithmetic).

The pages measure on Mistral-7B, Llama-3-8B and Qwen2.5-7B caches; there are
no weights here, so caches with those shapes are drawn from a generator:

* keys before RoPE: K_pre[h][t][d] = z * lam[h][d], z ~ N(0, 1),
  lam ~ lognormal(0, 0.5) per (head, channel); outlier channels are scaled
  (4 of 128 channels per head x8, or a fixed number of (head, channel) pairs
  per layer x20 for the Qwen-shaped cache);
* then split-half rotary embedding at the token's position with the model's
  theta, evaluated in fp64 with direct cos/sin, then rounded to bf16;
* values: V = z * lam_V, lam_V ~ lognormal(0, 0.3), no rotation.

Every layer draws from its own ``torch.Generator`` seeded ``seed*1000 + layer``
on the device it runs on (CPU and CUDA streams differ; parity tests always
hand the same tensors to both sides).  Used by the tests, the benchmark and
the smoke check, and shared by the CUDA path and the oracle.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

D = 128


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    heads: int
    tokens: int
    theta: float
    seed: int
    bits_k: int = 3
    bits_v: int = 2
    evict_pct: int = 0
    window: int = 64
    # outliers: ("per_head", count, factor) or ("per_layer", count, factor)
    outliers: tuple = ("per_head", 4, 8.0)
    protected_layers: tuple = ()
    # decode-append regime
    sequences: int = 1
    append_steps: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def quantised_layers(self) -> list[int]:
        return [l for l in range(self.layers) if l not in self.protected_layers]


WORKLOADS = {
    # 1 layer, 8 KV heads, 2048 tokens, theta 1e4, K3V2, no eviction, seed 0
    "tiny": Workload("tiny", 1, 8, 2048, 1e4, 0),
    # Mistral-7B-shaped: 32 layers, 8 KV heads, 32768 tokens, theta 1e6,
    # 60% eviction, BOS + 64-token window, seed 1
    "mistral7b_32k": Workload("mistral7b_32k", 32, 8, 32768, 1e6, 1, evict_pct=60, window=64),
    # Llama-3-8B-shaped: 32 layers, 8 KV heads, 131072 tokens, theta 5e5, no eviction, seed 2
    "llama3_8b_128k": Workload("llama3_8b_128k", 32, 8, 131072, 5e5, 2),
    # Qwen2.5-7B-shaped: 28 layers, 4 KV heads, 65536 tokens, theta 1e6, 5 (head, channel)
    # pairs x20 per layer, layers 0, 1, 26, 27 kept bf16, others 35% eviction, window 128
    "qwen25_7b_64k": Workload("qwen25_7b_64k", 28, 4, 65536, 1e6, 3, evict_pct=35, window=128,
                              outliers=("per_layer", 5, 20.0), protected_layers=(0, 1, 26, 27)),
    # decode-append: 64 sequences x 32 layers x 8 heads, 16384-token caches, 256 append
    # steps of one token per (sequence, layer), K2V2, theta 1e4, seed 4
    "decode_append": Workload("decode_append", 32, 8, 16384, 1e4, 4, bits_k=2, bits_v=2,
                              sequences=64, append_steps=256),
}


def layer_generator(seed: int, layer: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + int(layer))
    return g


def _scales(wl: Workload, g: torch.Generator, device):
    H = wl.heads
    lam_k = torch.exp(0.5 * torch.randn(H, D, generator=g, device=device, dtype=torch.float32))
    kind, count, factor = wl.outliers
    if kind == "per_head":
        for h in range(H):
            idx = torch.randperm(D, generator=g, device=device)[:count]
            lam_k[h, idx] *= factor
    else:
        idx = torch.randperm(H * D, generator=g, device=device)[:count]
        lam_k.view(-1)[idx] *= factor
    lam_v = torch.exp(0.3 * torch.randn(H, D, generator=g, device=device, dtype=torch.float32))
    return lam_k, lam_v


def rope_forward_fp64(x: torch.Tensor, positions: torch.Tensor, theta: float) -> torch.Tensor:
    """Split-half RoPE in fp64 with direct cos/sin (data synthesis only).

    x [..., T, 128] fp64, positions [T] int64."""
    i = torch.arange(D // 2, dtype=torch.float64, device=x.device)
    w = torch.pow(torch.tensor(float(theta), dtype=torch.float64, device=x.device), -i / 64.0)
    ang = positions.to(torch.float64)[:, None] * w[None, :]
    c, s = torch.cos(ang), torch.sin(ang)
    a, b = x[..., : D // 2], x[..., D // 2:]
    return torch.cat([a * c - b * s, b * c + a * s], dim=-1)


def gen_layer(wl: Workload, layer: int, device="cpu", tokens: int | None = None,
              pos0: int = 0, seed_offset: int = 0, head_chunk: int = 1):
    """One layer's (K, V) as bf16 [H][T][128] tensors on ``device``.

    ``tokens`` overrides the length (for small cases); ``pos0`` shifts the RoPE
    positions (appended tokens); ``seed_offset`` selects an independent stream
    (e.g. per sequence or per append step)."""
    T = wl.tokens if tokens is None else int(tokens)
    H = wl.heads
    g = layer_generator(wl.seed + seed_offset, layer, device)
    lam_k, lam_v = _scales(wl, g, device)
    K = torch.empty(H, T, D, dtype=torch.bfloat16, device=device)
    V = torch.empty(H, T, D, dtype=torch.bfloat16, device=device)
    pos = torch.arange(pos0, pos0 + T, dtype=torch.int64, device=device)
    for h0 in range(0, H, head_chunk):
        h1 = min(H, h0 + head_chunk)
        z = torch.randn(h1 - h0, T, D, generator=g, device=device, dtype=torch.float32)
        kpre = (z * lam_k[h0:h1, None, :]).to(torch.float64)
        K[h0:h1] = rope_forward_fp64(kpre, pos, wl.theta).to(torch.bfloat16)
        del z, kpre
        z = torch.randn(h1 - h0, T, D, generator=g, device=device, dtype=torch.float32)
        V[h0:h1] = (z * lam_v[h0:h1, None, :]).to(torch.bfloat16)
        del z
    return K, V


def ar1_noise(shape, rho: float, g: torch.Generator, device, block: int = 64) -> torch.Tensor:
    """Unit-variance Gaussian noise [..., T, D] correlated along the token axis:
    z_t = rho z_{t-1} + sqrt(1 - rho^2) e_t (an AR(1) process per channel),
    computed block by block (a scaled cumulative sum inside each block of 64
    tokens, the carry between blocks)."""
    *lead, T, Dd = shape
    e = torch.randn(*lead, T, Dd, generator=g, device=device, dtype=torch.float64)
    out = torch.empty_like(e)
    c = (1.0 - rho * rho) ** 0.5
    t = torch.arange(block, dtype=torch.float64, device=device)
    up = (rho ** t)[:, None]           # rho^k
    down = (rho ** (-t))[:, None]      # rho^-k
    carry = e[..., 0, :]               # z_0 ~ N(0, 1)
    for b0 in range(0, T, block):
        b1 = min(T, b0 + block)
        k = b1 - b0
        x = c * e[..., b0:b1, :]
        if b0 == 0:
            x = x.clone()
            x[..., 0, :] = carry
            z = up[:k] * torch.cumsum(x * down[:k], dim=-2)
        else:
            z = up[:k] * (rho * carry[..., None, :] + torch.cumsum(x * down[:k], dim=-2))
        out[..., b0:b1, :] = z
        carry = z[..., -1, :]
    return out.to(torch.float32)


def gen_layer_correlated(wl: Workload, layer: int, device="cpu", rho: float = 0.95,
                         tokens: int | None = None):
    """gen_layer with token-to-token correlation: the same per-channel scales,
    outliers and rotary embedding, but z drawn as an AR(1) process along the
    tokens (rho between neighbours) instead of independently, the way
    consecutive tokens of a real cache resemble each other."""
    T = wl.tokens if tokens is None else int(tokens)
    g = layer_generator(wl.seed + 7919, layer, device)
    lam_k, lam_v = _scales(wl, g, device)
    pos = torch.arange(T, dtype=torch.int64, device=device)
    zk = ar1_noise((wl.heads, T, D), rho, g, device)
    kpre = (zk * lam_k[:, None, :]).to(torch.float64)
    K = rope_forward_fp64(kpre, pos, wl.theta).to(torch.bfloat16)
    zv = ar1_noise((wl.heads, T, D), rho, g, device)
    V = (zv * lam_v[:, None, :]).to(torch.bfloat16)
    return K, V


def gen_prerope_keys(wl: Workload, layer: int, device="cpu", tokens: int | None = None):
    """The keys of ``gen_layer`` before rotation (fp64), for RoPE pins."""
    T = wl.tokens if tokens is None else int(tokens)
    H = wl.heads
    g = layer_generator(wl.seed, layer, device)
    lam_k, _ = _scales(wl, g, device)
    out = []
    for h in range(H):
        z = torch.randn(1, T, D, generator=g, device=device, dtype=torch.float32)
        out.append((z * lam_k[h:h + 1, None, :]).to(torch.float64))
        torch.randn(1, T, D, generator=g, device=device, dtype=torch.float32)  # V draw
    return torch.cat(out, 0)

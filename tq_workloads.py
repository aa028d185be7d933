"""Seeded synthetic inputs for the codec's workloads.

Holds no step of the method: only random fp16 tensors with the shapes, value
distributions and outlier structure of the workloads below. Every tensor is
drawn in float32 from a seeded torch generator, scaled in float32, and cast
once to fp16 (round to nearest even). The same module feeds the CUDA path and
the fp64 oracle (which reads the same fp16 bytes), so no random number is
ever re-implemented.

Workloads (names used by the tests and ``bench.py``):

* ``single_tensor``: 4096 x 128, N(0,1), seed 0; 1% of the vectors (41, picked
  by randperm) get one coordinate (randint) multiplied by 20.
* ``llama_layer``: K and V of shape [8, 8192, 8, 128], N(0,1); K seed 1,
  V seed 2; in K, 4 channels per head (randperm(128)[:4], seed 3) are x10 at
  every position (RoPE-like outlier channels).
* ``long_context_layer``: layer l of an 80-layer cache, K and V
  [1, 131072, 8, 128], N(0,1) (seeds 1000+2l and 1000+2l+1) times a
  per-(layer, tensor, head, channel) scale exp(0.5 N(0,1)) (seed 7).
* ``decode_step``: query [16, 32, 128] = N(0,1)/sqrt(128) (seed 11), K and V
  sources [16, 32768, 8, 128] N(0,1) (seeds 12, 13).
* ``append_stream``: 256 sequences x 8 heads, one token per step, N(0,1) with
  each coordinate x20 with probability 0.005 (seed 21 + run).
* ``stress_rows``: the seven stress distributions of the parity stress test
  (``STRESS_KINDS``; see the function).
"""

from __future__ import annotations

import math

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_f16(shape, seed: int, device="cpu", scale: float = 1.0) -> torch.Tensor:
    """N(0, scale^2) in float32, cast once to fp16."""
    x = torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(torch.float16)


def single_tensor(n: int = 4096, d: int = 128, seed: int = 0, outlier_frac: float = 0.01,
                  outlier_scale: float = 20.0, device="cpu") -> torch.Tensor:
    g = _gen(seed, "cpu")
    x = torch.randn(n, d, generator=g, dtype=torch.float32)
    k = int(round(outlier_frac * n))
    rows = torch.randperm(n, generator=g)[:k]
    cols = torch.randint(0, d, (k,), generator=g)
    x[rows, cols] *= outlier_scale
    return x.to(torch.float16).to(device)


def llama_layer(B: int = 8, S: int = 8192, H: int = 8, d: int = 128, device="cuda",
                k_seed: int = 1, v_seed: int = 2, channel_seed: int = 3, n_channels: int = 4,
                channel_scale: float = 10.0):
    """(K, V) fp16 [B, S, H, d]; K has n_channels outlier channels per head."""
    k = torch.randn(B, S, H, d, generator=_gen(k_seed, device), device=device, dtype=torch.float32)
    gc = _gen(channel_seed, "cpu")
    scale = torch.ones(H, d, dtype=torch.float32)
    for h in range(H):
        scale[h, torch.randperm(d, generator=gc)[:n_channels]] = channel_scale
    k = (k * scale.to(device)).to(torch.float16)
    v = randn_f16((B, S, H, d), v_seed, device)
    return k, v


def long_context_scales(n_layers: int = 80, H: int = 8, d: int = 128, seed: int = 7) -> torch.Tensor:
    """exp(0.5 N(0,1)) per (layer, tensor K/V, head, channel), float32 [L, 2, H, d]."""
    z = torch.randn(n_layers, 2, H, d, generator=_gen(seed, "cpu"), dtype=torch.float32)
    return torch.exp(0.5 * z)


def long_context_layer(layer: int, S: int = 131072, H: int = 8, d: int = 128, device="cuda",
                       scales: torch.Tensor | None = None):
    """(K, V) fp16 [1, S, H, d] of one layer of the 80-layer cache."""
    if scales is None:
        scales = long_context_scales(H=H, d=d)
    out = []
    for t in range(2):
        x = torch.randn(1, S, H, d, generator=_gen(1000 + 2 * layer + t, device), device=device,
                        dtype=torch.float32)
        out.append((x * scales[layer, t].to(device)).to(torch.float16))
    return out[0], out[1]


def decode_step(B: int = 16, Hq: int = 32, Hkv: int = 8, S: int = 32768, d: int = 128, device="cuda",
                q_seed: int = 11, k_seed: int = 12, v_seed: int = 13):
    """(q [B,Hq,d], K [B,S,Hkv,d], V [B,S,Hkv,d]) fp16."""
    q = randn_f16((B, Hq, d), q_seed, device, scale=1.0 / math.sqrt(d))
    k = randn_f16((B, S, Hkv, d), k_seed, device)
    v = randn_f16((B, S, Hkv, d), v_seed, device)
    return q, k, v


def append_stream(run: int, steps: int, n_seq: int = 256, H: int = 8, d: int = 128, device="cuda",
                  p_outlier: float = 0.005, outlier_scale: float = 20.0) -> torch.Tensor:
    """fp16 [steps, n_seq, H, d]: the new token of every sequence at each step."""
    g = _gen(21 + run, device)
    x = torch.randn(steps, n_seq, H, d, generator=g, device=device, dtype=torch.float32)
    hit = torch.rand(steps, n_seq, H, d, generator=g, device=device) < p_outlier
    x = torch.where(hit, x * outlier_scale, x)
    return x.to(torch.float16)


def edge_vectors(d: int, device="cpu") -> torch.Tensor:
    """Degenerate rows: zero, constant, single spikes, fp16 max, subnormals, alternating."""
    rows = [torch.zeros(d), torch.ones(d), torch.full((d,), -3.5)]
    for k in (0, 1, d // 2, d - 1):
        e = torch.zeros(d)
        e[k] = 1.0
        rows.append(e)
    e = torch.zeros(d)
    e[3] = -7.0
    rows.append(e)
    rows.append(torch.full((d,), 65504.0))
    rows.append(torch.full((d,), 2.0 ** -24))
    rows.append(torch.tensor([(-1.0) ** i * 2.0 ** -20 for i in range(d)]))
    rows.append(torch.tensor([(-1.0) ** (i // 3) for i in range(d)]))
    return torch.stack(rows).to(torch.float16).to(device)


STRESS_KINDS = ("gauss", "student3", "channel_lognormal", "outlier_x10", "dynamic_range", "sparse", "mean_dominated")


def stress_rows(kind: str, n: int, d: int, seed: int, device="cuda") -> torch.Tensor:
    """n x d rows of one of the stress distributions, float32 then fp16 once
    (values clamped to +-60000 before the cast):

    * ``gauss``: N(0,1);
    * ``student3``: N(0,1) / sqrt(chi^2_3 / 3) per element (heavy tails);
    * ``channel_lognormal``: N(0,1) times a per-channel exp(1.5 N(0,1));
    * ``outlier_x10``: N(0,1) with 4 channels (randperm) times 10;
    * ``dynamic_range``: N(0,1) times 2^k per element, k uniform in [-14, 13];
    * ``sparse``: N(0,1) kept with probability 0.1, else 0;
    * ``mean_dominated``: 3 + 0.01 N(0,1).
    """
    g = _gen(seed, device)
    x = torch.randn(n, d, generator=g, device=device, dtype=torch.float32)
    if kind == "gauss":
        pass
    elif kind == "student3":
        chi = torch.randn(n, d, 3, generator=g, device=device).pow(2).sum(-1) / 3
        x = x / chi.sqrt()
    elif kind == "channel_lognormal":
        x = x * torch.exp(torch.randn(1, d, generator=g, device=device) * 1.5)
    elif kind == "outlier_x10":
        cols = torch.randperm(d, generator=_gen(seed, "cpu"))[:4].to(device)
        x[:, cols] *= 10.0
    elif kind == "dynamic_range":
        x = x * torch.pow(2.0, torch.randint(-14, 14, (n, d), generator=g, device=device).float())
    elif kind == "sparse":
        x = x * (torch.rand(n, d, generator=g, device=device) < 0.1).float()
    elif kind == "mean_dominated":
        x = x * 0.01 + 3.0
    else:
        raise ValueError(f"unknown stress kind {kind!r}")
    return x.clamp(-60000.0, 60000.0).to(torch.float16)

"""Seeded synthetic INT8 workloads (no codec arithmetic here).

These stand in for the quantised ML tensors the Shannonic evaluation uses (§4 worked example:
an INT8 Llama k_proj weight; §5 Table 1: weights and activations; §6.2: KV / activation
transfer). Nothing in this module computes a histogram, an entropy code or a table: it only draws
numbers, so the CPU oracle and the CUDA path can be fed the same tensors.

Every generator takes a ``device`` so the large workloads can be drawn on the GPU; draws on a
given device are reproducible from the seed.
"""
from __future__ import annotations

import math

import torch

# Scales of the truncated discrete Laplace pmf  p(v) ∝ exp(-|v|/b), v ∈ [-128, 127],
# at which its entropy is 2, 4, 5.3 and 7.9 bits.
LAPLACE_B_FOR_ENTROPY = {2.0: 0.8116, 4.0: 2.9704, 5.3: 7.258, 7.9: 97.1673}

KV_SHAPE = (32, 2, 8, 8, 4096, 128)  # layers, K/V, batch, kv_heads, seq, head_dim


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def truncated_laplace_pmf(b: float) -> torch.Tensor:
    v = torch.arange(-128, 128, dtype=torch.float64)
    w = torch.exp(-v.abs() / b)
    return w / w.sum()


def laplace_int8(n: int, b: float, seed: int, device="cpu") -> torch.Tensor:
    """n i.i.d. draws of the truncated discrete Laplace(0, b) on [-128, 127] (inverse CDF)."""
    cdf = torch.cumsum(truncated_laplace_pmf(b), 0).to(device=device, dtype=torch.float64)
    cdf[-1] = 1.0
    g = _gen(seed, device)
    out = torch.empty(n, dtype=torch.int8, device=device)
    step = 1 << 26
    for s in range(0, n, step):
        m = min(step, n - s)
        u = torch.rand(m, generator=g, device=device, dtype=torch.float64)
        idx = torch.searchsorted(cdf, u, right=True).clamp_(max=255)
        out[s:s + m] = (idx - 128).to(torch.int8)
    return out


def weight_like_int8(rows: int = 4096, cols: int = 1024, seed: int = 1, device="cpu") -> torch.Tensor:
    """Weight-like tensor: N(0,1), 1% outliers scaled ×8, per-row absmax INT8 quantisation."""
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device)
    mask = torch.rand(rows, cols, generator=g, device=device) < 0.01
    w = torch.where(mask, w * 8.0, w)
    scale = w.abs().amax(dim=1, keepdim=True) / 127.0
    return torch.round(w / scale).clamp_(-127, 127).to(torch.int8).reshape(-1)


def int4_weight_like(rows: int = 4096, cols: int = 4096, group: int = 64, seed: int = 6, device="cpu") -> torch.Tensor:
    """INT4 group-wise quantised weight-like tensor, one value per byte (int8 in [-8, 7]).

    N(0,1) weights with 1% outliers x8 (as weight_like_int8), absmax-quantised to the symmetric
    4-bit grid per group of `group` consecutive values of a row: q = clamp(round(w / s), -8, 7),
    s = absmax / 7. The 4-bit alphabet enters the codec as 16 symbols of the byte alphabet."""
    g = _gen(seed, device)
    w = torch.randn(rows, cols, generator=g, device=device)
    mask = torch.rand(rows, cols, generator=g, device=device) < 0.01
    w = torch.where(mask, w * 8.0, w).reshape(rows, cols // group, group)
    s = w.abs().amax(dim=-1, keepdim=True).clamp_min(1e-30) / 7.0
    return torch.round(w / s).clamp_(-8, 7).to(torch.int8).reshape(-1)


def kv_cache_segment_int8_and_scales(layer: int, kv: int, seed: int = 2, device="cpu", shape=KV_SHAPE):
    """One (layer, K/V) slice of the INT8 KV cache [layers, 2, batch, kv_heads, seq, head_dim] and
    its dequantisation scales (float32, one per head_dim group, in group order).

    bf16 N(0,1) values times a per-channel scale ~ LogNormal(0, 0.5) (a channel is a
    (layer, K/V, kv_head, head_dim) position, shared over batch and seq), then absmax INT8
    quantisation per group of head_dim (=128) values: q = round(x / s), s = absmax / 127.
    """
    _, _, B, Hk, T, D = shape
    g = _gen(seed * 1_000_003 + layer * 2 + kv, device)
    scale = torch.exp(0.5 * torch.randn(Hk, D, generator=g, device=device))
    x = torch.randn(B, Hk, T, D, generator=g, device=device)
    x = (x * scale[None, :, None, :]).to(torch.bfloat16).float()
    s = x.abs().amax(dim=-1, keepdim=True).clamp_min(1e-30) / 127.0
    q = torch.round(x / s).clamp_(-127, 127).to(torch.int8).reshape(-1)
    return q, s.reshape(-1).float()


def kv_cache_segment_int8(layer: int, kv: int, seed: int = 2, device="cpu", shape=KV_SHAPE) -> torch.Tensor:
    """The INT8 values of kv_cache_segment_int8_and_scales."""
    return kv_cache_segment_int8_and_scales(layer, kv, seed, device, shape)[0]


def kv_cache_int8(seed: int = 2, device="cpu", shape=KV_SHAPE) -> torch.Tensor:
    """The whole KV cache, flattened; segment (layer, kv) is the contiguous slice
    [(2*layer + kv) * seg, (2*layer + kv + 1) * seg)."""
    L, KV = shape[0], shape[1]
    seg = math.prod(shape[2:])
    out = torch.empty(L * KV * seg, dtype=torch.int8, device=device)
    for layer in range(L):
        for kv in range(KV):
            i = layer * KV + kv
            out[i * seg:(i + 1) * seg] = kv_cache_segment_int8(layer, kv, seed, device, shape)
    return out


def kv_cache_scales(seed: int = 2, device="cpu", shape=KV_SHAPE) -> torch.Tensor:
    """Dequantisation scales of kv_cache_int8 (one float32 per head_dim group, in tensor order)."""
    L, KV = shape[0], shape[1]
    return torch.cat([kv_cache_segment_int8_and_scales(layer, kv, seed, device, shape)[1]
                      for layer in range(L) for kv in range(KV)])


def kv_cache_segments(shape=KV_SHAPE):
    seg = math.prod(shape[2:])
    return [(i * seg, seg) for i in range(shape[0] * shape[1])]


def activation_batch_int8(n_tensors: int = 1024, n: int = 65536, seed: int = 3, device="cpu"):
    """n_tensors activation-like INT8 tensors of n values, concatenated.

    Per tensor a family is drawn from {Laplace, Gaussian, ReLU(Gaussian) (50% zeros)} and a scale
    σ ~ LogUniform[1, 32] in INT8 units; values are rounded and clipped to [-128, 127].
    Returns (tensor, segments, families).
    """
    g = _gen(seed, device)
    fam = torch.randint(0, 3, (n_tensors,), generator=g, device=device)
    sigma = torch.exp(torch.rand(n_tensors, generator=g, device=device) * math.log(32.0))
    z = torch.randn(n_tensors, n, generator=g, device=device)
    u = torch.rand(n_tensors, n, generator=g, device=device).clamp_min(1e-12)
    sgn = torch.where(torch.rand(n_tensors, n, generator=g, device=device) < 0.5, -1.0, 1.0)
    lap = sgn * (-torch.log(u)) / math.sqrt(2.0)  # unit-variance Laplace
    x = torch.where((fam == 0)[:, None], lap, z)
    x = torch.where((fam == 2)[:, None], z.clamp_min(0.0), x)
    x = torch.round(x * sigma[:, None]).clamp_(-128, 127).to(torch.int8).reshape(-1)
    segs = [(i * n, n) for i in range(n_tensors)]
    return x, segs, fam.cpu().tolist()


def sweep_points():
    """The entropy × chunk × K × L grid of the 1 GiB stream sweep."""
    pts = []
    for H in (2.0, 4.0, 5.3, 7.9):
        for C in (1024, 4096, 16384):
            for K in (8, 16, 32):
                for L in (64, 128, 256):
                    pts.append({"H": H, "b": LAPLACE_B_FOR_ENTROPY[H], "C": C, "K": K, "L": L})
    return pts


def sweep_stream_int8(H: float, n: int = 1 << 30, seed: int = 4, device="cpu") -> torch.Tensor:
    return laplace_int8(n, LAPLACE_B_FOR_ENTROPY[H], seed, device)

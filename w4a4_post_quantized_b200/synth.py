"""Seeded synthetic inputs shaped like a VGGT transformer's linear layers.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds none of the quantization method's arithmetic: it only draws numbers and
lays them out.

Token layout (page "十亿参数的三维重建模型，能塞进手机吗？", section
"视觉几何基础 Transformer（VGGT）": every frame gets 1 camera token and 4
register tokens; observation 1 of section "双平滑细粒度量化（DSFQ）": those
first 5 tokens carry the outliers that make the activations heavy-tailed):

  * a frame is 1374 tokens: 5 special tokens (rows f*1374 + 0..4) followed by
    37 x 37 = 1369 patch tokens;
  * activations X ~ N(0, 1); special-token rows are scaled by 40; 8 seeded
    distinct feature channels are scaled by 15 in every row (so special-row
    cells on those channels are scaled by 600);
  * weights W ~ N(0, 0.02^2), bias ~ N(0, 0.01^2);
  * everything is rounded to bf16 (round to nearest even) and returned as raw
    uint16 bit patterns.

Random numbers come from numpy's PCG64 generator seeded with the given seed.
"""
from __future__ import annotations

import numpy as np

FRAME_TOKENS = 1374
SPECIAL_TOKENS = 5
SPECIAL_SCALE = 40.0
OUTLIER_CHANNELS = 8
OUTLIER_SCALE = 15.0


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def special_rows(M: int) -> np.ndarray:
    """Row indices of the camera + register tokens among M tokens."""
    starts = np.arange(0, M, FRAME_TOKENS)
    rows = (starts[:, None] + np.arange(SPECIAL_TOKENS)[None, :]).ravel()
    return rows[rows < M]


def outlier_channels(K: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64([seed, 0x0C4A]))
    return np.sort(rng.choice(K, size=min(OUTLIER_CHANNELS, K), replace=False))


def activations(M: int, K: int, seed: int, heavy_tailed: bool = True) -> np.ndarray:
    """bf16 bits [M, K] of VGGT-like activations (see module docstring)."""
    rng = np.random.Generator(np.random.PCG64([seed, 0xA11]))
    x = rng.standard_normal((M, K), dtype=np.float32)
    if heavy_tailed:
        x[special_rows(M)] *= np.float32(SPECIAL_SCALE)
        x[:, outlier_channels(K, seed)] *= np.float32(OUTLIER_SCALE)
    return to_bf16_bits(x)


def activations_device(M: int, K: int, seed: int, device, heavy_tailed: bool = True):
    """The same recipe as activations() drawn on a CUDA device with torch's
    generator (other random numbers, same distribution and structure): a
    torch.bfloat16 tensor [M, K].  For workloads whose inputs are too large to
    draw on the host (a fresh activation batch for each of a stack's layers)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 7919 + 0xA11)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if heavy_tailed:
        rows = torch.from_numpy(special_rows(M)).to(device)
        x[rows] *= SPECIAL_SCALE
        x[:, torch.from_numpy(outlier_channels(K, seed)).to(device)] *= OUTLIER_SCALE
    return x.to(torch.bfloat16)


def weights_device(N: int, K: int, seed: int, device, std: float = 0.02):
    """weights() drawn on a CUDA device (torch's generator): bf16 [N, K]."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 7919 + 0x3E1)
    return (torch.randn((N, K), generator=g, device=device) * std).to(torch.bfloat16)


def bias_device(N: int, seed: int, device, std: float = 0.01):
    """bias() drawn on a CUDA device (torch's generator): bf16 [N]."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 7919 + 0xB1A5)
    return (torch.randn(N, generator=g, device=device) * std).to(torch.bfloat16)


def weights(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64([seed, 0x3E1]))
    return to_bf16_bits(rng.standard_normal((N, K), dtype=np.float32) * np.float32(std))


def bias(N: int, seed: int, std: float = 0.01) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64([seed, 0xB1A5]))
    return to_bf16_bits(rng.standard_normal(N, dtype=np.float32) * np.float32(std))


def random_packed_codes(rows: int, K: int, seed: int) -> np.ndarray:
    """Uniform random bytes [rows, K/2]: every nibble is a uniform int4 code.
    Used to drive the integer GEMM with identical codes on both sides."""
    rng = np.random.Generator(np.random.PCG64([seed, 0xC0DE]))
    return rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)


def random_scales(n: int, seed: int, lo: float = 1e-3, hi: float = 1e-1) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64([seed, 0x5CA1]))
    return rng.uniform(lo, hi, size=n).astype(np.float32)


def calibration_rows(M: int) -> int:
    """Rows of a layer's own activations used as its calibration batch: the
    first frame (all rows when M is at most one frame)."""
    return min(M, FRAME_TOKENS)


# Workloads from the benchmark configuration list (token counts are frames x 1374).
CONFIGS = {
    "c1_single_linear": dict(frames=1, layers=[("linear", 1024, 1024)]),
    "c2_frame_qkv": dict(frames=8, layers=[("qkv", 1024, 3072)]),
    "c3_mlp_pair": dict(frames=8, layers=[("fc1", 1024, 4096), ("fc2", 4096, 1024)]),
    "c4_global_block": dict(frames=32, layers=[("qkv", 1024, 3072), ("proj", 1024, 1024),
                                               ("fc1", 1024, 4096), ("fc2", 4096, 1024)]),
    "c5_full_stack": dict(frames=64, blocks=48,
                          layers=[("qkv", 1024, 3072), ("proj", 1024, 1024),
                                  ("fc1", 1024, 4096), ("fc2", 4096, 1024)]),
}


# KV-cache vectors for the 3DTurboQuant codec (page "3DTurboQuant: Training-
# Free Near-Optimal Quantization for 3D Reconstruction Models", section 4.2:
# the DUSt3R KV cache, d = 1024, about 100 MB in fp32 = 24576 vectors).
KV_DIM = 1024
KV_VECTORS = 24576


def kv_vectors(n: int, d: int, seed: int) -> np.ndarray:
    """fp32 [n, d] KV-like vectors: N(0, 1) entries, 8 seeded outlier channels
    x15, and a per-vector scale drawn log-uniformly from [0.25, 4]."""
    rng = np.random.Generator(np.random.PCG64([seed, 0x4B56]))
    x = rng.standard_normal((n, d), dtype=np.float32)
    x[:, outlier_channels(d, seed)] *= np.float32(OUTLIER_SCALE)
    x *= np.exp(rng.uniform(np.log(0.25), np.log(4.0), size=(n, 1))).astype(np.float32)
    return x


def gaussian_matrix(d: int, seed: int) -> np.ndarray:
    """fp64 [d, d] of independent standard normal entries (the Gaussian matrix
    whose QR factor is a random rotation)."""
    rng = np.random.Generator(np.random.PCG64([seed, 0x6A55]))
    return rng.standard_normal((d, d))


def random_signs(d: int, seed: int) -> np.ndarray:
    """fp32 [d] of independent +-1 (the random sign vector of a rotation)."""
    rng = np.random.Generator(np.random.PCG64([seed, 0x516E]))
    return np.where(rng.random(d) < 0.5, np.float32(-1.0), np.float32(1.0)).astype(np.float32)

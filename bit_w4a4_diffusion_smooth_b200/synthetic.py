"""Seeded synthetic inputs for the SVDQuant W4A4 linear and the AWQ W4A16 projection.

This module holds input generation only: random draws, outlier placement and
the rounding of the draws to bf16.  It contains none of the layer's
arithmetic, so both the CUDA path and the CPU checker can take their inputs
from it.

The pages measure a 12B-class diffusion transformer at 1024x1024 (4096 image
tokens plus 512 text tokens) whose weights are not available here; these
generators stand in for its activations and weights with the same shapes and
with the outlier structure the pages describe: a few activation channels and a
few weight rows far larger than the rest ([Donmalab] "量化的核心挑戰：為什麼
4-bit 很難？"; [Remio] "SVDQuant 将棘手数值移出 4 位路径").

Recipe (all draws float64, then rounded once to float32 and RNE to bf16):
  activation X [M, K]  ~ N(0, 1); ceil(frac*K) channels chosen without
                          replacement are multiplied by `factor`
  weight W [K, N]      ~ N(0, std); ceil(frac*K) rows chosen without
                          replacement are multiplied by `factor`
  bias b [N]           ~ N(0, 0.01)
  AWQ scale a [K]      ~ LogUniform(0.5, 4) = exp(U(ln 0.5, ln 4)), float32
Each array takes its own child stream of numpy's SeedSequence(seed).
"""
import math
from dataclasses import dataclass, field

import numpy as np


def _f32_to_bf16_bits(x32):
    """RNE float32 -> bf16 bit patterns (uint16); inputs here are finite."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits):
    """Exact float32 value of bf16 bit patterns."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _streams(seed, n):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


def activation(m, k, seed, outlier_channels=0, factor=1.0, stream=0):
    """X [m, k] as bf16 bits; returns (bits uint16, outlier channel indices)."""
    g = _streams(seed, 8)[stream]
    x = g.standard_normal((m, k))
    idx = np.sort(g.choice(k, size=outlier_channels, replace=False)) if outlier_channels else \
        np.zeros(0, dtype=np.int64)
    x[:, idx] *= factor
    return _f32_to_bf16_bits(x.astype(np.float32)), idx


def weight(k, n, seed, std=0.02, outlier_rows=0, factor=1.0, stream=1):
    """W [k, n] as bf16 bits; returns (bits uint16, outlier row indices)."""
    g = _streams(seed, 8)[stream]
    w = g.standard_normal((k, n)) * std
    idx = np.sort(g.choice(k, size=outlier_rows, replace=False)) if outlier_rows else \
        np.zeros(0, dtype=np.int64)
    w[idx, :] *= factor
    return _f32_to_bf16_bits(w.astype(np.float32)), idx


def bias(n, seed, std=0.01, stream=2):
    g = _streams(seed, 8)[stream]
    return _f32_to_bf16_bits((g.standard_normal(n) * std).astype(np.float32))


def awq_scales(k, seed, lo=0.5, hi=4.0, stream=3):
    g = _streams(seed, 8)[stream]
    return np.exp(g.uniform(math.log(lo), math.log(hi), size=k)).astype(np.float32)


def count(frac, k):
    return int(math.ceil(frac * k - 1e-9))


@dataclass
class LinearCase:
    """One SVDQ W4A4 linear: X [m, k] -> Y [m, n], rank r."""
    name: str
    m: int
    k: int
    n: int
    rank: int
    seed: int
    x_outlier_channels: int = 0
    x_factor: float = 1.0
    w_outlier_rows: int = 0
    w_factor: float = 1.0
    gelu: bool = False
    gelu_col_begin: int = 0
    with_bias: bool = True

    def make(self):
        x, _ = activation(self.m, self.k, self.seed, self.x_outlier_channels, self.x_factor)
        w, _ = weight(self.k, self.n, self.seed, 0.02, self.w_outlier_rows, self.w_factor)
        b = bias(self.n, self.seed) if self.with_bias else None
        return x, w, b


@dataclass
class AwqCase:
    name: str
    m: int
    k: int
    n: int
    seed: int
    group: int = 64

    def make(self):
        x, _ = activation(self.m, self.k, self.seed)
        w, _ = weight(self.k, self.n, self.seed, 0.02)
        return x, w, bias(self.n, self.seed), awq_scales(self.k, self.seed)


# The five workloads.  Token count 4608 = 4096 image tokens (a 1024x1024 image
# in a 16x16-patch latent) + 512 text tokens.
TINY = LinearCase("tiny 64x256x256 r16", 64, 256, 256, 16, seed=0,
                  x_outlier_channels=4, x_factor=30.0)
QKV = LinearCase("attention QKV 4608x3072x9216 r32", 4608, 3072, 9216, 32, seed=1,
                 x_outlier_channels=count(0.01, 3072), x_factor=50.0,
                 w_outlier_rows=count(0.005, 3072), w_factor=8.0)
MLP_FC1 = LinearCase("MLP fc1 4608x3072x12288 r32 +GELU", 4608, 3072, 12288, 32, seed=2,
                     x_outlier_channels=count(0.01, 3072), x_factor=50.0,
                     w_outlier_rows=count(0.005, 3072), w_factor=8.0, gelu=True)
# fc2 takes fc1's GELU output as its activation; only its weight is drawn here.
MLP_FC2 = LinearCase("MLP fc2 4608x12288x3072 r32", 4608, 12288, 3072, 32, seed=2,
                     w_outlier_rows=count(0.005, 12288), w_factor=8.0)
AWQ = AwqCase("AWQ adaLN 2x3072x18432 g64", 2, 3072, 18432, seed=3)


@dataclass
class DitStep:
    """All projection linears of one denoising step of a 12B-class DiT."""
    dual_blocks: int = 19
    single_blocks: int = 38
    hidden: int = 3072
    img_tokens: int = 4096
    txt_tokens: int = 512
    mlp: int = 12288
    rank: int = 32
    seed: int = 4
    layers: list = field(default_factory=list)

    def __post_init__(self):
        h, t = self.hidden, self.img_tokens + self.txt_tokens
        for stream, m in (("img", self.img_tokens), ("txt", self.txt_tokens)):
            for name, k, n, gelu in (("qkv", h, 3 * h, False), ("out", h, h, False),
                                     ("fc1", h, self.mlp, True), ("fc2", self.mlp, h, False)):
                self.layers.append((f"dual.{stream}.{name}", m, k, n, gelu, 0, self.dual_blocks))
        # single-stream block: fused QKV + MLP-in (GELU on the MLP columns only)
        self.layers.append(("single.qkv_mlp", t, h, 3 * h + self.mlp, True, 3 * h,
                            self.single_blocks))
        self.layers.append(("single.out", t, h + self.mlp, h, False, 0, self.single_blocks))
        self.awq_layers = [("dual.adaln", 2, h, 6 * h, 2 * self.dual_blocks),
                           ("single.adaln", 2, h, 3 * h, self.single_blocks)]

    def w4a4_flops(self):
        return sum(2 * m * k * n * cnt for _, m, k, n, _, _, cnt in self.layers)

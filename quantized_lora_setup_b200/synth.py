"""Seeded synthetic weights with the shapes of the benchmark models.

This module only draws random numbers: it holds no part of the NF4 arithmetic, so the
tests may feed the same bytes to the CUDA library and to the CPU oracle.

Workloads (layer shapes are (out_features, in_features), stored row-major):

* ``tiny``  4 blocks x 7 linears (q,k,v,o 256x256; gate,up 688x256; down 256x688), fp16
  N(0, 0.02); two layers, drawn with the seed, Student-t nu=3 rescaled to std 0.02;
  K = 2, no byte budget.
* ``1.4b``  24 blocks x (fused qkv 6144x2048, o 2048x2048, up 8192x2048, down 2048x8192),
  fp16; per-layer std U(0.01, 0.04); 10 % of the layers Student-t nu=3 at that std;
  budget 0.2 GiB.
* ``7b``    32 blocks x (q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008), bf16
  N(0, s) with s = 0.01 + 0.02 * block / 31; 0.1 % of the input columns scaled by 20;
  budget 1 GiB.
* ``14b``   40 blocks x (q,o 5120x5120; k,v 1024x5120; gate,up 13824x5120; down
  5120x13824), bf16; per layer a seeded coin picks N(0, 0.02) or Student-t nu=4 rescaled
  to std 0.02; budgets 0.2, 1 and 4 GiB.

A Student-t variate is drawn as Z / sqrt(chi2_nu / nu) with chi2_nu a sum of nu squared
standard normals, so both the numpy (host) and the torch (device) generators need only
normal draws.  Layer ``l`` of a workload with seed ``s`` uses the stream
``s * 1000 + l``; the host and device streams differ, so a test always copies the exact
bytes one side saw to the other.
"""
from dataclasses import dataclass
from typing import List, Tuple

import numpy as np
import torch

GIB = 1 << 30


@dataclass(frozen=True)
class LayerSpec:
    name: str
    rows: int
    cols: int
    dtype: torch.dtype
    dist: str = "normal"        # "normal" | "t"
    sigma: float = 0.02
    nu: int = 0
    outlier_cols: Tuple[int, ...] = ()
    outlier_factor: float = 1.0

    @property
    def numel(self) -> int:
        return self.rows * self.cols


@dataclass(frozen=True)
class Workload:
    name: str
    layers: Tuple[LayerSpec, ...]
    budgets: Tuple[int, ...]
    k_cap: int = -1
    seed: int = 0

    @property
    def numel(self) -> int:
        return sum(l.numel for l in self.layers)

    @property
    def weight_bytes(self) -> int:
        return 2 * self.numel


def _blocks(prefix_shapes, nblocks):
    return [(f"blk{b}.{n}", r, c) for b in range(nblocks) for (n, r, c) in prefix_shapes]


def block_index(wl: Workload) -> List[int]:
    """Transformer block of every layer ("blk<b>.<name>"), for the block-level selection."""
    return [int(l.name.split(".", 1)[0][3:]) for l in wl.layers]


def tiny(seed: int = 0) -> Workload:
    shapes = _blocks([("q", 256, 256), ("k", 256, 256), ("v", 256, 256), ("o", 256, 256),
                      ("gate", 688, 256), ("up", 688, 256), ("down", 256, 688)], 4)
    rng = np.random.default_rng([seed, 1])
    heavy = set(rng.choice(len(shapes), size=2, replace=False).tolist())
    layers = tuple(
        LayerSpec(n, r, c, torch.float16, "t" if i in heavy else "normal", 0.02, 3 if i in heavy else 0)
        for i, (n, r, c) in enumerate(shapes))
    total = sum(2 * l.numel for l in layers)
    return Workload("tiny", layers, (total,), k_cap=2, seed=seed)


def model_1p4b(seed: int = 0) -> Workload:
    shapes = _blocks([("qkv", 6144, 2048), ("o", 2048, 2048), ("up", 8192, 2048),
                      ("down", 2048, 8192)], 24)
    rng = np.random.default_rng([seed, 2])
    sig = rng.uniform(0.01, 0.04, len(shapes))
    heavy = set(rng.choice(len(shapes), size=round(0.1 * len(shapes)), replace=False).tolist())
    layers = tuple(
        LayerSpec(n, r, c, torch.float16, "t" if i in heavy else "normal", float(sig[i]),
                  3 if i in heavy else 0)
        for i, (n, r, c) in enumerate(shapes))
    return Workload("1.4b", layers, (int(0.2 * GIB),), seed=seed)


def model_7b(seed: int = 0) -> Workload:
    per_block = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                 ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
    rng = np.random.default_rng([seed, 3])
    layers = []
    for b in range(32):
        sigma = 0.01 + 0.02 * b / 31
        for (n, r, c) in per_block:
            k = max(1, round(0.001 * c))
            cols = tuple(sorted(rng.choice(c, size=k, replace=False).tolist()))
            layers.append(LayerSpec(f"blk{b}.{n}", r, c, torch.bfloat16, "normal", sigma, 0,
                                    cols, 20.0))
    return Workload("7b", tuple(layers), (1 * GIB,), seed=seed)


def model_14b(seed: int = 0) -> Workload:
    shapes = _blocks([("q", 5120, 5120), ("k", 1024, 5120), ("v", 1024, 5120), ("o", 5120, 5120),
                      ("gate", 13824, 5120), ("up", 13824, 5120), ("down", 5120, 13824)], 40)
    rng = np.random.default_rng([seed, 4])
    coin = rng.integers(0, 2, len(shapes))
    layers = tuple(
        LayerSpec(n, r, c, torch.bfloat16, "t" if coin[i] else "normal", 0.02, 4 if coin[i] else 0)
        for i, (n, r, c) in enumerate(shapes))
    return Workload("14b", layers, (int(0.2 * GIB), 1 * GIB, 4 * GIB), seed=seed)


WORKLOADS = {"tiny": tiny, "1.4b": model_1p4b, "7b": model_7b, "14b": model_14b}

# Standalone dequantization: matrices from 4096x4096 up to 28672x8192, N(0, 0.02) source.
DEQUANT_SHAPES = [(4096, 4096), (4096, 11008), (8192, 8192), (14336, 4096), (28672, 8192)]


def workload(name: str, seed: int = 0) -> Workload:
    return WORKLOADS[name](seed)


def _t_scale(nu: int) -> float:
    # a Student-t variate with nu > 2 has variance nu / (nu - 2)
    return float(np.sqrt((nu - 2) / nu))


def layer_host(spec: LayerSpec, seed: int, index: int) -> torch.Tensor:
    """The layer's weights on the host (CPU tensor of spec.dtype, shape (rows, cols))."""
    rng = np.random.default_rng(seed * 1000 + index)
    z = rng.standard_normal((spec.rows, spec.cols), dtype=np.float32)
    if spec.dist == "t":
        chi2 = np.zeros_like(z)
        for _ in range(spec.nu):
            chi2 += rng.standard_normal((spec.rows, spec.cols), dtype=np.float32) ** 2
        z = z / np.sqrt(chi2 / spec.nu) * _t_scale(spec.nu)
    z = z * np.float32(spec.sigma)
    if spec.outlier_cols:
        z[:, list(spec.outlier_cols)] *= np.float32(spec.outlier_factor)
    return torch.from_numpy(z).to(spec.dtype)


def layer_device(spec: LayerSpec, seed: int, index: int, device="cuda") -> torch.Tensor:
    """The layer's weights drawn directly on the device (a different stream than layer_host)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + index)
    shape = (spec.rows, spec.cols)
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if spec.dist == "t":
        chi2 = torch.zeros_like(z)
        for _ in range(spec.nu):
            chi2.add_(torch.randn(shape, generator=g, device=device, dtype=torch.float32).square_())
        z.div_(chi2.div_(spec.nu).sqrt_()).mul_(_t_scale(spec.nu))
        del chi2
    z.mul_(spec.sigma)
    if spec.outlier_cols:
        idx = torch.tensor(spec.outlier_cols, device=device)
        z[:, idx] *= spec.outlier_factor
    return z.to(spec.dtype)


def normal_matrix_device(rows: int, cols: int, seed: int, sigma: float = 0.02,
                         dtype=torch.bfloat16, device="cuda") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty((rows, cols), dtype=dtype, device=device)
    step = max(1, (1 << 26) // cols)  # bounded fp32 temporaries
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = (torch.randn((r1 - r0, cols), generator=g, device=device) * sigma).to(dtype)
    return out


def random_bits_host(n: int, seed: int, dtype=torch.bfloat16, sigma: float = 0.02) -> torch.Tensor:
    """n normal weights on the host as a flat tensor (for ragged sizes in tests)."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(n, dtype=np.float32) * np.float32(sigma)
    return torch.from_numpy(z).to(dtype)


def bits_u16(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a 16-bit CPU tensor (for the oracle)."""
    t = t.detach().contiguous().cpu().reshape(-1)
    return t.view(torch.int16).numpy().view(np.uint16)


__all__ = ["GIB", "LayerSpec", "Workload", "block_index", "tiny", "model_1p4b", "model_7b", "model_14b",
           "WORKLOADS", "DEQUANT_SHAPES", "workload", "layer_host", "layer_device",
           "normal_matrix_device", "random_bits_host", "bits_u16"]

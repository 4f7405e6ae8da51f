"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module only makes inputs: random BF16 weight matrices shaped like the
MLP projections of a Llama-3.1-8B-class model, activations, and a few
structured matrices for edge cases.  It holds none of the compression
method's arithmetic (no palette, no Huffman code, no rebuild), so the CPU
oracle and the CUDA path can both draw from it without sharing any of the
computation they are compared on.

Every array is BF16 carried as its raw 16-bit pattern in ``numpy.uint16``.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "weight_matrix",
    "activations",
    "all_patterns_matrix",
    "small_integer_matrix",
    "WORKLOADS",
    "stack_sigmas",
    "stack_layer",
    "stack_layer_device",
    "weight_matrix_device",
]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (round to nearest, ties to even).

    Only finite inputs are produced by the generators below; NaN is kept a
    quiet NaN for completeness.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = ((u[nan] >> np.uint64(16)) | np.uint64(0x40)).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def weight_matrix(rows: int, cols: int, sigma: float, outlier_rate: float,
                  outlier_scale: float, seed: int) -> np.ndarray:
    """N(0, sigma) weights in BF16 with a sparse set of scaled outliers.

    Recipe: ``rng = default_rng(seed)``; ``w = standard_normal(float32) *
    sigma``; entries with ``rng.random() < outlier_rate`` are multiplied by
    ``outlier_scale``; then RNE to BF16.  The outliers carry exponents that
    fall outside a top-16 palette, which is what forces whole 64-element
    rows to be stored verbatim.
    """
    rng = np.random.default_rng(seed)
    n = rows * cols
    w = rng.standard_normal(n, dtype=np.float32) * np.float32(sigma)
    if outlier_rate > 0:
        mask = rng.random(n) < outlier_rate
        w[mask] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(w).reshape(rows, cols)


def activations(batch: int, cols: int, seed: int) -> np.ndarray:
    """Token activations x[batch, cols] ~ N(0, 1), rounded to BF16."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal((batch, cols), dtype=np.float32))


def all_patterns_matrix(rows: int = 1024, cols: int = 64) -> np.ndarray:
    """Every one of the 65536 BF16 bit patterns exactly once (±0, subnormals,
    ±Inf, every NaN payload), shuffled with a fixed seed so that rare and
    common exponents share 64-element rows."""
    assert rows * cols == 65536
    v = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    np.random.default_rng(7).shuffle(v)
    return v.reshape(rows, cols)


def small_integer_matrix(rows: int, cols: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Integers drawn uniformly from [lo, hi], as BF16 (exact for |v| <= 256)."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.integers(lo, hi + 1, size=(rows, cols)).astype(np.float32))


def stack_sigmas(n_layers: int = 32) -> np.ndarray:
    """Per-layer sigma for the 32-layer stack: uniform in [0.01, 0.05]."""
    return np.random.default_rng(1000).uniform(0.01, 0.05, n_layers)


# Named workloads.  Shapes follow Llama-3.1-8B's MLP: d_model 4096,
# ffn 14336; gate/up are [14336, 4096] (out x in), down is [4096, 14336].
WORKLOADS = {
    # 256x512 matrix, 0.05% outliers x200, batch 4: the small parity case.
    "small_256x512": dict(rows=256, cols=512, sigma=0.02, outlier_rate=5e-4,
                          outlier_scale=200.0, seed=0, batch=4),
    # gate_proj-shaped decode-throughput case.
    "gate_14336x4096": dict(rows=14336, cols=4096, sigma=0.02, outlier_rate=1e-4,
                            outlier_scale=100.0, seed=1),
    # One SwiGLU MLP block (gate, up, down) at seeds seed, seed+10, seed+20.
    "mlp_block_4096_14336": dict(d_model=4096, ffn=14336, sigma=0.02, outlier_rate=1e-4,
                                 outlier_scale=100.0, seed=2),
}


def stack_layer(layer: int, n_layers: int = 32, d_model: int = 4096, ffn: int = 14336,
                outlier_rate: float = 1e-3, outlier_scale: float = 100.0):
    """Layer `layer` of the 32-layer MLP stack: gate [ffn, d], up [ffn, d],
    down [d, ffn] with the layer's sigma and seeds 2000 + 3*layer + j."""
    sigma = float(stack_sigmas(n_layers)[layer])
    seed = 2000 + 3 * layer
    return (weight_matrix(ffn, d_model, sigma, outlier_rate, outlier_scale, seed),
            weight_matrix(ffn, d_model, sigma, outlier_rate, outlier_scale, seed + 1),
            weight_matrix(d_model, ffn, sigma, outlier_rate, outlier_scale, seed + 2))


def weight_matrix_device(rows: int, cols: int, sigma: float, outlier_rate: float, outlier_scale: float,
                         seed: int, device):
    """`weight_matrix`'s recipe drawn on a torch device with torch's
    generator seeded `seed` (so the values differ from `weight_matrix`'s):
    N(0, sigma), entries below `outlier_rate` in a uniform draw scaled by
    `outlier_scale`, RNE to BF16.  Returns an int16 tensor of the BF16
    patterns.  For the timed cases that need many or large matrices
    quickly; every parity case uses `weight_matrix`."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * sigma
    if outlier_rate > 0:
        mask = torch.rand(rows, cols, generator=g, device=device) < outlier_rate
        w = torch.where(mask, w * outlier_scale, w)
    return w.to(torch.bfloat16).view(torch.int16)


def stack_layer_device(layer: int, device, n_layers: int = 32, d_model: int = 4096, ffn: int = 14336,
                       outlier_rate: float = 1e-3, outlier_scale: float = 100.0):
    """Layer `layer` of the 32-layer stack drawn on a torch device
    (`weight_matrix_device` with the layer's sigma and seeds
    2000 + 3*layer + j): gate, up, down as int16 tensors."""
    sigma = float(stack_sigmas(n_layers)[layer])
    shapes = ((ffn, d_model), (ffn, d_model), (d_model, ffn))
    return tuple(weight_matrix_device(r, c, sigma, outlier_rate, outlier_scale, 2000 + 3 * layer + j, device)
                 for j, (r, c) in enumerate(shapes))


def mlp_block(d_model: int = 4096, ffn: int = 14336, sigma: float = 0.02,
              outlier_rate: float = 1e-4, outlier_scale: float = 100.0, seed: int = 2):
    """gate [ffn, d], up [ffn, d], down [d, ffn] at seeds seed, seed+10, seed+20."""
    gate = weight_matrix(ffn, d_model, sigma, outlier_rate, outlier_scale, seed)
    up = weight_matrix(ffn, d_model, sigma, outlier_rate, outlier_scale, seed + 10)
    down = weight_matrix(d_model, ffn, sigma, outlier_rate, outlier_scale, seed + 20)
    return gate, up, down

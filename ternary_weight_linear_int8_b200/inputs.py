"""Seeded synthetic inputs for the W1.58A8 BitLinear path.

This module only draws random numbers and shapes them into the workloads; it
holds none of the method's arithmetic (no quantisation, no packing, no
matmul).  Both the CUDA path and the CPU oracle are fed the same bytes from
here, so a parity test compares the two on identical inputs.

Recipe (every workload):
  * ``rng = numpy.random.default_rng(seed)`` (PCG64);
  * activations ``x = rng.standard_normal(shape, float32)``, optionally with
    outlier channels scaled by 20, then rounded to bfloat16 (round to nearest
    even, done by torch's CPU cast) and returned as the raw uint16 bit
    patterns;
  * weights ``W = rng.standard_normal((N, K), float32) * 0.02`` (fp32,
    out x in, row-major like ``nn.Linear``).

Seeds: the small single-layer case draws x then W from seed 0; elsewhere the
activations use seed 0 and weight matrix ``l`` uses seed ``1000 + l``.
"""
from __future__ import annotations

import numpy as np
import torch

WEIGHT_SIGMA = np.float32(0.02)
OUTLIER_FRACTION = 0.01
OUTLIER_GAIN = np.float32(20.0)


def to_bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (torch CPU cast, nearest-even) and return uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def activations(shape, seed: int = 0, outliers: bool = False,
                rng: np.random.Generator | None = None) -> np.ndarray:
    """bf16 activations ~N(0,1) as uint16 bits, shape ``[M, K]``.

    With ``outliers`` a seed-chosen set of ``round(0.01*K)`` channels (the same
    channels for every token) is scaled by 20 before the bf16 rounding.
    """
    rng = np.random.default_rng(seed) if rng is None else rng
    M, K = shape
    x = rng.standard_normal((M, K), dtype=np.float32)
    if outliers:
        n_out = int(round(OUTLIER_FRACTION * K))
        ch = rng.choice(K, size=n_out, replace=False)
        x[:, ch] *= OUTLIER_GAIN
    return to_bf16_bits(x)


def weights(N: int, K: int, seed: int = 1000,
            rng: np.random.Generator | None = None) -> np.ndarray:
    """fp32 weights ~N(0, 0.02), shape ``[N, K]``."""
    rng = np.random.default_rng(seed) if rng is None else rng
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= WEIGHT_SIGMA
    return w


def single_layer(M: int = 8, K: int = 512, N: int = 400, seed: int = 0):
    """The small single BitLinear case: x [8,512], W [400,512], one seed, x first."""
    rng = np.random.default_rng(seed)
    x = activations((M, K), rng=rng)
    w = weights(N, K, rng=rng)
    return x, w


def layer_seed(layer: int) -> int:
    return 1000 + layer


# Workload shapes (sizes only; the arithmetic lives elsewhere).
DECODE_2B = {"hidden": 2560, "inter": 6912, "layers": 30}
FFN_100B = {"hidden": 8192, "inter": 28672}
BATCHED_DECODE_M = (1, 4, 16, 64)
PREFILL_M = 4096

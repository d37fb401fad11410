"""Seeded synthetic inputs for the BitStack residual-block linear.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It only draws random numbers and names shapes: it holds no step of the
method's arithmetic (no scaling statistic, no decomposition, no packing, no
reconstruction).  Every draw comes from ``numpy.random.default_rng`` seeded with
``(1000 * config + matrix, stream)`` so that each kind of input has its own stream.

Shapes follow the workloads the pages evaluate on: Llama-3-8B linears
(q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096, down 4096x14336), k = 16 kept
singular vectors, and 16 decomposition iterations per weight (README of BitStack,
"Decomposition" command: ``--niter 16 --k 16``).  The pages measure on trained Llama
checkpoints and public text corpora, which are not available here; the Gaussian
weights with outlier input channels below stand in for them.
"""
from __future__ import annotations

import numpy as np

STREAMS = {
    "W": 0,          # weight matrix entries
    "outlier": 1,    # which input channels are outliers
    "calib": 2,      # calibration activations
    "x": 3,          # layer inputs
    "n": 4,          # per-matrix loaded block counts
    "blocks": 5,     # synthetic residual blocks (signs and factors)
    "order": 6,      # per-matrix importance weights for the global block order
    "svd": 7,        # random test matrices for randomized SVD
    "plan": 8,       # residual-norm decay per block for load-order planning
}

K_DEFAULT = 16

# Llama-3-8B linear shapes, (out_features, in_features) per kind, per decoder layer.
LLAMA3_8B_LINEARS = (
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
)
LLAMA3_8B_LAYERS = 32


def generator(config: int, matrix: int = 0, stream: str = "W") -> np.random.Generator:
    """The seeded generator for one kind of draw of one matrix of one config."""
    return np.random.default_rng([1000 * int(config) + int(matrix), STREAMS[stream]])


def weight(m: int, d: int, gen: np.random.Generator, std: float = 0.02,
           outlier_frac: float = 0.0, outlier_scale: float = 10.0,
           outlier_gen: np.random.Generator | None = None) -> np.ndarray:
    """A float32 m x d weight with N(0, std^2) entries.

    When ``outlier_frac`` > 0, round(outlier_frac * d) input channels (columns),
    picked without replacement from ``outlier_gen``, are multiplied by
    ``outlier_scale``.
    """
    W = gen.standard_normal((m, d), dtype=np.float64) * std
    if outlier_frac > 0.0:
        count = int(round(outlier_frac * d))
        og = outlier_gen if outlier_gen is not None else gen
        cols = og.choice(d, size=count, replace=False)
        W[:, cols] *= outlier_scale
    return W.astype(np.float32)


def calibration(rows: int, d: int, gen: np.random.Generator) -> np.ndarray:
    """float32 calibration activations, rows x d, N(0, 1)."""
    return gen.standard_normal((rows, d), dtype=np.float64).astype(np.float32)


def activations(b: int, d: int, gen: np.random.Generator) -> np.ndarray:
    """float32 layer inputs, b x d, N(0, 1); callers round them to fp16 or bf16."""
    return gen.standard_normal((b, d), dtype=np.float64).astype(np.float32)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even); returns uint16 bits.

    A storage-format conversion (IEEE round to nearest even on the upper 16 bits),
    not part of the method.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def random_signs(m: int, d: int, gen: np.random.Generator) -> np.ndarray:
    """A uniformly random m x d boolean matrix; True marks a -1 entry."""
    return gen.integers(0, 2, size=(m, d), dtype=np.uint8).astype(bool)


def random_factors(rows: int, k: int, gen: np.random.Generator, std: float) -> np.ndarray:
    """An fp16 rows x k matrix with N(0, std^2) entries."""
    return (gen.standard_normal((rows, k), dtype=np.float64) * std).astype(np.float16)


def synthetic_block(m: int, d: int, k: int, gen: np.random.Generator, level: int = 0):
    """One synthetic residual block: (neg signs m x d, U fp16 m x k, V fp16 d x k).

    The factor scale shrinks with the block's level, as the residual a decomposition
    works on shrinks from one iteration to the next: std = 0.12 / sqrt(level + 1).
    Used wherever only the block's shape and byte count matter (timing) or where the
    oracle is evaluated on the same blocks (parity on large stacks).
    """
    std = 0.12 / np.sqrt(level + 1.0)
    neg = random_signs(m, d, gen)
    U = random_factors(m, k, gen, std)
    V = random_factors(d, k, gen, std)
    return neg, U, V


def synthetic_inv_scale(d: int, gen: np.random.Generator) -> np.ndarray:
    """float32 per-input-channel inverse scales near 1 (a calibration-like spread)."""
    return (1.0 / np.sqrt(gen.chisquare(64, size=d) / 64.0)).astype(np.float32)


def n_loaded_draws(count: int, gen: np.random.Generator, lo: int = 2, hi: int = 12) -> np.ndarray:
    """Per-matrix loaded block counts drawn uniformly from lo..hi inclusive."""
    return gen.integers(lo, hi + 1, size=count)


def order_weights(count: int, gen: np.random.Generator) -> np.ndarray:
    """Per-matrix importance weights a ~ U(0.5, 1.5) for the stand-in global order."""
    return gen.uniform(0.5, 1.5, size=count)


def llama3_8b_matrices(layers: int = LLAMA3_8B_LAYERS):
    """[(layer, kind, m, d)] for every linear of the decoder stack, layer-major."""
    return [(layer, kind, m, d) for layer in range(layers) for (kind, m, d) in LLAMA3_8B_LINEARS]

"""Seeded synthetic operands shaped like Llama-3.1-8B projection and attention inputs.

This module only draws inputs. It holds none of the pruning, quantization or
energy arithmetic, so both the CUDA path and the CPU oracle can be fed the
same bytes from it. Every generator uses ``numpy.random.default_rng(seed)``,
draws in float32 and rounds to bf16 with round-to-nearest-even (bf16 arrays are
returned as their raw ``uint16`` bit patterns).

The workloads restate the operand families that "Is 2:4 Sparsity Still Worth
It? Semi-Structured Sparsity versus Quantization in LLM Inference" compares
(intro: linear-layer weights and inputs, attention Q, K, V and probabilities
P; §3: projections over 2K to 16K tokens). No dataset or trained weight is
used; these draws stand in for them.
"""
from __future__ import annotations

import numpy as np


def bf16_bits(f32: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def gaussian_f32(rows: int, k: int, seed: int = 0) -> np.ndarray:
    """i.i.d. N(0, 1) float32 matrix [rows, k]."""
    return np.random.default_rng(seed).standard_normal((rows, k), dtype=np.float32)


def gaussian_bf16(rows: int, k: int, seed: int = 0, std: float = 1.0) -> np.ndarray:
    """i.i.d. N(0, std^2) matrix [rows, k] rounded to bf16."""
    x = np.random.default_rng(seed).standard_normal((rows, k), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return bf16_bits(x)


def linear_input(tokens: int = 4096, k: int = 4096, seed: int = 1, n_outlier: int = 8,
                 outlier_factor: float = 50.0, outlier_seed: int = 1234):
    """Linear-layer input X [tokens, k]: Student-t with nu = 4 scaled by 1/sqrt(2)
    (unit variance), with ``n_outlier`` fixed channels (drawn once from
    ``outlier_seed`` without replacement) multiplied by ``outlier_factor``
    before the bf16 rounding. Returns (bf16 bits, outlier channel indices)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4.0, size=(tokens, k)).astype(np.float32) / np.float32(np.sqrt(2.0))
    chans = np.sort(np.random.default_rng(outlier_seed).choice(k, size=n_outlier, replace=False))
    x[:, chans] *= np.float32(outlier_factor)
    return bf16_bits(x), chans


def linear_weight(out_features: int = 14336, k: int = 4096, seed: int = 2, norm_seed: int = 3):
    """Linear-layer weight W [out_features, k] ~ N(0, 0.02^2) in bf16, and the
    Wanda input-channel norms n [k] = exp(N(0, 1)) in float32."""
    w = gaussian_bf16(out_features, k, seed=seed, std=0.02)
    norms = np.exp(np.random.default_rng(norm_seed).standard_normal(k)).astype(np.float32)
    return w, norms


def attention_qkv(heads: int = 32, seq: int = 8192, d: int = 128, seed: int = 4) -> np.ndarray:
    """One of Q, K or V: [heads * seq, d] ~ N(0, 1) in bf16, pruned along d."""
    return gaussian_bf16(heads * seq, d, seed=seed)


def attention_probs(heads: int = 32, seq: int = 2048, d: int = 128, seed: int = 7,
                    logit_std: float = 3.0) -> np.ndarray:
    """Attention probabilities P [heads * seq, seq]: logits ~ N(0, logit_std^2)
    divided by sqrt(d), softmax over the key axis in float32, rounded to bf16."""
    rng = np.random.default_rng(seed)
    out = np.empty((heads * seq, seq), dtype=np.uint16)
    step = 4096
    for r0 in range(0, heads * seq, step):
        rr = min(step, heads * seq - r0)
        z = rng.standard_normal((rr, seq), dtype=np.float32) * np.float32(logit_std / np.sqrt(d))
        z -= z.max(axis=1, keepdims=True)
        np.exp(z, out=z)
        z /= z.sum(axis=1, keepdims=True)
        out[r0:r0 + rr] = bf16_bits(z)
    return out


def attention_logits(heads: int = 32, seq: int = 2048, seed: int = 9, logit_std: float = 3.0) -> np.ndarray:
    """Attention logits [heads * seq, seq] ~ N(0, logit_std^2) in bf16 (the
    1/sqrt(d) scale is left to the consumer)."""
    rng = np.random.default_rng(seed)
    out = np.empty((heads * seq, seq), dtype=np.uint16)
    step = 4096
    for r0 in range(0, heads * seq, step):
        rr = min(step, heads * seq - r0)
        out[r0:r0 + rr] = bf16_bits(rng.standard_normal((rr, seq), dtype=np.float32) * np.float32(logit_std))
    return out


def sweep_operand(tokens: int, k: int, seed: int = 8, outlier_frac: float = 0.001,
                  outlier_factor: float = 100.0) -> np.ndarray:
    """Throughput-sweep operand [tokens, k]: N(0, 1) with ``outlier_frac`` of the
    elements (uniform positions) multiplied by ``outlier_factor``; bf16."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((tokens, k), dtype=np.float32)
    n_out = int(round(outlier_frac * tokens * k))
    if n_out:
        idx = rng.choice(tokens * k, size=n_out, replace=False)
        x.reshape(-1)[idx] *= np.float32(outlier_factor)
    return bf16_bits(x)


def ties_and_specials(rows: int, k: int, seed: int = 11) -> np.ndarray:
    """bf16 operand built to stress tie-breaking and special values: small
    integer magnitudes (many equal scores), +-0, subnormal bf16, all-zero
    rows and groups, and large magnitudes (up to 6e4, so squares stay well
    inside binary32)."""
    rng = np.random.default_rng(seed)
    x = rng.integers(-3, 4, size=(rows, k)).astype(np.float32)
    bits = bf16_bits(x)
    u = rng.random((rows, k))
    bits[u < 0.05] = 0x8000                                               # -0
    sub = rng.integers(1, 0x80, size=(rows, k), dtype=np.uint16)          # subnormal bf16
    sgn = (rng.random((rows, k)) < 0.5).astype(np.uint16) << np.uint16(15)
    m = (u >= 0.05) & (u < 0.10)
    bits[m] = (sub | sgn)[m]
    big = bf16_bits(rng.uniform(1e3, 6e4, size=(rows, k)).astype(np.float32))
    m = (u >= 0.10) & (u < 0.11)
    bits[m] = big[m] | sgn[m]
    if rows > 2:
        bits[1] = 0                                                       # an all-zero row
    bits[:, 8:12] = 0                                                     # an all-zero group per row
    return bits

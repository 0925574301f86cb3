"""Seeded synthetic inputs for the H-BitLinear forward pass.

This module only draws random numbers and stores them: it holds none of the
method's arithmetic (no norm, no transform, no quantiser). Both the CPU
oracle (through the tests) and the CUDA path (through the tests and the
benchmark) are fed from here, so that the two see the same bytes.

Why the activations look like this: the BitNet v2 walkthrough article
(m.jxzklqfsx.com, section "H-BitLinear模塊" and Figs. 1-3) describes the
inputs of the attention output projection Wo and the FFN down projection
Wdown as sharply peaked at zero with a few outlier channels. The recipe
below imitates that with a Laplace (or normal) body, optional exact zeros,
and a fixed set of outlier columns scaled up by a factor. The values are
rounded once to bf16 (round to nearest even) on the host; the GPU and the
oracle both receive those bf16 bit patterns.

Stream layout (so that a prefix of rows does not depend on the row count):
  generator X = numpy PCG64 seeded with [seed, layer, 0]
    1. outlier columns: choice(K, n_outlier, replace=False)
    2. per token row, in order: K body values, then (if zero_frac > 0)
       K uniforms for the zero mask
  generator W = numpy PCG64 seeded with [seed, layer, 1]
    W[K, N] = 0.02 * standard_normal (float32), drawn in one call
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "LayerSpec",
    "WORKLOADS",
    "activations",
    "weights",
    "layer",
    "qkv_states",
]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the uint16 bit patterns.

    Inputs must be finite (the generators never produce NaN or Inf)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class LayerSpec:
    """One H-BitLinear layer workload: activations [M, K] (bf16) and weights [K, N] (fp32)."""

    name: str
    M: int
    K: int
    N: int
    abits: int
    had_block: int  # 0 = one transform over all of K (K a power of two); 1 = none; else block size
    dist: str  # "normal" or "laplace"
    scale: float  # std (normal) or diversity b (laplace) of the body
    zero_frac: float  # fraction of body values set to exactly 0
    outlier_frac: float  # fraction of the K channels that are outliers
    outlier_factor: float  # multiplier applied to outlier channels
    seed: int
    layer: int = 0
    note: str = field(default="", compare=False)

    @property
    def n_outlier(self) -> int:
        if self.outlier_frac <= 0:
            return 0
        return max(1, int(round(self.outlier_frac * self.K)))

    def with_m(self, M: int) -> "LayerSpec":
        return LayerSpec(
            self.name, M, self.K, self.N, self.abits, self.had_block, self.dist, self.scale,
            self.zero_frac, self.outlier_frac, self.outlier_factor, self.seed, self.layer, self.note,
        )


# The five H-BitLinear workload families (sizes follow the 1.3B / 3B / 7B-like Wo and Wdown
# shapes) and one plain BitLinear. The 7B pair is listed at its largest token count; other token
# counts use with_m().
WORKLOADS: dict[str, LayerSpec] = {
    "single_a8_16x256": LayerSpec(
        "single_a8_16x256", 16, 256, 256, 8, 0, "normal", 1.0, 0.0, 4 / 256, 50.0, 0,
        note="single layer, a8, 4 outlier channels x50"),
    "wo_1p3b_a4": LayerSpec(
        "wo_1p3b_a4", 2048, 2048, 2048, 4, 0, "laplace", 0.05, 0.3, 0.01, 40.0, 1,
        note="1.3B-like Wo, 70% Laplace(0,0.05) + 30% zeros, 1% outliers x40"),
    "wdown_3b_a4": LayerSpec(
        "wdown_3b_a4", 4096, 8192, 2560, 4, 0, "laplace", 0.1, 0.0, 0.005, 60.0, 2,
        note="3B-like Wdown, Laplace(0,0.1), 0.5% outliers x60"),
    "wo_7b_a4": LayerSpec(
        "wo_7b_a4", 8192, 4096, 4096, 4, 0, "laplace", 0.05, 0.0, 0.01, 50.0, 3, 0,
        note="7B-like Wo, Laplace(0,0.05), 1% outliers x50"),
    "wdown_7b_a4": LayerSpec(
        "wdown_7b_a4", 8192, 16384, 4096, 4, 0, "laplace", 0.05, 0.0, 0.01, 50.0, 3, 1,
        note="7B-like Wdown, Laplace(0,0.05), 1% outliers x50"),
    "wdown_nonpow2_a4": LayerSpec(
        "wdown_nonpow2_a4", 8192, 11008, 4096, 4, 256, "laplace", 0.05, 0.0, 0.01, 50.0, 4,
        note="Wdown with K=11008 = 43 x 256, block-diagonal transform"),
    # A plain BitLinear (no rotation, had_block = 1). The walkthrough article (section
    # "H-BitLinear模塊") describes the inputs of the attention and FFN input projections as roughly
    # Gaussian, unlike the outlier-heavy Wo/Wdown inputs: a normal body without outlier channels.
    "qkv_7b_plain_a4": LayerSpec(
        "qkv_7b_plain_a4", 8192, 4096, 12288, 4, 1, "normal", 1.0, 0.0, 0.0, 1.0, 5,
        note="7B-like fused QKV projection 4096 -> 12288, no transform, N(0,1) inputs"),
}

# Token counts of the 7B-like layer pair sweep.
SWEEP_TOKENS_7B = (1, 16, 64, 512, 8192)


def activations(spec: LayerSpec, rows: int | None = None) -> np.ndarray:
    """bf16 bit patterns [rows, K] (uint16) for the spec; rows defaults to spec.M.

    Row i is the same for every row count (the stream is drawn row by row)."""
    M = spec.M if rows is None else rows
    K = spec.K
    rng = np.random.default_rng([spec.seed, spec.layer, 0])
    cols = rng.choice(K, size=spec.n_outlier, replace=False) if spec.n_outlier else np.empty(0, np.int64)
    out = np.empty((M, K), dtype=np.uint16)
    fac = np.ones(K, dtype=np.float32)
    fac[cols] = spec.outlier_factor
    for i in range(M):
        if spec.dist == "normal":
            v = rng.standard_normal(K, dtype=np.float32) * np.float32(spec.scale)
        elif spec.dist == "laplace":
            v = rng.laplace(0.0, spec.scale, size=K).astype(np.float32)
        else:
            raise ValueError(f"unknown distribution {spec.dist!r}")
        if spec.zero_frac > 0:
            v[rng.random(K) < spec.zero_frac] = 0.0
        out[i] = f32_to_bf16_bits(v * fac)
    return out


def weights(spec: LayerSpec) -> np.ndarray:
    """Latent fp32 weights W [K, N] ~ N(0, 0.02^2)."""
    rng = np.random.default_rng([spec.seed, spec.layer, 1])
    return rng.standard_normal((spec.K, spec.N), dtype=np.float32) * np.float32(0.02)


def layer(name: str, M: int | None = None) -> tuple[LayerSpec, np.ndarray, np.ndarray]:
    """(spec, X bf16 bits [M, K], W fp32 [K, N]) for a named workload."""
    spec = WORKLOADS[name]
    if M is not None:
        spec = spec.with_m(M)
    return spec, activations(spec), weights(spec)


def qkv_states(M: int, H: int, D: int, seed: int = 6, row_stride: int | None = None) -> np.ndarray:
    """bf16 bit patterns [M, row_stride] of attention states: M tokens of H heads x D features from
    the row start, N(0, 1) (the pages give no distribution for the QKV states), drawn row by row
    from numpy PCG64 seeded with [seed, H, D]; features past H*D (another projection's slice of a
    fused QKV row) are N(0, 1) as well."""
    stride = H * D if row_stride is None else row_stride
    rng = np.random.default_rng([seed, H, D])
    out = np.empty((M, stride), dtype=np.uint16)
    for i in range(M):
        out[i] = f32_to_bf16_bits(rng.standard_normal(stride, dtype=np.float32))
    return out

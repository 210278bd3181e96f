"""Seeded synthetic layer inputs shared by the tests, the bench and the oracle.

This module draws random numbers and nothing else: it holds none of the
SVDQuant arithmetic (no smoothing, no SVD, no quantisation, no product).
Both the CUDA path and the CPU oracle read the same bytes from here.

The inputs stand in for the diffusion-transformer layers that the SVDQuant
technical review evaluates (FLUX.1 joint-attention QKV, MLP and single-stream
linears; PixArt-Sigma linears; review section 8).  No model weights or prompt
sets are used.  Every array of bf16 values is returned as its uint16 bit
pattern; `bf16_bits_to_f64` turns it into exactly equal float64 values.

Recipe (per layer):
  * X [M, K]: N(0, 1); `n_out_ch` channels (columns) chosen without
    replacement are multiplied by a factor (a fixed factor, or log-uniform in
    [lo, hi]) -- the activation outliers the smoothing step targets.
  * W [N, K] (nn.Linear layout; the math weight is its transpose, K x N):
    N(0, 0.02); `n_out_rows` input channels (columns of this array, rows of
    the math weight) multiplied by a factor.
  * b [N]: N(0, 0.01).
  * optional LoRA A [K, k] and B [k, N]: N(0, 0.01) each.
Draw order: X, outlier channel indices, outlier factors, W, outlier row
indices, b, A, B.  fp64 draws are rounded to fp32 (numpy cast) and then to
bf16 with round-to-nearest-even on the bit pattern.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "LayerSpec", "LayerInputs", "make_layer", "f64_to_bf16_bits",
    "bf16_bits_to_f64", "WORKLOADS", "pixart_points", "layer_spec",
]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Input-format conversion: fp64 -> fp32 (numpy RNE) -> bf16 bits (RNE)."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64 values."""
    u = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    M: int
    K: int
    N: int
    rank: int
    seed: int
    n_out_ch: int            # activation outlier channels
    ch_factor: tuple         # (lo, hi): log-uniform factor; lo == hi: fixed
    n_out_rows: int          # weight outlier input channels
    row_factor: float
    lora_rank: int = 0
    group: int = 64


@dataclasses.dataclass
class LayerInputs:
    spec: LayerSpec
    X: np.ndarray            # uint16 [M, K] bf16 bits
    W: np.ndarray            # uint16 [N, K] bf16 bits (nn.Linear layout)
    b: np.ndarray            # uint16 [N]
    A: np.ndarray | None     # uint16 [K, lora_rank]
    B: np.ndarray | None     # uint16 [lora_rank, N]
    out_channels: np.ndarray
    out_rows: np.ndarray


def _proportional(spec_frac: float, K: int) -> int:
    return int(round(spec_frac * K))


def layer_spec(name: str, M: int, K: int, N: int, rank: int, seed: int,
               lora_rank: int = 0, tiny: bool = False) -> LayerSpec:
    """Outlier model: the tiny one (8 channels x50, 4 rows x20) or the
    proportional one (1 % of channels x log-uniform[20, 100], 0.5 % of
    input-channel rows x10), both as listed for these workloads."""
    if tiny:
        return LayerSpec(name, M, K, N, rank, seed, 8, (50.0, 50.0), 4, 20.0,
                         lora_rank)
    return LayerSpec(name, M, K, N, rank, seed, _proportional(0.01, K),
                     (20.0, 100.0), _proportional(0.005, K), 10.0, lora_rank)


def make_layer(spec: LayerSpec, rows: int | None = None) -> LayerInputs:
    """Draw one layer's inputs.  `rows` (<= M) truncates X after drawing all
    M rows, so a smaller case keeps the full-size statistics' first rows."""
    rng = np.random.default_rng(spec.seed)
    M, K, N = spec.M, spec.K, spec.N
    X = rng.standard_normal((M, K))
    ch = np.sort(rng.choice(K, size=spec.n_out_ch, replace=False))
    lo, hi = spec.ch_factor
    if lo == hi:
        fac = np.full(spec.n_out_ch, lo)
    else:
        fac = np.exp(rng.uniform(math.log(lo), math.log(hi), size=spec.n_out_ch))
    X[:, ch] *= fac[None, :]
    W = rng.normal(0.0, 0.02, size=(N, K))
    rws = np.sort(rng.choice(K, size=spec.n_out_rows, replace=False))
    W[:, rws] *= spec.row_factor
    b = rng.normal(0.0, 0.01, size=N)
    A = B = None
    if spec.lora_rank:
        A = rng.normal(0.0, 0.01, size=(K, spec.lora_rank))
        B = rng.normal(0.0, 0.01, size=(spec.lora_rank, N))
    if rows is not None:
        X = X[:rows]
    return LayerInputs(
        spec=spec, X=f64_to_bf16_bits(X), W=f64_to_bf16_bits(W),
        b=f64_to_bf16_bits(b),
        A=None if A is None else f64_to_bf16_bits(A),
        B=None if B is None else f64_to_bf16_bits(B),
        out_channels=ch, out_rows=rws)


# The five workloads.  Seeds: tiny 0, QKV 1, MLP pair 2, single-stream 3,
# PixArt sweep 4000 + point index.
WORKLOADS = {
    "tiny": layer_spec("tiny", 256, 512, 512, 16, 0, tiny=True),
    "flux_qkv": layer_spec("flux_qkv", 4608, 3072, 9216, 32, 1),
    "flux_mlp_fc1": layer_spec("flux_mlp_fc1", 4608, 3072, 12288, 32, 2),
    # fc2's weights and outlier rows; its activation is GELU(fc1 output) in
    # the chained pair.  As a standalone point its X uses this same spec.
    "flux_mlp_fc2": layer_spec("flux_mlp_fc2", 4608, 12288, 3072, 32, 20),
    "flux_ss_in": layer_spec("flux_ss_in", 4608, 3072, 21504, 32, 3, lora_rank=16),
    "flux_ss_out": layer_spec("flux_ss_out", 4608, 15360, 3072, 32, 30, lora_rank=16),
}


def pixart_points():
    """The PixArt-Sigma-like sweep: (K, N) in {1152->1152, 1152->3456,
    1152->4608, 4608->1152}, M in {256, 1024, 4096, 16384}, r in {16, 32, 64}."""
    shapes = [(1152, 1152), (1152, 3456), (1152, 4608), (4608, 1152)]
    pts = []
    idx = 0
    for (K, N) in shapes:
        for M in (256, 1024, 4096, 16384):
            for r in (16, 32, 64):
                pts.append(layer_spec(f"pixart_K{K}_N{N}_M{M}_r{r}", M, K, N, r,
                                      4000 + idx))
                idx += 1
    return pts

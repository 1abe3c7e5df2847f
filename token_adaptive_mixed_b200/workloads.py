"""Seeded synthetic inputs for the mixed-bit linear layer (shared by tests and bench).

This module only draws random numbers in the shapes, scales and structure of the
Llama-shaped workloads the layer is measured on; it holds none of the layer's
own arithmetic (no quantiser, no routing logits, no GEMM). The MoBiQuant pages
evaluate on LLaMA-2/3 models with WikiText2 and zero-shot suites (explainer
[en] §4 "Experimental Results"); neither weights nor data exist here, so these
draws stand in for them, with the layer shapes of those models.

Recipe (every array is drawn from ``numpy.random.default_rng(seed)`` in fp32,
then rounded to its storage type with round-to-nearest-even):
  * weights W[N,K] ~ N(0, sigma^2); "outlier input columns" = a random subset of
    columns (drawn without replacement) multiplied by 10 before rounding to fp16;
  * activations X[T,K] ~ N(0,1), rounded to bf16; optionally a random subset of
    tokens multiplied by a factor (large-token outliers);
  * router Wr[K,S] ~ N(0, 1/K) in fp32;
  * router bias (when a target mix of slice counts is asked for): chosen from a
    Gaussian model of the logits, l ~ N(0, Wr^T Wr) (times the token factor for
    the scaled tokens), by bisection on a fixed Monte-Carlo sample, so that
    P(argmax = j) matches the target fractions. It depends on Wr only, never on X.
  * two-layer MLP scorer (threshold routing): W1[K,H] ~ N(0, 1/K), b1[H] ~
    N(0, 0.1^2), W2[H,S-1] ~ N(0, 2/H) (He scale after the ReLU), b2[S-1] =
    the given offsets (0 by default), all fp32; with tau = 1 and delta = 0.5
    each residual slice is then active for about half of the tokens.
"""
from __future__ import annotations

import dataclasses
from typing import Sequence

import numpy as np
import torch

S_DEFAULT = 3
G_DEFAULT = 128


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 numpy -> bf16 torch tensor (CPU), round to nearest even."""
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor -> its uint16 bit patterns as numpy."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def draw_weights(rng: np.random.Generator, N: int, K: int, sigma: float, n_outlier_cols: int) -> np.ndarray:
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(sigma)
    if n_outlier_cols > 0:
        cols = rng.choice(K, n_outlier_cols, replace=False)
        W[:, cols] *= np.float32(10.0)
    return W.astype(np.float16)


def draw_activations(rng: np.random.Generator, T: int, K: int, scaled_frac: float = 0.0,
                     scale: float = 1.0, return_rows: bool = False):
    X = rng.standard_normal((T, K), dtype=np.float32)
    rows = np.zeros(0, np.int64)
    if scaled_frac > 0.0 and T > 0:
        m = int(round(scaled_frac * T))
        rows = rng.choice(T, m, replace=False)
        X[rows] *= np.float32(scale)
    return (to_bf16(X), np.sort(rows)) if return_rows else to_bf16(X)


def draw_router(rng: np.random.Generator, K: int, S: int) -> np.ndarray:
    return (rng.standard_normal((K, S), dtype=np.float32) / np.float32(np.sqrt(K))).astype(np.float32)


def bias_for_mix(Wr: np.ndarray, targets: Sequence[float], scaled_frac: float = 0.0, scale: float = 1.0,
                 samples: int = 200_000, seed: int = 12345) -> np.ndarray:
    """Bias b (b[0] = 0) such that a Gaussian model of the logits gives the target mix.

    Model: for x ~ N(0, I_K), the logit vector x.Wr is N(0, C) with C = Wr^T Wr;
    a fraction ``scaled_frac`` of tokens has x scaled by ``scale``. The fractions
    P(argmax_j (l_j + b_j) = j) are estimated on one fixed sample and matched by
    alternating bisection on b[1..S-1].
    """
    S = Wr.shape[1]
    targets = np.asarray(targets, np.float64)
    C = Wr.astype(np.float64).T @ Wr.astype(np.float64)
    L = np.linalg.cholesky(C + 1e-12 * np.eye(S))
    rng = np.random.default_rng(seed)
    Z = rng.standard_normal((samples, S)) @ L.T
    amp = np.where(rng.random(samples) < scaled_frac, scale, 1.0)
    Z *= amp[:, None]
    b = np.zeros(S)

    def frac(bb):
        return np.bincount(np.argmax(Z + bb, axis=1), minlength=S) / samples

    for _ in range(12):
        for j in range(1, S):
            lo, hi = -20.0, 20.0
            for _ in range(40):
                mid = 0.5 * (lo + hi)
                bb = b.copy()
                bb[j] = mid
                if frac(bb)[j] < targets[j]:
                    lo = mid
                else:
                    hi = mid
            b[j] = 0.5 * (lo + hi)
    return b.astype(np.float32)


@dataclasses.dataclass
class Layer:
    """One linear layer's inputs: fp16 weights, bf16 activations, fp32 router."""
    name: str
    W: np.ndarray | torch.Tensor  # fp16 [N, K] (numpy on the host, or a torch tensor)
    X: torch.Tensor        # bf16 [T, K] (CPU)
    Wr: np.ndarray         # fp32 [K, S]
    bias: np.ndarray | None  # fp32 [S] or None
    scaled_tokens: np.ndarray = dataclasses.field(default_factory=lambda: np.zeros(0, np.int64))  # rows of X scaled

    @property
    def N(self) -> int:
        return self.W.shape[0]

    @property
    def K(self) -> int:
        return self.W.shape[1]

    @property
    def T(self) -> int:
        return self.X.shape[0]


def layer(name: str, N: int, K: int, T: int, seed: int, sigma: float = 0.02, outlier_frac_cols: float = 0.0,
          n_outlier_cols: int | None = None, token_scaled_frac: float = 0.0, token_scale: float = 1.0,
          mix: Sequence[float] | None = None, S: int = S_DEFAULT) -> Layer:
    rng = np.random.default_rng(seed)
    m = n_outlier_cols if n_outlier_cols is not None else int(round(outlier_frac_cols * K))
    W = draw_weights(rng, N, K, sigma, m)
    X, scaled = draw_activations(rng, T, K, token_scaled_frac, token_scale, return_rows=True)
    Wr = draw_router(rng, K, S)
    bias = None if mix is None else bias_for_mix(Wr, mix, token_scaled_frac, token_scale)
    return Layer(name, W, X, Wr, bias, scaled)


# ---- the five workloads -----------------------------------------------------

def tiny(T: int = 16) -> Layer:
    """Tiny single layer: N=256, K=512, 4 outlier columns x10, T=16, seed 0."""
    return layer("tiny_256x512", 256, 512, T, seed=0, n_outlier_cols=4)


DECODE_SHAPES = ((4096, 4096), (11008, 4096), (4096, 11008))  # (N, K): q/k/v/o, gate/up, down
DECODE_TOKENS = (1, 4, 16)


def decode(N: int, K: int, T: int, seed: int = 1) -> Layer:
    """Decode GEMV: Llama-7B projection shape, 0.5% outlier columns x10, seed 1."""
    return layer(f"decode_{N}x{K}_T{T}", N, K, T, seed=seed, outlier_frac_cols=0.005)


def prefill() -> Layer:
    """Prefill: T=2048, N=11008, K=4096, 20 outlier columns, bias for a 1/3-1/3-1/3 mix, seed 2."""
    return layer("prefill_11008x4096_T2048", 11008, 4096, 2048, seed=2, n_outlier_cols=20,
                 mix=(1 / 3, 1 / 3, 1 / 3))


def skewed_prefill(T: int = 4096) -> Layer:
    """Large skewed prefill: N=28672, K=8192, sigma 0.015, 1% outlier columns, 2% tokens x8,
    bias for a 70/20/10 mix, seed 4."""
    return layer(f"skewed_prefill_28672x8192_T{T}", 28672, 8192, T, seed=4, sigma=0.015,
                 outlier_frac_cols=0.01, token_scaled_frac=0.02, token_scale=8.0, mix=(0.7, 0.2, 0.1))


LLAMA7B_PROJECTIONS = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                       ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008))
LLAMA7B_LAYERS = 32


def full_model_projection(layer_idx: int, proj_idx: int, T: int = 8, device: str = "cpu") -> Layer:
    """One projection of the 32-layer Llama-2-7B-shaped stack (seed 1000*layer + proj, base seed 3).

    Weights ~ N(0, 0.02^2) without outlier columns, drawn with torch.Generator on
    ``device`` (the 6.5e9-parameter stack is drawn on the GPU); X is batch-8 and
    the router random per projection.
    """
    name, N, K = LLAMA7B_PROJECTIONS[proj_idx]
    seed = 3 * 1_000_000 + 1000 * layer_idx + proj_idx
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    W = (torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02).to(torch.float16)
    rng = np.random.default_rng(seed)
    X = draw_activations(rng, T, K)
    Wr = draw_router(rng, K, S_DEFAULT)
    return Layer(f"L{layer_idx}.{name}", W, X, Wr, None)


# ---- MLP scorer for threshold routing -----------------------------------------

@dataclasses.dataclass
class MlpRouter:
    """Inputs of threshold routing with a two-layer MLP scorer."""
    name: str
    X: torch.Tensor        # bf16 [T, K] (CPU)
    W1: np.ndarray         # fp32 [K, H]
    b1: np.ndarray         # fp32 [H]
    W2: np.ndarray         # fp32 [H, S-1]
    b2: np.ndarray         # fp32 [S-1]

    @property
    def T(self) -> int:
        return self.X.shape[0]

    @property
    def K(self) -> int:
        return self.X.shape[1]

    @property
    def H(self) -> int:
        return self.W1.shape[1]

    @property
    def S(self) -> int:
        return self.W2.shape[1] + 1


def mlp_router(name: str, T: int, K: int, H: int, seed: int, S: int = S_DEFAULT,
               b2: Sequence[float] | None = None, token_scaled_frac: float = 0.0,
               token_scale: float = 1.0) -> MlpRouter:
    rng = np.random.default_rng(seed)
    X = draw_activations(rng, T, K, token_scaled_frac, token_scale)
    W1 = (rng.standard_normal((K, H), dtype=np.float32) / np.float32(np.sqrt(K))).astype(np.float32)
    b1 = (rng.standard_normal(H, dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    W2 = (rng.standard_normal((H, S - 1), dtype=np.float32) * np.float32(np.sqrt(2.0 / H))).astype(np.float32)
    b2a = np.zeros(S - 1, np.float32) if b2 is None else np.asarray(b2, np.float32).reshape(S - 1)
    return MlpRouter(name, X, W1, b1, W2, b2a)


def mlp_route_decode(T: int = 16) -> MlpRouter:
    """Threshold routing at decode: T tokens of a K=4096 hidden state, H=128 scorer, S=3, seed 7."""
    return mlp_router(f"mlp_route_K4096_H128_T{T}", T, 4096, 128, seed=7)


def mlp_route_prefill(T: int = 2048) -> MlpRouter:
    """Threshold routing at prefill: T=2048 tokens, K=4096, H=128, S=3, seed 8."""
    return mlp_router(f"mlp_route_K4096_H128_T{T}", T, 4096, 128, seed=8)

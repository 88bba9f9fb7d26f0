"""Seeded synthetic workloads for the TTQ hot path.

This module only draws random numbers and arranges them into layer-shaped
tensors; it holds none of the method's arithmetic, so both the CUDA path and
the CPU oracle may take their inputs from it.

The pages evaluate perplexity on WikiText-2, PTB and C4 with trained OPT,
Qwen3 and Gemma checkpoints (TTQ review, "Main results"); neither datasets
nor weights are available here, so seeded tensors with the layer SHAPES of
those models stand in for them. Every recipe below is deterministic in its
seed (numpy ``default_rng``), and bf16/fp16 rounding is done by torch
(round-to-nearest-even).

Recipes (one per workload):
  single-768      W 768x768 fp32 ~ N(0, 0.02^2); X 128x768 fp32 ~ N(0, 1),
                  8 seeded outlier channels x20; b=4, g=32.
  opt125m-block   q,k,v,o 768x768, fc1 3072x768, fc2 768x3072 bf16
                  W ~ N(0, 0.02^2); X T=2048 bf16 Student-t(nu=4),
                  1% outlier channels x30; q, k, v share one input; b=3, g=32.
  gemma1b-mlp     attn 1152x1152, up 6912x1152, down 1152x6912 bf16;
                  T=1024, X ~ N(0, 1); b=4, g=64; rank-16 factors from a
                  truncated SVD of W, the residual W - B A is what is stored.
  llama7b-prefill attn 4096x4096, up 11008x4096, down 4096x11008 bf16;
                  X T=4096 ~ N(0,1) with 0.5% outlier channels x50; b=4, g=128.
  decode-sweep    14336x4096 and 4096x14336 bf16, quantized once from a
                  T=512 prompt (llama-style X), then T in {1, 4, 16},
                  b in {2,3,4,5}, g in {16,32,64,128}.
Weights are [N, K] (out x in); the outlier channel count is ceil(frac * K).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

ALPHA, LAMBDA, P = 0.5, 0.1, 2.0


@dataclass(frozen=True)
class Layer:
    name: str
    N: int
    K: int
    input_name: str  # layers with the same input_name share X


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    bits: int
    group: int
    dtype: torch.dtype
    layers: tuple
    x_kind: str  # "gauss" or "student_t"
    outlier_frac: float = 0.0
    outlier_count: int = 0
    outlier_factor: float = 1.0
    rank: int = 0
    w_std: float = 0.02
    alpha: float = ALPHA
    lam: float = LAMBDA
    p: float = P
    extra: dict = field(default_factory=dict)


_OPT = (Layer("q", 768, 768, "attn_in"), Layer("k", 768, 768, "attn_in"),
        Layer("v", 768, 768, "attn_in"), Layer("o", 768, 768, "attn_out"),
        Layer("fc1", 3072, 768, "mlp_in"), Layer("fc2", 768, 3072, "mlp_mid"))
_GEMMA = (Layer("attn", 1152, 1152, "attn_in"),
          Layer("up", 6912, 1152, "mlp_in"),
          Layer("down", 1152, 6912, "mlp_mid"))
_LLAMA = (Layer("attn", 4096, 4096, "attn_in"),
          Layer("up", 11008, 4096, "mlp_in"),
          Layer("down", 4096, 11008, "mlp_mid"))
_DECODE = (Layer("up", 14336, 4096, "mlp_in"),
           Layer("down", 4096, 14336, "mlp_mid"))

WORKLOADS = {
    "single-768": Workload("single-768", 0, 128, 4, 32, torch.float32,
                           (Layer("linear", 768, 768, "in"),), "gauss",
                           outlier_count=8, outlier_factor=20.0),
    "opt125m-block": Workload("opt125m-block", 1, 2048, 3, 32, torch.bfloat16,
                              _OPT, "student_t", outlier_frac=0.01,
                              outlier_factor=30.0),
    "gemma1b-mlp": Workload("gemma1b-mlp", 2, 1024, 4, 64, torch.bfloat16,
                            _GEMMA, "gauss", rank=16),
    "llama7b-prefill": Workload("llama7b-prefill", 3, 4096, 4, 128,
                                torch.bfloat16, _LLAMA, "gauss",
                                outlier_frac=0.005, outlier_factor=50.0),
    "decode-sweep": Workload("decode-sweep", 4, 512, 4, 128, torch.bfloat16,
                             _DECODE, "gauss", outlier_frac=0.005,
                             outlier_factor=50.0,
                             extra={"decode_T": (1, 4, 16),
                                    "bits": (2, 3, 4, 5),
                                    "groups": (16, 32, 64, 128)}),
}


def seed_for(wl: Workload, salt: int = 0) -> int:
    return 1000 + wl.index * 100 + salt


def activations(T: int, K: int, seed: int, kind: str = "gauss",
                outlier_frac: float = 0.0, outlier_count: int = 0,
                outlier_factor: float = 1.0, nu: float = 4.0) -> np.ndarray:
    """[T, K] float32 activations with seeded outlier channels."""
    rng = np.random.default_rng(seed)
    if kind == "student_t":
        X = rng.standard_t(nu, size=(T, K))
    else:
        X = rng.standard_normal((T, K))
    count = outlier_count or int(math.ceil(outlier_frac * K))
    if count:
        cols = rng.choice(K, size=count, replace=False)
        X[:, cols] *= outlier_factor
    return X.astype(np.float32)


def weights(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, K)) * std).astype(np.float32)


def spectral_weights(N: int, K: int, seed: int, strong: int = 32,
                     sigma0: float = 20.0, decay: float = 0.85,
                     std: float = 0.02) -> np.ndarray:
    """[N, K] float32 weights with a planted decaying spectrum: ``strong``
    rank-one components of sizes sigma0 * decay^i along seeded Gaussian
    directions (normalised by sqrt(N) and sqrt(K), so nearly orthonormal),
    plus i.i.d. N(0, std^2) noise. Stands in for trained projections, whose
    spectra have a few large singular values above a flat bulk."""
    rng = np.random.default_rng(seed)
    G = rng.standard_normal((N, strong)) / math.sqrt(N)
    H = rng.standard_normal((strong, K)) / math.sqrt(K)
    sig = sigma0 * decay ** np.arange(strong)
    W = (G * sig[None, :]) @ H + rng.standard_normal((N, K)) * std
    return W.astype(np.float32)


def probe_vectors(r: int, K: int, seed: int) -> np.ndarray:
    """[r, K] float32 standard Gaussian vectors: the random draws of a
    randomized factorisation, generated once and handed to both the kernels
    and the oracle as an input."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((r, K)).astype(np.float32)


def lowrank_checkpoint(W: np.ndarray, r: int, dtype=torch.bfloat16):
    """Stores a layer as residual + rank-r factors, the way a checkpoint in
    the W = W_q + B A form would ship it (TTQ review, Proposed method,
    bullet 5): B = U_r diag(sigma_r), A = V_r^T from a truncated SVD of W,
    both rounded to ``dtype``; the residual R = W - B A is formed in fp32
    from the rounded factors and rounded to ``dtype``.
    Returns torch CPU tensors (R [N,K], A [r,K], B [N,r]).
    """
    U, S, Vt = np.linalg.svd(W.astype(np.float64), full_matrices=False)
    B = torch.from_numpy((U[:, :r] * S[None, :r]).astype(np.float32)).to(dtype)
    A = torch.from_numpy(Vt[:r, :].astype(np.float32)).to(dtype)
    R = torch.from_numpy(W) - B.float() @ A.float()
    return R.to(dtype), A, B


def to_dtype(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype)


def make_inputs(wl: Workload, T: int | None = None, layers=None):
    """Builds a workload's tensors on the CPU.

    Returns dict with "X": {input_name: tensor [T, K]} and
    "W": {layer_name: tensor [N, K]} (the residual when rank > 0), plus
    "A"/"B" per layer when rank > 0. Tensors are in ``wl.dtype``.
    """
    T = T or wl.T
    use = [l for l in wl.layers if layers is None or l.name in layers]
    out = {"X": {}, "W": {}, "A": {}, "B": {}}
    for li, layer in enumerate(wl.layers):
        if layer not in use:
            continue
        if layer.input_name not in out["X"]:
            salt = 10 + sorted({l.input_name for l in wl.layers}).index(
                layer.input_name)
            X = activations(T, layer.K, seed_for(wl, salt), wl.x_kind,
                            wl.outlier_frac, wl.outlier_count,
                            wl.outlier_factor)
            out["X"][layer.input_name] = to_dtype(X, wl.dtype)
        W = weights(layer.N, layer.K, seed_for(wl, 50 + li), wl.w_std)
        if wl.rank:
            R, A, B = lowrank_checkpoint(W, wl.rank, wl.dtype)
            out["W"][layer.name], out["A"][layer.name] = R, A
            out["B"][layer.name] = B
        else:
            out["W"][layer.name] = to_dtype(W, wl.dtype)
    return out

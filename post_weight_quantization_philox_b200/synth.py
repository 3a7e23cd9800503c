"""Seeded synthetic inputs for the GSQ layer-reconstruction step.

This module only draws data; it holds none of the method's arithmetic.  Both
the CUDA path and the oracle receive the arrays it returns, so it is the one
piece the two sides share.

The GSQ pages calibrate on FineWeb-Edu / OpenThoughts / OpenPlatypus and
quantize trained Llama-3.1 weights; none of these is available, so seeded
tensors with the same projection shapes and value distributions stand in:

* weights  ~ N(0, 0.02^2) (Student-t(nu=5) x 0.02 for the down_proj shape),
* calibration activations ~ N(0, 1) with a few outlier channels (the first m
  entries of a seeded permutation of K, multiplied by a fixed factor),
* weight seed 1000 + config number, activation seed 2000 + config number,
  numpy ``default_rng``; bf16 configs are rounded to bf16 (nearest-even) and
  handed over as exact fp32 values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

GRID_2BIT, GRID_TERNARY, GRID_3BIT_LOCAL = 0, 1, 2


@dataclass(frozen=True)
class LayerConfig:
    """One single-layer reconstruction workload."""
    number: int
    name: str
    N: int              # out features (rows of W)
    K: int              # in features
    T: int              # calibration tokens
    grid: int
    steps: int
    w_dist: str = "normal"       # "normal" | "student_t5"
    w_bf16: bool = True
    x_bf16: bool = True
    outlier_cols: int = 0
    outlier_scale: float = 1.0
    lr: float = 1e-3
    tau0: float = 1.0
    tau1: float = 0.05
    group: int = 128

    @property
    def coords(self) -> int:
        return self.N * self.K


CONFIGS = {
    # Single linear layer, fp32 inputs, 4 outlier channels x10, 20 steps.
    "c1_small_256x512": LayerConfig(1, "c1_small_256x512", 256, 512, 256,
                                    GRID_2BIT, 20, w_bf16=False, x_bf16=False,
                                    outlier_cols=4, outlier_scale=10.0),
    # Llama-3.1-8B q_proj shape, 1% outlier channels x20, 2-bit, 500 steps.
    "c2_qproj_4096x4096": LayerConfig(2, "c2_qproj_4096x4096", 4096, 4096,
                                      4096, GRID_2BIT, 500, outlier_cols=41,
                                      outlier_scale=20.0),
    # Llama-3.1-8B down_proj shape, Student-t weights, 3-bit local, 300 steps.
    "c3_downproj_4096x14336": LayerConfig(3, "c3_downproj_4096x14336", 4096,
                                          14336, 4096, GRID_3BIT_LOCAL, 300,
                                          w_dist="student_t5"),
    # Llama-3.1-8B gate_proj shape, ternary mask x sign, 500 steps.
    "c4_gateproj_14336x4096": LayerConfig(4, "c4_gateproj_14336x4096", 14336,
                                          4096, 4096, GRID_TERNARY, 500),
    # Llama-3.1-70B q_proj shape on 8 x 2048 calibration tokens (Q stage).
    "c5_70b_qproj_8192x8192": LayerConfig(5, "c5_70b_qproj_8192x8192", 8192,
                                          8192, 16384, GRID_2BIT, 200),
    # Llama-3.1-70B k_proj shape on 8 x 2048 tokens (K stage).
    "c5_70b_kproj_1024x8192": LayerConfig(5, "c5_70b_kproj_1024x8192", 1024,
                                          8192, 16384, GRID_2BIT, 200),
}


def bf16_values(a: np.ndarray) -> np.ndarray:
    """Nearest-even bf16 values of a, returned as float32 (input preparation)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def make_weight(cfg: LayerConfig, seed: int | None = None,
                rows: slice | None = None) -> np.ndarray:
    """Weight W (N x K) as float32 (bf16 values when cfg.w_bf16)."""
    rng = np.random.default_rng(1000 + cfg.number if seed is None else seed)
    if cfg.w_dist == "student_t5":
        W = (rng.standard_t(5.0, size=(cfg.N, cfg.K)) * 0.02).astype(np.float32)
    else:
        W = rng.normal(0.0, 0.02, size=(cfg.N, cfg.K)).astype(np.float32)
    if rows is not None:
        W = W[rows]
    return bf16_values(W) if cfg.w_bf16 else np.ascontiguousarray(W)


def make_calib(cfg: LayerConfig, seed: int | None = None) -> np.ndarray:
    """Calibration activations X (T x K) as float32 (bf16 values when cfg.x_bf16)."""
    rng = np.random.default_rng(2000 + cfg.number if seed is None else seed)
    X = rng.normal(0.0, 1.0, size=(cfg.T, cfg.K)).astype(np.float32)
    if cfg.outlier_cols:
        cols = rng.permutation(cfg.K)[: cfg.outlier_cols]
        X[:, cols] *= cfg.outlier_scale
    return bf16_values(X) if cfg.x_bf16 else X


def small_config(N: int, K: int, T: int, grid: int, steps: int = 5,
                 number: int = 90, **kw) -> LayerConfig:
    """A small workload for parity tests (same distributions, other shapes)."""
    return LayerConfig(number, f"small_{N}x{K}x{T}_g{grid}", N, K, T, grid,
                       steps, **kw)


def tau_schedule(tau0: float, tau1: float, steps: int) -> np.ndarray:
    """Geometric annealing tau0 -> tau1 over `steps` steps (float32)."""
    if steps <= 1:
        return np.array([tau0], np.float32)
    i = np.arange(steps, dtype=np.float64)
    return (tau0 * (tau1 / tau0) ** (i / (steps - 1))).astype(np.float32)


def random_logits(shape, seed: int, ties: bool = True) -> np.ndarray:
    """Random logits for harden/pack tests; with ties, some entries repeat."""
    rng = np.random.default_rng(seed)
    l = rng.normal(0.0, 2.0, size=shape).astype(np.float32)
    if ties:
        # quantise a share of entries to a coarse lattice so exact ties occur
        m = rng.random(size=shape) < 0.3
        l[m] = np.round(l[m])
    return l


def random_grad(shape, seed: int, scale: float = 1e-2) -> np.ndarray:
    """A seeded stand-in weight gradient for testing the backward in isolation."""
    rng = np.random.default_rng(seed)
    return (rng.normal(0.0, scale, size=shape)).astype(np.float32)


# ------------------------------------------- block stage: SwiGLU MLP inputs

# Llama-3.1-70B block MLP on 8 sequences x 2048 tokens
MLP_STAGE = {"c5_70b_mlp": dict(T=16384, H=8192, F=28672, grid=GRID_2BIT, steps=200)}


def make_mlp_stage(T: int, H: int, F: int, seed: int = 5005):
    """Normalised MLP input Xn (T x H, unit RMS rows, bf16 values) and
    N(0, 0.02^2) bf16 gate / up (F x H) and down (H x F) projections."""
    rng = np.random.default_rng(seed)
    X = rng.normal(0.0, 1.0, size=(T, H)).astype(np.float32)
    X /= np.sqrt(np.mean(X.astype(np.float64) ** 2, axis=1, keepdims=True)).astype(np.float32)
    Wg = rng.normal(0.0, 0.02, size=(F, H)).astype(np.float32)
    Wu = rng.normal(0.0, 0.02, size=(F, H)).astype(np.float32)
    Wd = rng.normal(0.0, 0.02, size=(H, F)).astype(np.float32)
    return bf16_values(X), bf16_values(Wg), bf16_values(Wu), bf16_values(Wd)


def random_target(T: int, H: int, scale: float, seed: int = 5006) -> np.ndarray:
    """A seeded N(0, scale^2) stand-in for a block-output target."""
    rng = np.random.default_rng(seed)
    return rng.normal(0.0, scale, size=(T, H)).astype(np.float32)


# ----------------------------------------- block stage: attention V/O inputs

# Llama-3.1-70B attention: 64 query heads, 8 key/value heads of 128, 8 x 2048
ATTN_STAGE = {"c5_70b_attn": dict(nseq=8, S=2048, nh=64, nkv=8, d=128, grid=GRID_2BIT,
                                  steps=200)}


def make_attn_stage(nseq: int, S: int, nh: int, nkv: int, d: int = 128, seed: int = 6006):
    """Normalised attention input Xa (nseq S x nh d, unit RMS rows) and
    N(0, 0.02^2) query (H x H), key and value (nkv d x H) and output (H x H)
    projections, all bf16 values."""
    rng = np.random.default_rng(seed)
    H, Hk = nh * d, nkv * d
    X = rng.normal(0.0, 1.0, size=(nseq * S, H)).astype(np.float32)
    X /= np.sqrt(np.mean(X.astype(np.float64) ** 2, axis=1, keepdims=True)).astype(np.float32)
    Ws = [rng.normal(0.0, 0.02, size=shape).astype(np.float32)
          for shape in ((H, H), (Hk, H), (Hk, H), (H, H))]
    return (bf16_values(X), *[bf16_values(W) for W in Ws])

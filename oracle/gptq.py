"""GPTQ as the initial assignment of the GSQ grids -- test infrastructure.

The GSQ pages start the logits from a GPTQ solution (agihunt.info summary,
optimisation paragraph).  GPTQ itself is the published algorithm of
Frantar, Ashkboos, Hoefler and Alistarh, "GPTQ: Accurate Post-Training
Quantization for Generative Pre-trained Transformers" (ICLR 2023): columns are
quantized one at a time in input order and the rounding error of each column
is pushed onto the columns not yet quantized through the inverse Hessian of
the layer objective (optimal brain surgeon updates), using the upper Cholesky
factor U of H^-1.  Restated here in plain numpy, fp64, one column at a time
(no lazy batching), for the GSQ grids and group-128 symmetric scales:

  H = bf16(X)^T bf16(X)                     (the GEMM operand the library keeps)
  dead inputs (H_ii = 0): H_ii = 1, W[:, i] = 0
  H += damp * mean(diag(H)) * I             (damp = 0.01 by default)
  U = upper Cholesky factor of H^-1         (H^-1 = U^T U)
  for each column j:
      at the first column of a group: s = absmax(current group) / c_max (fp32)
      level = nearest grid level to w_j / s (first level on ties; s = 0 -> 0)
      err_j = (w_j - s c_level) / U_jj
      w_(j+1..) -= err_j U_(j, j+1..)

Only tests/, the entry's smoke check and the bench's CPU legs use this module.
"""
from __future__ import annotations

import numpy as np

LEVELS = {0: np.array([-1.5, -0.5, 0.5, 1.5]), 1: np.array([-1.0, 0.0, 1.0]),
          2: np.arange(8) - 3.5}


def _bf16(x):
    """Nearest-even bf16 values of fp32 x, as float64."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (r.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def hessian(X) -> np.ndarray:
    Xb = _bf16(X)
    return Xb.T @ Xb


def prepare(W, X, damp: float = 0.01):
    """Damped Hessian and the weight with dead inputs zeroed (fp64)."""
    W = np.array(W, dtype=np.float64)
    H = hessian(X)
    dead = np.diag(H) == 0
    H[dead, dead] = 1.0
    W[:, dead] = 0.0
    H[np.diag_indices_from(H)] += damp * np.mean(np.diag(H))
    return W, H


def gptq(mode: int, W, X, group: int = 128, damp: float = 0.01, cols: int | None = None):
    """Returns (levels int8 N x K, scales fp32 N x K/group, err N x K, W after
    the updates, damped H).  With cols, stops after that many columns."""
    W, H = prepare(W, X, damp)
    N, K = W.shape
    U = np.linalg.cholesky(np.linalg.inv(H)).T
    c = LEVELS[mode]
    cmax = np.float32(c.max())
    levels = np.zeros((N, K), np.int8)
    scales = np.zeros((N, K // group), np.float32)
    err = np.zeros((N, K))
    for j in range(K if cols is None else cols):
        if j % group == 0:
            absmax = np.abs(W[:, j:j + group]).max(axis=1).astype(np.float32)
            scales[:, j // group] = absmax / cmax
        s = scales[:, j // group].astype(np.float64)
        r = np.divide(W[:, j], s, out=np.zeros(N), where=s > 0)
        lev = np.argmin(np.abs(r[:, None] - c[None, :]), axis=1)
        q = s * c[lev]
        e = (W[:, j] - q) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        W[:, j] = q
        levels[:, j] = lev
        err[:, j] = e
    return levels, scales, err, W, H


def quantized(mode: int, levels, scales, group: int = 128) -> np.ndarray:
    return np.repeat(scales.astype(np.float64), group, axis=1) * LEVELS[mode][levels]

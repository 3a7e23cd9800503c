"""The oracle of the staged block pipeline: a plain fp64 restatement of how GSQ
quantizes a stack of transformer blocks one after another.

Test infrastructure only (imported by ``tests/`` alone).  It shares no code
with the CUDA library.

Source: the agihunt.info summary of GSQ, optimisation paragraph -- blocks are
quantized in order, each block sees the output of the already quantized
prefix, and inside a block the query and key projections are quantized first
(each on its own output), then the value and output projections together,
then the MLP on the block output.  The pages give only that order; the
readings taken where they are silent:

* the block is a Llama-style pre-norm block: h = x + Attn(RMSNorm(x)),
  y = h + MLP(RMSNorm(h)), RMSNorm with unit gain and eps = 1e-5, rotary
  embedding (rotate-half) with theta = 500000, causal attention with grouped
  key/value heads, SwiGLU MLP;
* the residual stream stays in full precision; the GEMM operands are rounded
  to bf16 where the library keeps them in bf16 (``round_bf16``);
* stage Q / K: the layer objective on the normalised block input xa with the
  full-precision weight's own output as target;
* stage V/O: attention probabilities from the frozen quantized Q, K; target
  the full-precision attention output on the same xa;
* stage MLP: input RMSNorm(h_q) with h_q the residual after the quantized
  attention; target y_fp - h_q, so the MLP is trained on the block output
  (its loss is the block-output error ||x_out - y_fp||^2);
* the next block's input is x_out = h_q + MLP_q(RMSNorm(h_q));
* Philox keys: stage j (0 Q, 1 K, 2 V/O, 3 MLP) uses seed ^ (j << 56), and
  weight i inside a joint stage additionally ^ (i << 48).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import (GRID_2BIT, GRID_TERNARY, attn_init, attn_probs, attn_recon_error, attn_step,
               bf16_round, harden, init, mlp_init, mlp_recon_error, mlp_step, recon_error,
               reference_output, step)

RMS_EPS = 1e-5
ROPE_THETA = 500000.0
MASK64 = (1 << 64) - 1


@dataclass(frozen=True)
class BlockDims:
    nseq: int
    S: int
    nh: int
    nkv: int
    d: int
    F: int

    @property
    def T(self) -> int:
        return self.nseq * self.S

    @property
    def H(self) -> int:
        return self.nh * self.d

    @property
    def Hk(self) -> int:
        return self.nkv * self.d


WEIGHTS = ("q", "k", "v", "o", "gate", "up", "down")


def weight_shapes(dm: BlockDims):
    H, Hk, F = dm.H, dm.Hk, dm.F
    return {"q": (H, H), "k": (Hk, H), "v": (Hk, H), "o": (H, H),
            "gate": (F, H), "up": (F, H), "down": (H, F)}


def stage_seed(seed: int, stage: int) -> int:
    return (seed ^ (stage << 56)) & MASK64


def rmsnorm(x, eps: float = RMS_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) per row, unit gain, fp64."""
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)


def _r(a, on: bool):
    return bf16_round(a) if on else np.asarray(a, np.float64)


def attention_out(xa, Wq, Wk, Wv, Wo, dm: BlockDims, theta=ROPE_THETA, round_bf16=True):
    """Attention sublayer output (T x H): P from Wq, Wk (rotary, causal,
    grouped heads), V = xa Wv^T, o_(s,h) = P_(s,h) V_(s, h // grp), o Wo^T."""
    P = attn_probs(xa, Wq, Wk, dm.nseq, dm.S, dm.nh, dm.nkv, dm.d, theta, round_bf16)
    xa64 = np.asarray(xa, np.float64)
    V = _r(xa64 @ np.asarray(Wv, np.float64).T, round_bf16)
    grp = dm.nh // dm.nkv
    o = np.zeros((dm.T, dm.H))
    for s in range(dm.nseq):
        rows = slice(s * dm.S, (s + 1) * dm.S)
        for h in range(dm.nh):
            g = h // grp
            o[rows, h * dm.d:(h + 1) * dm.d] = (P[s, h].astype(np.float64)
                                                @ V[rows, g * dm.d:(g + 1) * dm.d])
    o = _r(o, round_bf16)
    return o @ np.asarray(Wo, np.float64).T


def mlp_out(xm, Wg, Wu, Wd, round_bf16=True):
    """SwiGLU MLP output (T x H): (silu(xm Wg^T) * xm Wu^T) Wd^T."""
    xm = np.asarray(xm, np.float64)
    a = xm @ np.asarray(Wg, np.float64).T
    b = xm @ np.asarray(Wu, np.float64).T
    hh = _r(a / (1.0 + np.exp(-a)) * b, round_bf16)
    return hh @ np.asarray(Wd, np.float64).T


def block_forward(x, W: dict, dm: BlockDims, theta=ROPE_THETA, eps=RMS_EPS,
                  round_bf16=True) -> dict:
    """One pre-norm block on the residual stream x (T x H):
    xa = RMSNorm(x), attn = Attn(xa), h = x + attn, xm = RMSNorm(h),
    y = h + MLP(xm).  Returns every named intermediate (fp64; xa and xm as
    the bf16 GEMM operands when round_bf16)."""
    x = np.asarray(x, np.float64)
    xa = _r(rmsnorm(x, eps), round_bf16)
    attn = attention_out(xa, W["q"], W["k"], W["v"], W["o"], dm, theta, round_bf16)
    h = x + attn
    xm = _r(rmsnorm(h, eps), round_bf16)
    mlp = mlp_out(xm, W["gate"], W["up"], W["down"], round_bf16)
    return {"xa": xa, "attn": attn, "h": h, "xm": xm, "mlp": mlp, "y": h + mlp}


def block_forward_rows(x, W: dict, dm: BlockDims, s: int, positions, theta=ROPE_THETA,
                       eps=RMS_EPS, round_bf16=True) -> np.ndarray:
    """y of the block at `positions` of sequence s, computed from rows
    0..max(positions) of that sequence only (causal attention needs nothing
    later): for checking samples of layers too large for block_forward."""
    from . import attn_prob_row
    positions = list(positions)
    last = max(positions) + 1
    rows = np.asarray(x[s * dm.S:s * dm.S + last], np.float64)
    xa = _r(rmsnorm(rows, eps), round_bf16)
    V = _r(xa @ np.asarray(W["v"], np.float64).T, round_bf16)
    grp = dm.nh // dm.nkv
    xa32 = np.ascontiguousarray(xa, np.float32)
    o = np.zeros((len(positions), dm.H))
    for i, p in enumerate(positions):
        for h in range(dm.nh):
            g = h // grp
            # the probability row of query p only needs keys 0..p of this sequence
            prow = attn_prob_row(xa32, W["q"], W["k"], 1, last, dm.nh, dm.nkv, 0, h, p, dm.d,
                                 theta, round_bf16)
            o[i, h * dm.d:(h + 1) * dm.d] = (prow[:p + 1].astype(np.float64)
                                             @ V[:p + 1, g * dm.d:(g + 1) * dm.d])
    o = _r(o, round_bf16)
    hrows = rows[positions] + o @ np.asarray(W["o"], np.float64).T
    xm = _r(rmsnorm(hrows, eps), round_bf16)
    return hrows + mlp_out(xm, W["gate"], W["up"], W["down"], round_bf16)


LEVEL_VALUES = {GRID_2BIT: np.array([-1.5, -0.5, 0.5, 1.5]),
                GRID_TERNARY: np.array([-1.0, 0.0, 1.0]),
                2: np.arange(8) - 3.5}


def hard_weight(st) -> np.ndarray:
    """bf16(s_g c_level) of the hard choice of a layer state (fp32 values)."""
    lev = harden(st.mode, st.logits, st.i0)
    w = np.repeat(st.s.astype(np.float64), st.group, axis=1) * LEVEL_VALUES[st.mode][lev]
    return bf16_round(w).astype(np.float32)


def quantize_block(x, W: dict, dm: BlockDims, mode: int, taus, lr: float, seed: int,
                   beta1=0.9, beta2=0.99, theta=ROPE_THETA, eps=RMS_EPS) -> dict:
    """GSQ's staged reconstruction of one block from its input x (the output
    of the quantized prefix).  taus: four temperature schedules (Q, K, V/O,
    MLP).  Returns the block output x_out, the hard weights, and per stage the
    step losses and the final hard reconstruction error (abs, rel)."""
    f32 = lambda a: np.ascontiguousarray(a, np.float32)  # noqa: E731
    fp = block_forward(x, W, dm, theta, eps, True)
    xa = f32(fp["xa"])
    hard, stats = {}, {}
    # Q and K, each on its own output
    for j, name in enumerate(("q", "k")):
        st = init(mode, W[name], seed=stage_seed(seed, j))
        Y = reference_output(W[name], xa)
        losses = [step(st, xa, Y, float(t), lr, beta1, beta2) for t in taus[j]]
        stats[name] = dict(losses=losses, recon=recon_error(st, xa, Y))
        hard[name] = hard_weight(st)
    # V and O jointly, probabilities from the frozen quantized Q, K
    P = attn_probs(xa, hard["q"], hard["k"], dm.nseq, dm.S, dm.nh, dm.nkv, dm.d, theta, True)
    R = fp["attn"]
    at = attn_init(mode, W["v"], W["o"], seed=stage_seed(seed, 2))
    dims = (dm.nseq, dm.S, dm.nh, dm.nkv, dm.d)
    losses = [attn_step(at, xa, P, R, dims, float(t), lr, beta1, beta2) for t in taus[2]]
    hard["v"], hard["o"] = hard_weight(at.v), hard_weight(at.o)
    attn_q = attention_out(xa, hard["q"], hard["k"], hard["v"], hard["o"], dm, theta, True)
    stats["vo"] = dict(losses=losses, recon=attn_recon_error(at, xa, P, R, dims))
    h = np.asarray(x, np.float64) + attn_q
    # the MLP on the block output
    xm = f32(bf16_round(rmsnorm(h, eps)))
    Rm = fp["y"] - h
    ms = mlp_init(mode, W["gate"], W["up"], W["down"], seed=stage_seed(seed, 3))
    losses = [mlp_step(ms, xm, Rm, float(t), lr, beta1, beta2) for t in taus[3]]
    hard["gate"], hard["up"], hard["down"] = (hard_weight(ms.gate), hard_weight(ms.up),
                                              hard_weight(ms.down))
    mlp_q = mlp_out(xm, hard["gate"], hard["up"], hard["down"], True)
    x_out = h + mlp_q
    stats["mlp"] = dict(losses=losses, recon=mlp_recon_error(ms, xm, Rm))
    return {"x_out": x_out, "hard": hard, "stats": stats, "y_fp": fp["y"], "xa": fp["xa"],
            "attn_fp": fp["attn"], "h": h, "xm": xm}


def quantize_stack(x0, blocks, dm: BlockDims, mode: int, taus, lr: float, seeds,
                   beta1=0.9, beta2=0.99) -> list:
    """Blocks in order; block b sees the output of the quantized blocks < b."""
    out, x = [], np.asarray(x0, np.float64)
    for W, seed in zip(blocks, seeds):
        r = quantize_block(x, W, dm, mode, taus, lr, seed, beta1, beta2)
        r["x_in"] = x
        out.append(r)
        x = r["x_out"]
    return out

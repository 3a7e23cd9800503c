"""The oracle of GSQ on GGUF K-Quant formats: a plain numpy restatement.

Test infrastructure only (imported by ``tests/`` alone); it shares no code
with the CUDA library.

Source: the agihunt.info summary of GSQ, optimisation paragraph (in the
GGUF setting GSQ starts from an existing K-Quant and, after optimising,
projects the result back into the same format) and its results paragraph
(Qwen3-8B Q2_K and Q3_K_M, format unchanged); the thelatestinai.com /
fugumt.com abstract (starting from released GGUF checkpoints, projecting back
into the same deployment format).

Formats (256-weight super-blocks of 16 sub-blocks of 16 consecutive weights
of a row):
  Q2_K  w = d sc_j q - dmin m_j,  q in 0..3, sc_j, m_j in 0..15 (4 bits),
        d, dmin fp16; 84 bytes per block;
  Q3_K  w = d sc_j q,  q in -4..3, sc_j in -32..31 (6 bits, stored + 32),
        d fp16; 110 bytes per block.
Byte layout of a block (checked in the tests against the ``gguf`` package's
dequantizer):
  Q2_K  bytes 0..15: sc_j | m_j << 4; 16..79: 2-bit codes; 80..81 d; 82..83 dmin
  Q3_K  bytes 0..31: high code bits; 32..95: low 2 code bits; 96..107: 6-bit
        scales; 108..109 d
  2-bit fields: weight i = 128 h + 32 s + r sits in code byte 32 h + r at
  bits 2 s; Q3_K high bit of weight i in byte i % 32, bit i // 32; Q3_K
  scale u_j = sc_j + 32: low 4 bits in byte j % 8 at bit 4 (j // 8), high 2
  bits in byte 8 + j % 4 at bit 2 (j // 4).

GSQ on a K-Quant (readings, the pages give none of the details):
  * the start is the given blocks (a released checkpoint), or this module's
    min-max K-Quant of W: per sub-block a = (max - min') / 3, b = -min' with
    min' = min(0, min w) (Q2_K), a = -w_e / 4 with w_e the largest-magnitude
    weight (Q3_K); super-block d = fp16(max a / 15), dmin = fp16(max b / 15)
    (Q2_K), d = fp16(max |a| / 31) (Q3_K); codes sc = rint(a / d) clamped,
    weight codes the nearest level (first on ties), all in fp32;
  * per coordinate logits: 4 over q (Q2_K, full grid), 5 local shifts -2..+2
    around the start code clamped to [-4, 3] (Q3_K), +2 on the start code;
  * per sub-block continuous parameters trained with the logits: a_j, b_j
    (Q2_K) or a_j (Q3_K), starting at d sc_j and dmin m_j; soft weight
    w = a_j sum_k y_k c_k - b_j;
  * the layer loss, noise, Lion and temperature as in the GSQ grids (noise
    words: Q2_K as the 2-bit grid, Q3_K as the 3-bit local grid);
  * projection back: the hard codes (argmax) and the trained a_j, b_j
    re-encoded exactly as at the start (b_j and, for Q2_K, a_j clamped at 0).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import GRID_2BIT, GRID_3BIT_LOCAL, bf16_round, lion, uniforms

Q2_K, Q3_K = 0, 1
BLOCK_BYTES = {Q2_K: 84, Q3_K: 110}
NUM_LOGITS = {Q2_K: 4, Q3_K: 5}
QMIN = {Q2_K: 0, Q3_K: -4}
QMAX = {Q2_K: 3, Q3_K: 3}
F32 = np.float32


def _f16(x):
    return np.asarray(x, F32).astype(np.float16)


# ------------------------------------------------------------ block layout

def _put_codes2(blk, off, u):
    """2-bit fields u[0..255] into bytes off..off+63 of each block."""
    i = np.arange(256)
    h, s, r = i // 128, (i % 128) // 32, i % 32
    for k in range(256):
        blk[:, off + 32 * h[k] + r[k]] |= ((u[:, k] & 3) << (2 * s[k])).astype(np.uint8)


def _get_codes2(blk, off):
    i = np.arange(256)
    h, s, r = i // 128, (i % 128) // 32, i % 32
    return (blk[:, off + 32 * h + r] >> (2 * s)) & 3


def encode(fmt: int, q, sc, m, d, dmin=None) -> np.ndarray:
    """Blocks (nblk x bytes) from codes q (nblk x 256), sub-block codes sc, m
    (nblk x 16) and fp16 super-block factors d, dmin (nblk)."""
    q = np.asarray(q, np.int64)
    nblk = q.shape[0]
    blk = np.zeros((nblk, BLOCK_BYTES[fmt]), np.uint8)
    if fmt == Q2_K:
        blk[:, 0:16] = (np.asarray(sc, np.int64) | (np.asarray(m, np.int64) << 4)).astype(np.uint8)
        _put_codes2(blk, 16, q)
        blk[:, 80:82] = _f16(d).view(np.uint8).reshape(nblk, 2)
        blk[:, 82:84] = _f16(dmin).view(np.uint8).reshape(nblk, 2)
    else:
        u = q + 4                       # 0..7
        for i in range(256):
            blk[:, i % 32] |= ((u[:, i] >> 2) << (i // 32)).astype(np.uint8)
        _put_codes2(blk, 32, u & 3)
        us = np.asarray(sc, np.int64) + 32  # 0..63
        for j in range(16):
            blk[:, 96 + j % 8] |= ((us[:, j] & 15) << (4 * (j // 8))).astype(np.uint8)
            blk[:, 104 + j % 4] |= ((us[:, j] >> 4) << (2 * (j // 4))).astype(np.uint8)
        blk[:, 108:110] = _f16(d).view(np.uint8).reshape(nblk, 2)
    return blk


def decode(fmt: int, blk):
    """(q, sc, m, d, dmin) of blocks: codes, sub-block codes, fp16 factors
    as float32 (m and dmin zero for Q3_K)."""
    blk = np.asarray(blk, np.uint8)
    nblk = blk.shape[0]
    if fmt == Q2_K:
        q = _get_codes2(blk, 16).astype(np.int64)
        sc = (blk[:, 0:16] & 15).astype(np.int64)
        m = (blk[:, 0:16] >> 4).astype(np.int64)
        d = blk[:, 80:82].copy().view(np.float16).reshape(nblk).astype(F32)
        dmin = blk[:, 82:84].copy().view(np.float16).reshape(nblk).astype(F32)
        return q, sc, m, d, dmin
    low = _get_codes2(blk, 32).astype(np.int64)
    i = np.arange(256)
    hi = (blk[:, i % 32] >> (i // 32)) & 1
    q = low + 4 * hi.astype(np.int64) - 4
    j = np.arange(16)
    us = ((blk[:, 96 + j % 8] >> (4 * (j // 8))) & 15).astype(np.int64) | \
         ((((blk[:, 104 + j % 4] >> (2 * (j // 4))) & 3).astype(np.int64)) << 4)
    d = blk[:, 108:110].copy().view(np.float16).reshape(nblk).astype(F32)
    return q, us - 32, np.zeros_like(us), d, np.zeros(nblk, F32)


def dequant(fmt: int, blk, N: int, K: int) -> np.ndarray:
    """Weights (N x K, float32) of N * K / 256 blocks in row-major block order:
    fp32 products d sc (and dmin m), then times q, minus, as the format says."""
    q, sc, m, d, dmin = decode(fmt, blk)
    a = (d[:, None] * sc.astype(F32)).astype(F32)          # nblk x 16
    b = (dmin[:, None] * m.astype(F32)).astype(F32)
    w = np.repeat(a, 16, axis=1) * q.astype(F32) - np.repeat(b, 16, axis=1)
    return w.astype(F32).reshape(N, K)


# ------------------------------------------------------------- the start

def _levels(fmt):
    return np.arange(QMIN[fmt], QMAX[fmt] + 1)


def project(fmt: int, a, b=None):
    """Sub-block parameters (nblk x 16 fp32) -> (sc, m, d, dmin) of the
    format, all decisions in fp32 (rint ties to even)."""
    a = np.asarray(a, F32)
    nblk = a.shape[0]
    if fmt == Q2_K:
        a = np.maximum(a, F32(0))
        b = np.maximum(np.asarray(b, F32), F32(0))
        d = _f16(a.max(axis=1) / F32(15)).astype(F32)
        dm = _f16(b.max(axis=1) / F32(15)).astype(F32)
        with np.errstate(divide="ignore", invalid="ignore"):
            sc = np.where(d[:, None] > 0, np.rint(a / d[:, None]), 0)
            m = np.where(dm[:, None] > 0, np.rint(b / dm[:, None]), 0)
        return (np.clip(sc, 0, 15).astype(np.int64), np.clip(m, 0, 15).astype(np.int64), d, dm)
    d = _f16(np.abs(a).max(axis=1) / F32(31)).astype(F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        sc = np.where(d[:, None] > 0, np.rint(a / d[:, None]), 0)
    return np.clip(sc, -32, 31).astype(np.int64), np.zeros((nblk, 16), np.int64), d, \
        np.zeros(nblk, F32)


def nearest_codes(fmt: int, w, a, b):
    """Per weight the nearest level a q - b (first on ties), in fp32;
    w: nblk x 256, a, b: nblk x 16 fp32 (the quantized sub-block values)."""
    w = np.asarray(w, F32)
    A = np.repeat(np.asarray(a, F32), 16, axis=1)
    B = np.repeat(np.asarray(b, F32), 16, axis=1)
    lv = _levels(fmt)
    best = np.full(w.shape, np.inf, F32)
    code = np.zeros(w.shape, np.int64)
    for k in lv:
        dist = np.abs(w - ((A * F32(k)).astype(F32) - B).astype(F32)).astype(F32)
        better = dist < best
        best = np.where(better, dist, best)
        code = np.where(better, k, code)
    return code


def start(fmt: int, W) -> np.ndarray:
    """This module's min-max K-Quant of W (N x K, K % 256 == 0): blocks."""
    W = np.asarray(W, F32)
    N, K = W.shape
    w = W.reshape(-1, 256)
    sub = w.reshape(-1, 16, 16)
    if fmt == Q2_K:
        mn = np.minimum(sub.min(axis=2), F32(0))
        mx = sub.max(axis=2)
        a = ((mx - mn) / F32(3)).astype(F32)
        b = (-mn).astype(F32)
    else:
        idx = np.abs(sub).argmax(axis=2)
        we = np.take_along_axis(sub, idx[..., None], axis=2)[..., 0]
        a = (-we / F32(4)).astype(F32)
        b = np.zeros_like(a)
    sc, m, d, dm = project(fmt, a, b)
    aq = (d[:, None] * sc.astype(F32)).astype(F32)
    bq = (dm[:, None] * m.astype(F32)).astype(F32)
    q = nearest_codes(fmt, w, aq, bq)
    return encode(fmt, q, sc, m, d, dm)


# ---------------------------------------------------------------- the step

@dataclass
class KqState:
    fmt: int
    N: int
    K: int
    logits: np.ndarray   # (L, N, K) float32
    mom: np.ndarray
    a: np.ndarray        # (N, K / 16) float32
    ma: np.ndarray
    b: np.ndarray
    mb: np.ndarray
    q0: np.ndarray       # (N, K) int64: start codes
    seed: int = 0
    t: int = 0
    row0: int = 0        # first row of the layer (noise is keyed by the global coordinate)


def init_state(fmt: int, blocks, N: int, K: int, seed: int = 0, row0: int = 0) -> KqState:
    q, sc, m, d, dm = decode(fmt, blocks)
    a = (d[:, None] * sc.astype(F32)).astype(F32).reshape(N, K // 16)
    b = (dm[:, None] * m.astype(F32)).astype(F32).reshape(N, K // 16)
    q = q.reshape(N, K)
    L = NUM_LOGITS[fmt]
    logits = np.zeros((L, N, K), F32)
    if fmt == Q2_K:
        for k in range(4):
            logits[k][q == k] = 2.0
    else:
        logits[2] = 2.0
    return KqState(fmt, N, K, logits, np.zeros_like(logits), a, np.zeros_like(a), b,
                   np.zeros_like(b), q, seed, 0, row0)


def candidates(st: KqState) -> np.ndarray:
    """(L, N, K) level values c_k of every coordinate."""
    if st.fmt == Q2_K:
        return np.broadcast_to(np.arange(4, dtype=np.float64)[:, None, None],
                               (4, st.N, st.K)).copy()
    return np.stack([np.clip(st.q0 + k - 2, -4, 3) for k in range(5)]).astype(np.float64)


def noise(st: KqState, t: int) -> np.ndarray:
    mode = GRID_2BIT if st.fmt == Q2_K else GRID_3BIT_LOCAL
    u = uniforms(mode, st.seed, t, st.row0 * st.K, st.N * st.K).astype(np.float64)
    return (-np.log(-np.log(u))).T.reshape(-1, st.N, st.K)


def soft_weight(st: KqState, tau: float, t: int | None = None, use_noise: bool = True):
    """(y (L,N,K), u (N,K), w fp64, w_bf16 fp32) at step t."""
    t = st.t if t is None else t
    g = noise(st, t) if use_noise else 0.0
    z = (st.logits.astype(np.float64) + g) / float(tau)
    z -= z.max(axis=0, keepdims=True)
    y = np.exp(z)
    y /= y.sum(axis=0, keepdims=True)
    u = (y * candidates(st)).sum(axis=0)
    A = np.repeat(st.a.astype(np.float64), 16, axis=1)
    B = np.repeat(st.b.astype(np.float64), 16, axis=1)
    w = A * u - B
    return y, u, w, bf16_round(w).astype(F32)


def _lion(theta, mom, grad, lr, b1, b2):
    """Lion in place (the oracle's fp32 Lion: each blend one fused multiply-add)."""
    lion(theta, mom, np.ascontiguousarray(grad, F32), lr, b1, b2)


def gradients(st: KqState, y, u, dW, tau: float):
    """Logit and sub-block parameter gradients from dW (N x K)."""
    c = candidates(st)
    A = np.repeat(st.a.astype(np.float64), 16, axis=1)
    gw = np.asarray(dW, np.float64)
    acc = (y[None] * (c[:, None] - c[None])).sum(axis=1)   # sum_m y_m (c_k - c_m)
    dl = (A * gw / float(tau))[None] * y * acc
    da = (gw * u).reshape(st.N, -1, 16).sum(axis=2)
    db = -gw.reshape(st.N, -1, 16).sum(axis=2)
    return dl, da, db


def step(st: KqState, X, Yref, tau: float, lr: float, b1=0.9, b2=0.99, dumps=False):
    """One GSQ step on the K-Quant grid (in place); returns the loss."""
    y, u, w, wb = soft_weight(st, tau)
    Xb = bf16_round(np.asarray(X, np.float64))
    E = Xb @ wb.astype(np.float64).T - Yref
    loss = float((E * E).sum())
    dY = bf16_round(2.0 * E)
    dW = (dY.T @ Xb).astype(F32)
    dl, da, db = gradients(st, y, u, dW, tau)
    _lion(st.logits, st.mom, dl, lr, b1, b2)
    _lion(st.a, st.ma, da, lr, b1, b2)
    if st.fmt == Q2_K:
        _lion(st.b, st.mb, db, lr, b1, b2)
    st.t += 1
    if dumps:
        return loss, dict(w=w, dW=dW, dl=dl, da=da, db=db)
    return loss


def hard_codes(st: KqState) -> np.ndarray:
    k = np.argmax(st.logits, axis=0)   # first maximum
    if st.fmt == Q2_K:
        return k
    return np.clip(st.q0 + k - 2, -4, 3)


def export(st: KqState) -> np.ndarray:
    """Projection back into the format: hard codes and the re-encoded
    sub-block parameters."""
    nblk = st.N * st.K // 256
    sc, m, d, dm = project(st.fmt, st.a.reshape(nblk, 16), st.b.reshape(nblk, 16))
    return encode(st.fmt, hard_codes(st).reshape(nblk, 256), sc, m, d, dm)


def reference_output(W, X) -> np.ndarray:
    Xb = bf16_round(np.asarray(X, np.float64))
    return Xb @ np.asarray(W, np.float64).T


def recon_error(fmt: int, blocks, X, Yref, N: int, K: int):
    """||bf16(X) W_q^T - Yref||^2 (and relative) of the format's weight."""
    Wq = bf16_round(dequant(fmt, blocks, N, K).astype(np.float64))
    E = bf16_round(np.asarray(X, np.float64)) @ Wq.T - Yref
    e = float((E * E).sum())
    return e, e / float((Yref * Yref).sum())

"""The oracle: ctypes front end of ``gsq_oracle.c``, a plain CPU restatement of
the GSQ Gumbel-Softmax layer-reconstruction step.

Test infrastructure only.  Nothing in the product path may import it: only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` do.  It shares no code with the CUDA library; the two meet only
through the seeded input generators and the arrays the tests hand to both.

Method source: GSQ (arXiv 2604.18556) as summarised on agihunt.info (method
and optimisation paragraphs) and atlas.scime.ai (Approach); Philox4x32-10 from
Salmon et al., "Parallel random numbers: as easy as 1, 2, 3" (SC'11).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

from . import gptq  # noqa: F401  (GPTQ initial assignment, plain numpy)

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gsq_oracle.c")
LIB = os.path.join(HERE, "libgsq_oracle.so")

GRID_2BIT, GRID_TERNARY, GRID_3BIT_LOCAL = 0, 1, 2
NUM_LOGITS = {GRID_2BIT: 4, GRID_TERNARY: 4, GRID_3BIT_LOCAL: 5}
NUM_LEVELS = {GRID_2BIT: 4, GRID_TERNARY: 3, GRID_3BIT_LOCAL: 8}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, no contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(
            os.path.getmtime(SRC), os.path.getmtime(SRC[:-2] + ".h")):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-fPIC", "-shared", "-o", LIB + ".tmp", SRC,
               "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(LIB + ".tmp", LIB)
    return LIB


_lib = None

_i64, _i32, _u32, _u64 = C.c_int64, C.c_int, C.c_uint32, C.c_uint64
_f32, _f64, _p = C.c_float, C.c_double, C.c_void_p


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        sigs = {
            "gsqo_num_logits": (_i32, [_i32]),
            "gsqo_philox4x32_10": (None, [_p, _p, _p]),
            "gsqo_u01": (_f32, [_u32]),
            "gsqo_uniforms": (None, [_i32, _u64, _u32, _u64, _i64, _p]),
            "gsqo_bf16_round": (_f64, [_f64]),
            "gsqo_f16_round": (_f64, [_f64]),
            "gsqo_f16_bits": (C.c_uint16, [_f64]),
            "gsqo_init": (_i32, [_i32, _i64, _i64, _i32, _p, _p, _p, _p, _p, _p, _p]),
            "gsqo_reference_output": (None, [_i64, _i64, _i64, _p, _p, _p]),
            "gsqo_soft_weight": (None, [_i32, _i64, _i64, _i64, _i32, _p, _p, _p,
                                        _u64, _u32, _f32, _i32, _p, _p, _p, _p]),
            "gsqo_forward": (_f64, [_i64, _i64, _i64, _p, _p, _p, _p]),
            "gsqo_weight_grad": (None, [_i64, _i64, _i64, _p, _p, _p]),
            "gsqo_backward": (None, [_i32, _i64, _i64, _i32, _p, _p, _p, _p, _p,
                                     _f32, _p, _p]),
            "gsqo_lion": (None, [_i64, _p, _p, _p, _f32, _f32, _f32]),
            "gsqo_bf16_sr": (_f32, [_f32, _u32]),
            "gsqo_state16_store": (None, [_i32, _i64, _i64, _i64, _u64, _u32, _p, _p]),
            "gsqo_step": (_i32, [_i32, _i64, _i64, _i64, _i64, _i32, _p, _p, _p,
                                 _p, _p, _p, _p, _u64, _u32, _f32, _f32, _f32,
                                 _f32, _i32, _p, _p, _p, _p, _p, _p]),
            "gsqo_backward_lion": (_i32, [_i32, _i64, _i64, _i64, _i32, _p, _p,
                                          _p, _p, _p, _p, _u64, _u32, _f32,
                                          _f32, _f32, _f32, _i32, _p, _p]),
            "gsqo_harden": (None, [_i32, _i64, _i64, _p, _p, _p]),
            "gsqo_packed_words_per_row": (_i64, [_i32, _i64]),
            "gsqo_pack": (None, [_i32, _i64, _i64, _p, _p]),
            "gsqo_unpack": (None, [_i32, _i64, _i64, _p, _p]),
            "gsqo_recon_error": (None, [_i32, _i32, _i64, _i64, _i64, _i32, _p,
                                        _p, _p, _p, _p, _f32, _p, _p]),
            "gsqo_gemm_abt": (None, [_i64, _i64, _i64, _p, _p, _p]),
            "gsqo_scale_backward_lion": (None, [_i32, _i64, _i64, _i32, _p, _p, _p,
                                                _p, _p, _f32, _f32, _f32, _p]),
            "gsqo_scale_step": (_i32, [_i32, _i64, _i64, _i64, _i32, _p, _p, _p,
                                       _p, _p, _p, _f32, _f32, _f32, _p, _p, _p,
                                       _p]),
            "gsqo_mlp_forward_backward": (_f64, [_i64, _i64, _i64, _p, _p, _p, _p,
                                                 _p, _i32, _p, _p, _p]),
            "gsqo_attn_probs": (None, [_i64, _i64, _i64, _i64, _i64, _f64, _p, _p,
                                       _p, _i32, _p]),
            "gsqo_attn_prob_row": (None, [_i64, _i64, _i64, _i64, _i64, _f64, _p, _p,
                                          _p, _i32, _i64, _i64, _i64, _p]),
            "gsqo_attn_vo_forward_backward": (_f64, [_i64, _i64, _i64, _i64, _i64,
                                                     _p, _p, _p, _p, _p, _i32, _p, _p]),
        }
        for name, (res, args) in sigs.items():
            f = getattr(_lib, name)
            f.restype = res
            f.argtypes = args
    return _lib


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "arrays handed to the oracle must be contiguous"
    return a.ctypes.data


def _f32a(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ------------------------------------------------------------------ Philox

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, np.uint32)
    lib().gsqo_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def u01(x: int) -> float:
    return lib().gsqo_u01(x)


def uniforms(mode: int, seed: int, t: int, coord0: int, count: int) -> np.ndarray:
    L = NUM_LOGITS[mode]
    out = np.zeros((count, L), np.float32)
    lib().gsqo_uniforms(mode, seed, t, coord0, count, _ptr(out))
    return out


def bf16_round(x) -> np.ndarray:
    f = np.vectorize(lib().gsqo_bf16_round, otypes=[np.float64])
    return f(np.asarray(x, dtype=np.float64))


def f16_bits(x) -> np.ndarray:
    f = np.vectorize(lib().gsqo_f16_bits, otypes=[np.uint16])
    return f(np.asarray(x, dtype=np.float64))


# ------------------------------------------------------------------ state

@dataclass
class State:
    mode: int
    N: int
    K: int
    group: int
    logits: np.ndarray   # (L, N, K) float32
    mom: np.ndarray      # (L, N, K) float32
    s: np.ndarray        # (N, G) float32
    ms: np.ndarray       # (N, G) float32
    i0: np.ndarray       # (N, K) int8
    row0: int = 0
    seed: int = 0
    t: int = 0
    noise: bool = True
    # bf16 logits and momenta (the reduced-memory mode): after each Lion
    # update the logits are rounded stochastically and the momenta to nearest
    state16: bool = False

    def copy(self) -> "State":
        return State(self.mode, self.N, self.K, self.group, self.logits.copy(),
                     self.mom.copy(), self.s.copy(), self.ms.copy(),
                     self.i0.copy(), self.row0, self.seed, self.t, self.noise,
                     self.state16)


def bf16_sr(x: float, r9: int) -> float:
    """Stochastic rounding of an fp32 value to bf16 with a 9-bit threshold."""
    return lib().gsqo_bf16_sr(x, r9)


def state16_store(st: "State", t_next: int) -> None:
    """Rounds st.logits (stochastically) and st.mom (to nearest) to bf16 in
    place, thresholds from the Philox words of step t_next."""
    lib().gsqo_state16_store(st.mode, st.row0, st.N, st.K, st.seed, t_next,
                             _ptr(st.logits), _ptr(st.mom))


def init(mode: int, W, group: int = 128, init_idx=None, seed: int = 0,
         row0: int = 0, state16: bool = False) -> State:
    W = _f32a(W)
    N, K = W.shape
    L = NUM_LOGITS[mode]
    G = K // group
    st = State(mode, N, K, group, np.zeros((L, N, K), np.float32),
               np.zeros((L, N, K), np.float32), np.zeros((N, G), np.float32),
               np.zeros((N, G), np.float32), np.zeros((N, K), np.int8),
               row0=row0, seed=seed)
    ii = None if init_idx is None else np.ascontiguousarray(init_idx, np.int8)
    rc = lib().gsqo_init(mode, N, K, group, _ptr(W), _ptr(ii), _ptr(st.s),
                         _ptr(st.i0), _ptr(st.logits), _ptr(st.mom), _ptr(st.ms))
    if rc != 0:
        raise ValueError(f"gsqo_init failed ({rc})")
    st.state16 = state16  # the initial logits (0, +2) and momenta (0) are bf16 values
    return st


def reference_output(W, X) -> np.ndarray:
    W, X = _f32a(W), _f32a(X)
    N, K = W.shape
    T = X.shape[0]
    Y = np.zeros((T, N), np.float64)
    lib().gsqo_reference_output(N, K, T, _ptr(W), _ptr(X), _ptr(Y))
    return Y


def soft_weight(st: State, tau: float, t: int | None = None, noise=None):
    """Returns (y (L,N,K) f64, v (N,K) f64, w (N,K) f64, w_bf16 (N,K) f32)."""
    t = st.t if t is None else t
    noise = st.noise if noise is None else noise
    L, N, K = st.logits.shape
    y = np.zeros((L, N, K)); v = np.zeros((N, K)); w = np.zeros((N, K))
    wb = np.zeros((N, K), np.float32)
    lib().gsqo_soft_weight(st.mode, st.row0, N, K, st.group, _ptr(st.logits),
                           _ptr(st.s), _ptr(st.i0), st.seed, t, tau, int(noise),
                           _ptr(y), _ptr(v), _ptr(w), _ptr(wb))
    return y, v, w, wb


def forward(X, Wb, Yref):
    X, Wb = _f32a(X), _f32a(Wb)
    Yref = np.ascontiguousarray(Yref, np.float64)
    T, K = X.shape
    N = Wb.shape[0]
    dY = np.zeros((T, N), np.float32)
    loss = lib().gsqo_forward(N, K, T, _ptr(X), _ptr(Wb), _ptr(Yref), _ptr(dY))
    return loss, dY


def weight_grad(dY, X):
    dY, X = _f32a(dY), _f32a(X)
    T, K = X.shape
    N = dY.shape[1]
    dW = np.zeros((N, K), np.float32)
    lib().gsqo_weight_grad(N, K, T, _ptr(dY), _ptr(X), _ptr(dW))
    return dW


def backward(st: State, y, v, dW, tau: float):
    L, N, K = st.logits.shape
    y = np.ascontiguousarray(y, np.float64)
    v = np.ascontiguousarray(v, np.float64)
    dW = _f32a(dW)
    dl = np.zeros((L, N, K), np.float32)
    ds = np.zeros_like(st.s)
    lib().gsqo_backward(st.mode, N, K, st.group, _ptr(y), _ptr(v), _ptr(st.s),
                        _ptr(st.i0), _ptr(dW), tau, _ptr(dl), _ptr(ds))
    return dl, ds


def lion(theta, mom, grad, lr, beta1, beta2):
    """In place on float32 arrays."""
    assert theta.dtype == np.float32 and mom.dtype == np.float32
    g = _f32a(grad)
    lib().gsqo_lion(theta.size, _ptr(theta), _ptr(mom), _ptr(g), lr, beta1, beta2)


def step(st: State, X, Yref, tau: float, lr: float, beta1: float = 0.9,
         beta2: float = 0.99, dumps: bool = False):
    """One step in place; returns loss (and a dict of intermediates if dumps)."""
    X = _f32a(X)
    Yref = np.ascontiguousarray(Yref, np.float64)
    L, N, K = st.logits.shape
    T = X.shape[0]
    d = {}
    if dumps:
        d = dict(w=np.zeros((N, K)), dY=np.zeros((T, N), np.float32),
                 dW=np.zeros((N, K), np.float32),
                 dl=np.zeros((L, N, K), np.float32),
                 ds=np.zeros_like(st.s))
    loss = C.c_double(0.0)
    rc = lib().gsqo_step(st.mode, st.row0, N, K, T, st.group, _ptr(st.logits),
                         _ptr(st.mom), _ptr(st.s), _ptr(st.ms), _ptr(st.i0),
                         _ptr(X), _ptr(Yref), st.seed, st.t, tau, lr, beta1,
                         beta2, int(st.noise), C.byref(loss),
                         _ptr(d.get("w")), _ptr(d.get("dY")), _ptr(d.get("dW")),
                         _ptr(d.get("dl")), _ptr(d.get("ds")))
    if rc != 0:
        raise RuntimeError(f"gsqo_step failed ({rc})")
    if st.state16:
        state16_store(st, st.t + 1)
    st.t += 1
    return (loss.value, d) if dumps else loss.value


def backward_lion(st: State, dW, tau, lr, beta1=0.9, beta2=0.99):
    """A5 alone from a given dW at the state's current step (t unchanged)."""
    L, N, K = st.logits.shape
    dW = _f32a(dW)
    dl = np.zeros((L, N, K), np.float32)
    ds = np.zeros_like(st.s)
    rc = lib().gsqo_backward_lion(st.mode, st.row0, N, K, st.group,
                                  _ptr(st.logits), _ptr(st.mom), _ptr(st.s),
                                  _ptr(st.ms), _ptr(st.i0), _ptr(dW), st.seed,
                                  st.t, tau, lr, beta1, beta2, int(st.noise),
                                  _ptr(dl), _ptr(ds))
    if rc != 0:
        raise RuntimeError(f"gsqo_backward_lion failed ({rc})")
    if st.state16:
        state16_store(st, st.t + 1)
    return dl, ds


def scale_backward_lion(st: State, dW, lr, beta1=0.9, beta2=0.99):
    """Scale-only A5 from a given dW: the assignments frozen at the hard
    choice of st.logits, Lion on st.s / st.ms in place; returns ds."""
    L, N, K = st.logits.shape
    dW = _f32a(dW)
    ds = np.zeros_like(st.s)
    lib().gsqo_scale_backward_lion(st.mode, N, K, st.group, _ptr(st.logits),
                                   _ptr(st.i0), _ptr(st.s), _ptr(st.ms), _ptr(dW),
                                   lr, beta1, beta2, _ptr(ds))
    return ds


def scale_step(st: State, X, Yref, lr: float, beta1: float = 0.9, beta2: float = 0.99,
               dumps: bool = False):
    """One scale-only step in place (logits untouched, t unchanged); returns
    the loss (and the hard weight, dW and ds if dumps)."""
    X = _f32a(X)
    Yref = np.ascontiguousarray(Yref, np.float64)
    L, N, K = st.logits.shape
    T = X.shape[0]
    d = {}
    if dumps:
        d = dict(w=np.zeros((N, K), np.float32), dW=np.zeros((N, K), np.float32),
                 ds=np.zeros_like(st.s))
    loss = C.c_double(0.0)
    rc = lib().gsqo_scale_step(st.mode, N, K, T, st.group, _ptr(st.logits), _ptr(st.i0),
                               _ptr(st.s), _ptr(st.ms), _ptr(X), _ptr(Yref), lr, beta1,
                               beta2, C.byref(loss), _ptr(d.get("w")), _ptr(d.get("dW")),
                               _ptr(d.get("ds")))
    if rc != 0:
        raise RuntimeError(f"gsqo_scale_step failed ({rc})")
    return (loss.value, d) if dumps else loss.value


def harden(mode, logits, i0):
    logits = _f32a(logits)
    L, N, K = logits.shape
    i0 = np.ascontiguousarray(i0, np.int8)
    lev = np.zeros((N, K), np.uint8)
    lib().gsqo_harden(mode, N, K, _ptr(logits), _ptr(i0), _ptr(lev))
    return lev


def packed_words_per_row(mode, K):
    return lib().gsqo_packed_words_per_row(mode, K)


def pack(mode, level):
    level = np.ascontiguousarray(level, np.uint8)
    N, K = level.shape
    out = np.zeros((N, packed_words_per_row(mode, K)), np.uint32)
    lib().gsqo_pack(mode, N, K, _ptr(level), _ptr(out))
    return out


def unpack(mode, packed, K):
    packed = np.ascontiguousarray(packed, np.uint32)
    N = packed.shape[0]
    lev = np.zeros((N, K), np.uint8)
    lib().gsqo_unpack(mode, N, K, _ptr(packed), _ptr(lev))
    return lev


def recon_error(st: State, X, Yref, emode: int = 0, tau: float = 1.0):
    X = _f32a(X)
    Yref = np.ascontiguousarray(Yref, np.float64)
    T = X.shape[0]
    a, r = C.c_double(), C.c_double()
    lib().gsqo_recon_error(st.mode, emode, st.N, st.K, T, st.group,
                           _ptr(st.logits), _ptr(st.s), _ptr(st.i0), _ptr(X),
                           _ptr(Yref), tau, C.byref(a), C.byref(r))
    return a.value, r.value


def gemm_abt(A, B):
    A, B = _f32a(A), _f32a(B)
    M, Kc = A.shape
    N = B.shape[0]
    Cm = np.zeros((M, N))
    lib().gsqo_gemm_abt(M, N, Kc, _ptr(A), _ptr(B), _ptr(Cm))
    return Cm


# ------------------------------------------------- SwiGLU MLP joint stage

MLP_WEIGHTS = ("gate", "up", "down")


def mlp_forward_backward(Xn, R, Wg, Wu, Wd, round_bf16=True):
    """loss, dWg, dWu, dWd of the SwiGLU MLP stage (see gsq_oracle.h)."""
    Xn, Wg, Wu, Wd = _f32a(Xn), _f32a(Wg), _f32a(Wu), _f32a(Wd)
    R = np.ascontiguousarray(R, np.float64)
    T, H = Xn.shape
    F = Wg.shape[0]
    dWg = np.zeros((F, H), np.float32)
    dWu = np.zeros((F, H), np.float32)
    dWd = np.zeros((H, F), np.float32)
    loss = lib().gsqo_mlp_forward_backward(T, H, F, _ptr(Xn), _ptr(R), _ptr(Wg),
                                           _ptr(Wu), _ptr(Wd), int(round_bf16),
                                           _ptr(dWg), _ptr(dWu), _ptr(dWd))
    return loss, dWg, dWu, dWd


def weight_seed(seed: int, which: int) -> int:
    """Philox key of weight `which` of a block stage: the seed's high key word
    xored with which << 16, so every weight draws its own stream."""
    return (seed ^ (which << 48)) & 0xFFFFFFFFFFFFFFFF


@dataclass
class MlpState:
    gate: State
    up: State
    down: State
    t: int = 0

    def weights(self):
        return (self.gate, self.up, self.down)


def mlp_init(mode, Wg, Wu, Wd, group=128, seed=0):
    sts = [init(mode, W, group, seed=weight_seed(seed, i))
           for i, W in enumerate((Wg, Wu, Wd))]
    return MlpState(*sts)


def mlp_step(ms: MlpState, Xn, R, tau, lr, beta1=0.9, beta2=0.99, dumps=False):
    """One joint step: soft weights of the three weights (their own noise),
    SwiGLU forward/backward against R, then backward + Lion per weight."""
    wb = []
    for st in ms.weights():
        st.t = ms.t
        wb.append(soft_weight(st, tau)[3])
    loss, dWg, dWu, dWd = mlp_forward_backward(Xn, R, *wb)
    for st, dW in zip(ms.weights(), (dWg, dWu, dWd)):
        backward_lion(st, dW, tau, lr, beta1, beta2)
    ms.t += 1
    for st in ms.weights():
        st.t = ms.t
    if dumps:
        return loss, dict(w=wb, dW=(dWg, dWu, dWd))
    return loss


def mlp_recon_error(ms: MlpState, Xn, R, emode=0, tau=1.0):
    """||MLP(Xn) - R||^2 with the hard (emode 0) or noiseless soft (1) weights."""
    ws = []
    for st in ms.weights():
        if emode == 0:
            lev = harden(st.mode, st.logits, st.i0)
            vals = np.array([-1.5, -0.5, 0.5, 1.5]) if st.mode == GRID_2BIT else (
                np.array([-1.0, 0.0, 1.0]) if st.mode == GRID_TERNARY else np.arange(8) - 3.5)
            w = np.repeat(st.s, st.group, axis=1).astype(np.float64) * vals[lev]
            ws.append(bf16_round(w).astype(np.float32))
        else:
            ws.append(soft_weight(st, tau, noise=False)[3])
    loss, _, _, _ = mlp_forward_backward(Xn, R, *ws)
    return loss, loss / float((np.asarray(R, np.float64) ** 2).sum())


# ---------------------------------------------- attention V/O joint stage

def attn_probs(Xa, Wq, Wk, nseq, S, nh, nkv, d=128, theta=500000.0, round_bf16=True):
    """P[s, h, q, key] from the frozen query/key weights (see gsq_oracle.h)."""
    Xa, Wq, Wk = _f32a(Xa), _f32a(Wq), _f32a(Wk)
    P = np.zeros((nseq, nh, S, S), np.float32)
    lib().gsqo_attn_probs(nseq, S, nh, nkv, d, theta, _ptr(Xa), _ptr(Wq), _ptr(Wk),
                          int(round_bf16), _ptr(P))
    return P


def attn_prob_row(Xa, Wq, Wk, nseq, S, nh, nkv, s, h, q, d=128, theta=500000.0,
                  round_bf16=True):
    """P[s, h, q, :] computed on its own (d <= 256)."""
    Xa, Wq, Wk = _f32a(Xa), _f32a(Wq), _f32a(Wk)
    row = np.zeros(S, np.float32)
    lib().gsqo_attn_prob_row(nseq, S, nh, nkv, d, theta, _ptr(Xa), _ptr(Wq), _ptr(Wk),
                             int(round_bf16), s, h, q, _ptr(row))
    return row


def attn_vo_forward_backward(Xa, P, R, Wv, Wo, nseq, S, nh, nkv, d=128, round_bf16=True):
    Xa, P, Wv, Wo = _f32a(Xa), _f32a(P), _f32a(Wv), _f32a(Wo)
    R = np.ascontiguousarray(R, np.float64)
    H = nh * d
    dWv = np.zeros((nkv * d, H), np.float32)
    dWo = np.zeros((H, H), np.float32)
    loss = lib().gsqo_attn_vo_forward_backward(nseq, S, nh, nkv, d, _ptr(Xa), _ptr(P),
                                                _ptr(R), _ptr(Wv), _ptr(Wo),
                                                int(round_bf16), _ptr(dWv), _ptr(dWo))
    return loss, dWv, dWo


@dataclass
class AttnState:
    v: State
    o: State
    t: int = 0

    def weights(self):
        return (self.v, self.o)


def attn_init(mode, Wv, Wo, group=128, seed=0):
    return AttnState(init(mode, Wv, group, seed=weight_seed(seed, 0)),
                     init(mode, Wo, group, seed=weight_seed(seed, 1)))


def attn_step(at: AttnState, Xa, P, R, dims, tau, lr, beta1=0.9, beta2=0.99, dumps=False):
    """One joint V/O step; dims = (nseq, S, nh, nkv, d)."""
    wb = []
    for st in at.weights():
        st.t = at.t
        wb.append(soft_weight(st, tau)[3])
    loss, dWv, dWo = attn_vo_forward_backward(Xa, P, R, wb[0], wb[1], *dims)
    for st, dW in zip(at.weights(), (dWv, dWo)):
        backward_lion(st, dW, tau, lr, beta1, beta2)
    at.t += 1
    for st in at.weights():
        st.t = at.t
    if dumps:
        return loss, dict(w=wb, dW=(dWv, dWo))
    return loss


def attn_recon_error(at: AttnState, Xa, P, R, dims, emode=0, tau=1.0):
    ws = []
    for st in at.weights():
        if emode == 0:
            lev = harden(st.mode, st.logits, st.i0)
            vals = np.array([-1.5, -0.5, 0.5, 1.5]) if st.mode == GRID_2BIT else (
                np.array([-1.0, 0.0, 1.0]) if st.mode == GRID_TERNARY else np.arange(8) - 3.5)
            w = np.repeat(st.s, st.group, axis=1).astype(np.float64) * vals[lev]
            ws.append(bf16_round(w).astype(np.float32))
        else:
            ws.append(soft_weight(st, tau, noise=False)[3])
    loss, _, _ = attn_vo_forward_backward(Xa, P, R, ws[0], ws[1], *dims)
    return loss, loss / float((np.asarray(R, np.float64) ** 2).sum())

"""Pins of the oracle of GSQ on GGUF K-Quant formats (oracle/kquant.py): GSQ
starts from an existing K-Quant, optimises, and projects the result back into
the same format (agihunt.info summary, optimisation and results paragraphs).
CPU only.

* the block encoding and the dequantisation formula equal the ``gguf``
  package's K-Quant dequantizer (a library routine) on random blocks, and
  encode(decode(b)) == b;
* the start: every weight code is the nearest level of its sub-block (brute
  force, first on ties), every sub-block code the nearest integer to a / d
  within the format's range;
* projecting an unmoved state back gives the starting blocks bit for bit;
* logit and sub-block parameter gradients match central differences of the
  exact (unrounded) loss; logit gradients sum to zero per coordinate;
* tau -> 0 without noise collapses the soft weight to the hard one.
Planted mistakes in copies of oracle/kquant.py are each caught by a pin."""
import importlib.util
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def KQ(oracle_mod):
    from oracle import kquant
    return kquant


def weight(N=4, K=512, seed=3):
    from post_weight_quantization_philox_b200 import synth
    return synth.make_weight(synth.small_config(N, K, 8, 0, number=78), seed=seed)


def random_blocks(KQ, fmt, n, seed, full_range=False):
    rng = np.random.default_rng(seed)
    q = rng.integers(KQ.QMIN[fmt], KQ.QMAX[fmt] + 1, (n, 256))
    if fmt == KQ.Q2_K:
        sc = rng.integers(0, 16, (n, 16))
        m = rng.integers(0, 16, (n, 16))
        if full_range:
            sc[:, 3] = 15
            m[:, 5] = 15
        dmin = rng.uniform(1e-4, 2e-3, n)
    else:
        sc = rng.integers(-32, 32, (n, 16))
        m = np.zeros((n, 16), np.int64)
        if full_range:
            sc[:, 3] = 31
            sc = np.clip(sc, -31, 31)
        dmin = np.zeros(n)
    d = rng.uniform(1e-4, 2e-3, n)
    return KQ.encode(fmt, q, sc, m, d, dmin)


# ------------------------------------------------------------------ pins

def pin_layout_matches_gguf(KQ):
    import gguf
    from gguf import GGMLQuantizationType as G
    for fmt, qt in ((KQ.Q2_K, G.Q2_K), (KQ.Q3_K, G.Q3_K)):
        blk = random_blocks(KQ, fmt, 9, 1 + fmt)
        ref = gguf.quants.dequantize(blk, qt).reshape(9, 256)
        assert np.array_equal(KQ.dequant(fmt, blk, 9, 256), ref), fmt
        # arbitrary bytes (with sane fp16 factors) decode and re-encode exactly
        raw = np.random.default_rng(5).integers(0, 256, blk.shape).astype(np.uint8)
        for off in ((80, 82) if fmt == KQ.Q2_K else (108,)):
            raw[:, off:off + 2] = np.array([0.003], np.float16).view(np.uint8)
        assert np.array_equal(KQ.encode(fmt, *KQ.decode(fmt, raw)), raw), fmt
        assert np.array_equal(KQ.dequant(fmt, raw, 9, 256),
                              gguf.quants.dequantize(raw, qt).reshape(9, 256)), fmt


def pin_start_is_nearest(KQ):
    W = weight()
    for fmt in (KQ.Q2_K, KQ.Q3_K):
        blk = KQ.start(fmt, W)
        q, sc, m, d, dm = KQ.decode(fmt, blk)
        w = W.reshape(-1, 256).astype(np.float32)
        a = (d[:, None] * sc.astype(np.float32)).astype(np.float32)
        b = (dm[:, None] * m.astype(np.float32)).astype(np.float32)
        A, B = np.repeat(a, 16, axis=1), np.repeat(b, 16, axis=1)
        lv = np.arange(KQ.QMIN[fmt], KQ.QMAX[fmt] + 1)
        dist = np.stack([np.abs(w - ((A * np.float32(k)).astype(np.float32) - B)) for k in lv])
        assert np.array_equal(q, lv[np.argmin(dist, axis=0)]), fmt
        # sub-block codes: the nearest integer to the continuous value over
        # the format's range, against the start's own continuous values
        sub = w.reshape(-1, 16, 16)
        if fmt == KQ.Q2_K:
            mn = np.minimum(sub.min(axis=2), 0)
            cont = [((sub.max(axis=2) - mn) / np.float32(3)).astype(np.float32), -mn]
            codes, dens, rng_ = [sc, m], [d, dm], range(0, 16)
        else:
            idx = np.abs(sub).argmax(axis=2)
            we = np.take_along_axis(sub, idx[..., None], axis=2)[..., 0]
            cont, codes, dens, rng_ = [(-we / np.float32(4)).astype(np.float32)], [sc], [d], \
                range(-32, 32)
        for x, c, den in zip(cont, codes, dens):
            cand = np.array(list(rng_))
            err = np.abs(x[..., None] / den[:, None, None] - cand)
            best = err.min(axis=-1)
            mine = np.abs(x / den[:, None] - c)
            assert np.all(mine <= best + 1e-6), fmt


def pin_projection_round_trip(KQ):
    for fmt in (KQ.Q2_K, KQ.Q3_K):
        blk = random_blocks(KQ, fmt, 8, 11 + fmt, full_range=True)
        st = KQ.init_state(fmt, blk, 2, 1024)
        assert np.array_equal(KQ.export(st), blk), fmt


def _exact_loss(KQ, st, X, Y, tau, t):
    _, _, w, _ = KQ.soft_weight(st, tau, t)
    E = X @ w.T - Y
    return float((E * E).sum()), 2.0 * E.T @ X


def pin_gradients_central_differences(KQ):
    rng = np.random.default_rng(4)
    for fmt in (KQ.Q2_K, KQ.Q3_K):
        W = weight(2, 256, seed=7)
        X = rng.normal(0, 1, (6, 256))
        Y = X @ W.astype(np.float64).T
        st = KQ.init_state(fmt, KQ.start(fmt, W), 2, 256, seed=9)
        st.logits[:] = rng.normal(0, 1, st.logits.shape).astype(np.float32)
        st.b[:] = np.abs(st.b) + np.float32(1e-3)
        tau, t = 0.7, 3
        _, dW = _exact_loss(KQ, st, X, Y, tau, t)
        y, u, _, _ = KQ.soft_weight(st, tau, t)
        dl, da, db = KQ.gradients(st, y, u, dW, tau)
        assert np.allclose(dl.sum(axis=0), 0, atol=1e-9 * np.abs(dl).max())
        for arr, grad, idx in ((st.logits, dl, (1, 0, 37)), (st.logits, dl, (0, 1, 200)),
                               (st.a, da, (0, 3)), (st.a, da, (1, 15))) + \
                (((st.b, db, (0, 5)),) if fmt == KQ.Q2_K else ()):
            h = 1e-3 * max(1.0, abs(float(arr[idx])))
            old = arr[idx]
            arr[idx] = old + h
            lp, _ = _exact_loss(KQ, st, X, Y, tau, t)
            arr[idx] = old - h
            lm, _ = _exact_loss(KQ, st, X, Y, tau, t)
            arr[idx] = old
            h2 = (np.float64(np.float32(old + h)) - np.float64(np.float32(old - h)))
            fd = (lp - lm) / h2
            assert abs(fd - grad[idx]) <= 2e-3 * abs(fd) + 1e-6, (fmt, idx, fd, grad[idx])


def pin_tau_to_zero_is_hard(KQ):
    for fmt in (KQ.Q2_K, KQ.Q3_K):
        W = weight(2, 512, seed=12)
        st = KQ.init_state(fmt, KQ.start(fmt, W), 2, 512, seed=1)
        # distinct logits one apart: at tau 1e-4 the softmax is one-hot in fp64
        r = np.random.default_rng(2).random(st.logits.shape)
        st.logits[:] = np.argsort(np.argsort(r, axis=0), axis=0).astype(np.float32)
        _, _, w, _ = KQ.soft_weight(st, 1e-4, 0, use_noise=False)
        c = KQ.hard_codes(st)
        hard = np.repeat(st.a, 16, axis=1).astype(np.float64) * c - \
            np.repeat(st.b, 16, axis=1).astype(np.float64)
        assert np.allclose(w, hard, rtol=0, atol=1e-12), fmt


# ----------------------------------------------------------------- tests

def test_layout_matches_gguf(KQ):
    pin_layout_matches_gguf(KQ)


def test_start_is_nearest(KQ):
    pin_start_is_nearest(KQ)


def test_projection_round_trip(KQ):
    pin_projection_round_trip(KQ)


def test_gradients_central_differences(KQ):
    pin_gradients_central_differences(KQ)


def test_tau_to_zero_is_hard(KQ):
    pin_tau_to_zero_is_hard(KQ)


def test_steps_improve_the_start(KQ, oracle_mod):
    """A short GSQ run lowers the reconstruction error of the exported blocks
    below that of the starting K-Quant."""
    from post_weight_quantization_philox_b200 import synth
    rng = np.random.default_rng(6)
    N, K, T = 32, 512, 256
    W = weight(N, K, seed=21)
    X = synth.bf16_values(rng.normal(0, 1, (T, K)))
    Y = KQ.reference_output(W, X)
    for fmt in (KQ.Q2_K, KQ.Q3_K):
        blk = KQ.start(fmt, W)
        e0 = KQ.recon_error(fmt, blk, X, Y, N, K)[1]
        st = KQ.init_state(fmt, blk, N, K, seed=2)
        # one lr for logits and sub-block parameters: small enough that the
        # noisy early steps do not throw the sub-block scales off
        for tau in synth.tau_schedule(1.0, 0.05, 60):
            KQ.step(st, X, Y, float(tau), 1e-5)
        e1 = KQ.recon_error(fmt, KQ.export(st), X, Y, N, K)[1]
        assert e1 < e0, (fmt, e1, e0)


# ------------------------------------------------------- planted mistakes

MUTATIONS = [
    ("code_bit_order", "<< (2 * s[k])).astype(np.uint8)", "<< (2 * (3 - s[k]))).astype(np.uint8)",
     lambda K: pin_layout_matches_gguf(K)),
    ("q3_scale_offset", "us = np.asarray(sc, np.int64) + 32", "us = np.asarray(sc, np.int64) + 31",
     lambda K: pin_layout_matches_gguf(K)),
    ("sub_scale_floor", "sc = np.where(d[:, None] > 0, np.rint(a / d[:, None]), 0)\n            m",
     "sc = np.where(d[:, None] > 0, np.floor(a / d[:, None]), 0)\n            m",
     lambda K: pin_start_is_nearest(K)),
    ("q3_scale_range", "d = _f16(np.abs(a).max(axis=1) / F32(31)).astype(F32)",
     "d = _f16(np.abs(a).max(axis=1) / F32(32)).astype(F32)",
     lambda K: pin_projection_round_trip(K)),
    ("logit_grad_without_scale", "dl = (A * gw / float(tau))[None] * y * acc",
     "dl = (gw / float(tau))[None] * y * acc", lambda K: pin_gradients_central_differences(K)),
    ("min_grad_sign", "db = -gw.reshape(st.N, -1, 16).sum(axis=2)",
     "db = gw.reshape(st.N, -1, 16).sum(axis=2)", lambda K: pin_gradients_central_differences(K)),
    ("local_shift_unclamped", "return np.clip(st.q0 + k - 2, -4, 3)",
     "return st.q0 + k - 2", lambda K: pin_tau_to_zero_is_hard(K)),
]


def mutated(name, old, new):
    src = open(os.path.join(ROOT, "oracle", "kquant.py")).read()
    assert src.count(old) == 1, name
    spec = importlib.util.spec_from_loader(f"oracle.kquant_mut_{name}", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    sys.modules[spec.name] = mod
    exec(compile(src.replace(old, new), f"kquant_mut_{name}", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(oracle_mod, name, old, new, pin):
    with pytest.raises(AssertionError):
        pin(mutated(name, old, new))

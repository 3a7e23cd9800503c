"""Pins of the oracle's scale-only step (assignments frozen at the hard
choice of the logits, only the group scales trained; agihunt.info summary,
optimisation paragraph): central differences of the plain loss in the
scales, zero loss and zero gradient for on-grid weights, Lion's first-step
closed form, agreement with the full backward at a one-hot assignment.
CPU only."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

LEVELS = {0: np.array([-1.5, -0.5, 0.5, 1.5]), 1: np.array([-1.0, 0.0, 1.0]),
          2: np.arange(8) - 3.5}


def _exact_scales(st, rng):
    """Scales k / 64 with (2 c_max) (k + 1) < 256: every s c and
    (s +- 1/64) c is a bf16 value, so the hard weight carries no rounding."""
    kmax = {0: 64, 1: 64, 2: 35}[st.mode]
    st.s[...] = rng.integers(16, kmax + 1, size=st.s.shape) / 64.0


def _hard_weight(oracle_mod, st):
    lev = oracle_mod.harden(st.mode, st.logits, st.i0)
    vals = LEVELS[st.mode][lev]
    return np.repeat(st.s.astype(np.float64), st.group, axis=1) * vals


def _loss(X, W, Yref):
    E = X.astype(np.float64) @ W.T - Yref
    return float((E * E).sum())


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_scale_grad_central_differences(oracle_mod, mode):
    rng = np.random.default_rng(10 + mode)
    N, K, T = 3, 256, 48
    W = rng.normal(0, 0.5, (N, K)).astype(np.float32)
    X = synth.bf16_values(rng.normal(0, 1, (T, K)))  # the GEMM operand is bf16(X)
    Yref = X.astype(np.float64) @ (W.astype(np.float64) * 0.9).T
    st = oracle_mod.init(mode, W)
    _exact_scales(st, rng)
    s0 = st.s.copy()
    loss, d = oracle_mod.scale_step(st.copy(), X, Yref, 1e-3, dumps=True)
    assert np.isclose(loss, _loss(X, _hard_weight(oracle_mod, st), Yref), rtol=1e-12)
    h = 1.0 / 64
    G = K // st.group
    Wh = _hard_weight(oracle_mod, st)
    E = X.astype(np.float64) @ Wh.T - Yref
    c = Wh / np.repeat(s0.astype(np.float64), st.group, axis=1)  # level values
    for n in range(N):
        for g in range(G):
            sp, sm = st.copy(), st.copy()
            sp.s[n, g] = s0[n, g] + h
            sm.s[n, g] = s0[n, g] - h
            # the loss is quadratic in s_g, so the central difference is exact
            fd = (_loss(X, _hard_weight(oracle_mod, sp), Yref) -
                  _loss(X, _hard_weight(oracle_mod, sm), Yref)) / (2 * h)
            # the oracle's dW comes from bf16(2E) (relative error <= 2^-9 per
            # entry) as the GEMM operand, then fp32
            cols = slice(g * st.group, (g + 1) * st.group)
            xc = X[:, cols].astype(np.float64) @ c[n, cols]
            bound = 2.0 ** -9 * np.sum(np.abs(2 * E[:, n]) * np.abs(xc))
            bound += 1e-6 * np.sum(np.abs(2 * E[:, n])[:, None] * np.abs(X[:, cols] * c[n, cols]))
            assert abs(d["ds"][n, g] - fd) <= bound, (n, g, d["ds"][n, g], fd, bound)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_scale_step_on_grid_weight_is_a_fixed_point(oracle_mod, mode):
    rng = np.random.default_rng(20 + mode)
    N, K, T = 4, 256, 32
    vals = LEVELS[mode]
    lev = rng.integers(0, len(vals), size=(N, K))
    lev[:, ::128] = len(vals) - 1  # every group holds the top level: s = absmax / c_max
    kmax = {0: 64, 1: 64, 2: 35}[mode]  # s c exact in bf16
    s = rng.integers(16, kmax + 1, size=(N, K // 128)) / 64.0
    W = (np.repeat(s, 128, axis=1) * vals[lev]).astype(np.float32)
    X = synth.bf16_values(rng.normal(0, 1, (T, K)))
    Yref = X.astype(np.float64) @ W.astype(np.float64).T
    st = oracle_mod.init(mode, W)
    assert np.array_equal(st.s, s.astype(np.float32))
    loss, d = oracle_mod.scale_step(st, X, Yref, 1e-2, dumps=True)
    assert loss == 0.0
    assert np.all(d["ds"] == 0) and np.all(d["dW"] == 0)
    assert np.array_equal(st.s, s.astype(np.float32)) and np.all(st.ms == 0)


def test_scale_lion_first_step_closed_form(oracle_mod):
    rng = np.random.default_rng(30)
    N, K = 5, 384
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    st = oracle_mod.init(0, W)
    dW = rng.normal(0, 1e-2, (N, K)).astype(np.float32)
    s0 = st.s.copy()
    lr, b1, b2 = np.float32(1e-3), np.float32(0.9), np.float32(0.99)
    ds = oracle_mod.scale_backward_lion(st, dW, float(lr), float(b1), float(b2))
    assert np.array_equal(st.s, (s0 - lr * np.sign(ds)).astype(np.float32))
    assert np.array_equal(st.ms, (np.float32(1) - b2) * ds)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_scale_grad_equals_full_backward_at_one_hot(oracle_mod, mode):
    """With the noise off and tau -> 0 the soft assignment is one-hot at the
    argmax, so the full backward's scale gradient must equal the
    scale-only one (given the same dW)."""
    rng = np.random.default_rng(40 + mode)
    N, K = 3, 256
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    st = oracle_mod.init(mode, W)
    st.noise = False
    dW = rng.normal(0, 1e-2, (N, K)).astype(np.float32)
    _, ds_full = oracle_mod.backward_lion(st.copy(), dW, 1e-6, 1e-3)
    ds_scale = oracle_mod.scale_backward_lion(st.copy(), dW, 1e-3)
    assert np.allclose(ds_scale, ds_full, rtol=1e-6, atol=0)


def test_scale_steps_reduce_the_loss(oracle_mod):
    rng = np.random.default_rng(50)
    N, K, T = 8, 256, 64
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    X = rng.normal(0, 1, (T, K)).astype(np.float32)
    Yref = oracle_mod.reference_output(W, X)
    st = oracle_mod.init(0, W)
    losses = [oracle_mod.scale_step(st, X, Yref, 2e-4) for _ in range(15)]
    assert losses[-1] < 0.9 * losses[0]

"""Pins of the oracle's GPTQ initial assignment (Frantar et al., ICLR 2023;
GSQ starts from it: agihunt.info summary, optimisation paragraph): exact
round-to-nearest when the Hessian is diagonal, the first column's update
against the damped least-squares closed form, the optimal-brain-surgeon loss
identity over the whole loop, dead inputs, and a lower error than
round-to-nearest on correlated inputs.  CPU only."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth


def _hadamard(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _correlated(T, K, seed):
    rng = np.random.default_rng(seed)
    base = rng.normal(0, 1, (T, K // 8))
    mix = rng.normal(0, 1, (K // 8, K))
    return synth.bf16_values(base @ mix + 0.3 * rng.normal(0, 1, (T, K)))


def test_bf16_rounding_matches_torch(oracle_mod):
    G = oracle_mod.gptq
    x = np.random.default_rng(0).normal(0, 3, 10000).astype(np.float32)
    assert np.array_equal(G._bf16(x), synth.bf16_values(x).astype(np.float64))


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_diagonal_hessian_is_round_to_nearest(oracle_mod, mode):
    """Orthogonal input columns: H is diagonal, U is diagonal, no error is
    fed forward, so GPTQ equals round-to-nearest with absmax scales."""
    G = oracle_mod.gptq
    K = 256
    X = _hadamard(K)[:, :K] * 0.5  # exact in bf16, X^T X = (K / 4) I
    W = np.random.default_rng(1 + mode).normal(0, 0.02, (64, K)).astype(np.float32)
    lev, s, err, _, _ = G.gptq(mode, W, X)
    st = oracle_mod.init(mode, W)
    assert np.array_equal(s, st.s)
    rtn = st.i0 if mode == 2 else oracle_mod.harden(mode, st.logits, st.i0)
    assert np.array_equal(lev.astype(np.int64), rtn.astype(np.int64))


@pytest.mark.parametrize("mode", [0, 2])
def test_first_column_update_is_damped_least_squares(oracle_mod, mode):
    """After fixing column 0 to its grid value q0, the other columns must
    minimise (w' - w)^T H (w' - w): w'_(1..) = w_(1..) + H_(1..,1..)^-1 H_(1..,0) (w0 - q0)."""
    G = oracle_mod.gptq
    K, N = 128, 8
    X = _correlated(96, K, 2)
    W = np.random.default_rng(3).normal(0, 0.02, (N, K)).astype(np.float32)
    lev, s, err, Wafter, H = G.gptq(mode, W, X, cols=1)
    q0 = s[:, 0].astype(np.float64) * G.LEVELS[mode][lev[:, 0]]
    d0 = W[:, 0].astype(np.float64) - q0
    step = np.linalg.solve(H[1:, 1:], H[1:, 0])
    expect = W[:, 1:].astype(np.float64) + np.outer(d0, step)
    assert np.allclose(Wafter[:, 1:], expect, rtol=1e-9, atol=1e-14)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_loss_identity_over_the_loop(oracle_mod, mode):
    """Optimal brain surgeon: fixing column j raises (w - w0)^T H (w - w0) by
    exactly err_j^2, so the final loss of every row is the sum of its err^2."""
    G = oracle_mod.gptq
    K, N = 256, 12
    X = _correlated(200, K, 4 + mode)
    W = np.random.default_rng(5 + mode).normal(0, 0.02, (N, K)).astype(np.float32)
    lev, s, err, _, H = G.gptq(mode, W, X)
    Q = G.quantized(mode, lev, s)
    D = Q - W.astype(np.float64)
    loss = np.einsum("nk,kl,nl->n", D, H, D)
    assert np.allclose(loss, (err ** 2).sum(axis=1), rtol=1e-8)


def test_dead_inputs_are_zeroed(oracle_mod):
    G = oracle_mod.gptq
    K = 128
    X = _correlated(64, K, 6)
    X[:, [3, 77]] = 0.0
    W = np.random.default_rng(7).normal(0, 0.02, (6, K)).astype(np.float32)
    lev, s, err, Wafter, H = G.gptq(0, W, X)
    assert np.all(np.isfinite(err)) and np.all(np.isfinite(s))
    Q = G.quantized(0, lev, s)
    # a dead input contributes nothing to the loss, and its weight is rounded from 0
    assert np.allclose(np.abs(Q[:, [3, 77]]), 0.5 * s[:, 0:1])


@pytest.mark.parametrize("mode", [0, 2])
def test_gptq_beats_round_to_nearest_on_correlated_inputs(oracle_mod, mode):
    G = oracle_mod.gptq
    K, N = 256, 32
    X = _correlated(512, K, 8)
    W = np.random.default_rng(9).normal(0, 0.02, (N, K)).astype(np.float32)
    lev, s, _, _, H = G.gptq(mode, W, X)
    st = oracle_mod.init(mode, W)
    rtn_lev = st.i0 if mode == 2 else oracle_mod.harden(mode, st.logits, st.i0)
    W64 = W.astype(np.float64)

    def loss(Q):
        D = Q - W64
        return np.einsum("nk,kl,nl->", D, H, D)

    assert loss(G.quantized(mode, lev, s)) < 0.9 * loss(G.quantized(mode, rtn_lev, st.s))

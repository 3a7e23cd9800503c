"""Pins of the oracle's SwiGLU MLP joint stage (the block's MLP trained on
the block output; GSQ staging, agihunt.info summary, optimisation paragraph):
torch autograd in fp64, central finite differences, zero loss on the exact
target, and rounding consistency.  CPU only."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth


def _problem(T=16, H=128, F=256, seed=0):
    rng = np.random.default_rng(seed)
    Xn = rng.normal(0, 1, (T, H)).astype(np.float32)
    Wg = rng.normal(0, 0.05, (F, H)).astype(np.float32)
    Wu = rng.normal(0, 0.05, (F, H)).astype(np.float32)
    Wd = rng.normal(0, 0.05, (H, F)).astype(np.float32)
    R = rng.normal(0, 0.1, (T, H))
    return Xn, R, Wg, Wu, Wd


def _torch_loss_and_grads(Xn, R, Wg, Wu, Wd):
    import torch
    X = torch.tensor(Xn, dtype=torch.float64)
    g = torch.tensor(Wg, dtype=torch.float64, requires_grad=True)
    u = torch.tensor(Wu, dtype=torch.float64, requires_grad=True)
    d = torch.tensor(Wd, dtype=torch.float64, requires_grad=True)
    a = X @ g.T
    b = X @ u.T
    pred = (torch.nn.functional.silu(a) * b) @ d.T
    loss = ((pred - torch.tensor(R)) ** 2).sum()
    loss.backward()
    return loss.item(), g.grad.numpy(), u.grad.numpy(), d.grad.numpy()


def test_mlp_matches_torch_autograd(oracle_mod):
    Xn, R, Wg, Wu, Wd = _problem()
    loss, dWg, dWu, dWd = oracle_mod.mlp_forward_backward(Xn, R, Wg, Wu, Wd, round_bf16=False)
    tl, tg, tu, td = _torch_loss_and_grads(Xn, R, Wg, Wu, Wd)
    assert np.isclose(loss, tl, rtol=1e-12)
    for ours, ref in ((dWg, tg), (dWu, tu), (dWd, td)):
        assert np.allclose(ours, ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


def test_mlp_central_differences(oracle_mod):
    Xn, R, Wg, Wu, Wd = _problem(T=8, H=128, F=128, seed=1)
    _, dWg, dWu, dWd = oracle_mod.mlp_forward_backward(Xn, R, Wg, Wu, Wd, round_bf16=False)
    rng = np.random.default_rng(2)
    h = 2.0 ** -12
    for which, W, dW in ((0, Wg, dWg), (1, Wu, dWu), (2, Wd, dWd)):
        for _ in range(6):
            i, j = rng.integers(W.shape[0]), rng.integers(W.shape[1])
            Wp, Wm = W.copy(), W.copy()
            Wp[i, j] += h
            Wm[i, j] -= h
            args_p = [Wg, Wu, Wd]; args_p[which] = Wp
            args_m = [Wg, Wu, Wd]; args_m[which] = Wm
            lp = oracle_mod.mlp_forward_backward(Xn, R, *args_p, round_bf16=False)[0]
            lm = oracle_mod.mlp_forward_backward(Xn, R, *args_m, round_bf16=False)[0]
            fd = (lp - lm) / (2 * h)
            assert abs(dW[i, j] - fd) <= 1e-4 * (abs(fd) + 1e-3 * np.abs(dW).max())


def test_mlp_zero_loss_on_its_own_output(oracle_mod):
    Xn, _, Wg, Wu, Wd = _problem(seed=3)
    a = Xn.astype(np.float64) @ Wg.T.astype(np.float64)
    b = Xn.astype(np.float64) @ Wu.T.astype(np.float64)
    R = (a / (1 + np.exp(-a)) * b) @ Wd.T.astype(np.float64)
    loss, dWg, dWu, dWd = oracle_mod.mlp_forward_backward(Xn, R, Wg, Wu, Wd, round_bf16=False)
    assert loss < 1e-20
    assert np.abs(dWg).max() < 1e-9 and np.abs(dWd).max() < 1e-9


def test_mlp_bf16_rounding_is_a_small_perturbation(oracle_mod):
    Xn, R, Wg, Wu, Wd = _problem(seed=4)
    l0, g0, u0, d0 = oracle_mod.mlp_forward_backward(Xn, R, Wg, Wu, Wd, round_bf16=False)
    l1, g1, u1, d1 = oracle_mod.mlp_forward_backward(Xn, R, Wg, Wu, Wd, round_bf16=True)
    assert abs(l1 - l0) <= 1e-2 * l0
    for a, b in ((g0, g1), (u0, u1), (d0, d1)):
        assert np.linalg.norm(a - b) <= 2e-2 * np.linalg.norm(a)


def test_mlp_step_uses_distinct_noise_per_weight(oracle_mod):
    """Each weight of a stage draws from its own Philox key."""
    ks = {oracle_mod.weight_seed(5, i) for i in range(3)}
    assert len(ks) == 3
    u = [oracle_mod.uniforms(0, oracle_mod.weight_seed(5, i), 0, 0, 64) for i in range(3)]
    assert not np.array_equal(u[0], u[1]) and not np.array_equal(u[1], u[2])
    # the key's high word carries the weight index in bits 16..
    assert (oracle_mod.weight_seed(5, 2) >> 32) == (2 << 16)


def test_mlp_step_trajectory_reduces_loss(oracle_mod):
    T, H, F = 32, 128, 256
    rng = np.random.default_rng(6)
    Xn = rng.normal(0, 1, (T, H)).astype(np.float32)
    Wg = synth.bf16_values(rng.normal(0, 0.05, (F, H)).astype(np.float32))
    Wu = synth.bf16_values(rng.normal(0, 0.05, (F, H)).astype(np.float32))
    Wd = synth.bf16_values(rng.normal(0, 0.05, (H, F)).astype(np.float32))
    a = Xn.astype(np.float64) @ Wg.T.astype(np.float64)
    b = Xn.astype(np.float64) @ Wu.T.astype(np.float64)
    R = (a / (1 + np.exp(-a)) * b) @ Wd.T.astype(np.float64)
    ms = oracle_mod.mlp_init(0, Wg, Wu, Wd, seed=7)
    r0 = oracle_mod.mlp_recon_error(ms, Xn, R, 0)[1]
    for tau in synth.tau_schedule(1.0, 0.05, 30):
        oracle_mod.mlp_step(ms, Xn, R, float(tau), 5e-3)
    r1 = oracle_mod.mlp_recon_error(ms, Xn, R, 0)[1]
    assert 0 < r1 < r0

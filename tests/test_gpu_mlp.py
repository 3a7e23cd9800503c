"""Parity of the SwiGLU MLP block stage (gate, up, down quantized jointly
against the block output) with the oracle, through the C ABI.  Needs a B200.
Tolerances as in test_gpu_parity: bit-exact init, soft weights within the
fp32 contract, loss 1e-2, weight gradients 1e-2 normwise, Lion identical
away from near-ties, final hard reconstruction error within 2%."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    return gsq


def bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def mlp_fp(Xn, Wg, Wu, Wd):
    a = Xn.astype(np.float64) @ Wg.T.astype(np.float64)
    b = Xn.astype(np.float64) @ Wu.T.astype(np.float64)
    return (a / (1.0 + np.exp(-a)) * b) @ Wd.T.astype(np.float64)


def case(T, H, F, seed=11):
    Xn, Wg, Wu, Wd = synth.make_mlp_stage(T, H, F, seed=seed)
    R = mlp_fp(Xn, Wg, Wu, Wd).astype(np.float32)  # the full-precision output
    return Xn, R, Wg, Wu, Wd


SHAPES = [(256, 256, 512), (128, 384, 640)]


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_mlp_init_bit_exact(g, oracle_mod, mode):
    Xn, R, Wg, Wu, Wd = case(*SHAPES[0])
    m = g.gsq_mlp_init(Xn, R, Wg, Wu, Wd, grid_mode=mode, seed=3)
    ms = oracle_mod.mlp_init(mode, Wg, Wu, Wd, seed=3)
    for i, st in enumerate(ms.weights()):
        assert np.array_equal(m.get(i, g.GSQ_DBG_SCALES), st.s)
        assert np.array_equal(m.get(i, g.GSQ_DBG_LOGITS), st.logits)
    RT = m.get(g.GSQ_MLP_STAGE, g.GSQ_MLP_DBG_RT)
    assert np.array_equal(RT, R.T)
    m.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES)
def test_mlp_one_step(g, oracle_mod, mode, shape):
    T, H, F = shape
    Xn, R, Wg, Wu, Wd = case(T, H, F)
    m = g.gsq_mlp_init(Xn, R, Wg, Wu, Wd, grid_mode=mode, seed=9)
    ms = oracle_mod.mlp_init(mode, Wg, Wu, Wd, seed=9)
    tau, lr = 0.7, 1e-3
    m.step(tau, lr)
    loss, d = oracle_mod.mlp_step(ms, Xn, R.astype(np.float64), tau, lr, dumps=True)
    assert abs(m.last_loss() - loss) <= 1e-2 * loss
    for i in range(3):
        wb = bits_to_f32(m.get(i, g.GSQ_DBG_WHAT))
        assert (wb != d["w"][i]).mean() < 1e-3
        dW = m.get(i, g.GSQ_DBG_DW)
        ref = d["dW"][i]
        assert np.linalg.norm(dW - ref) / np.linalg.norm(ref) < 1e-2
        agree = (m.get(i, g.GSQ_DBG_LOGITS) == ms.weights()[i].logits).mean()
        assert agree > 0.99
    # stage intermediates against the oracle's soft weights
    aT = m.get(g.GSQ_MLP_STAGE, g.GSQ_MLP_DBG_AT)
    a_ref = Xn.astype(np.float64) @ d["w"][0].T.astype(np.float64)
    assert np.linalg.norm(aT.T - a_ref) / np.linalg.norm(a_ref) < 1e-3
    m.close()


@pytest.mark.parametrize("mode", [0, 2])
def test_mlp_trajectory(g, oracle_mod, mode):
    T, H, F = SHAPES[0]
    Xn, R, Wg, Wu, Wd = case(T, H, F, seed=21)
    m = g.gsq_mlp_init(Xn, R, Wg, Wu, Wd, grid_mode=mode, seed=0)
    ms = oracle_mod.mlp_init(mode, Wg, Wu, Wd, seed=0)
    R64 = R.astype(np.float64)
    r0 = oracle_mod.mlp_recon_error(ms, Xn, R64, 0)[1]
    for tau in synth.tau_schedule(1.0, 0.05, 15):
        m.step(float(tau), 2e-3)
        loss = oracle_mod.mlp_step(ms, Xn, R64, float(tau), 2e-3)
        assert abs(m.last_loss() - loss) <= 1e-2 * loss
    a, r = m.recon_error(g.GSQ_RECON_HARD)
    ra, rr = oracle_mod.mlp_recon_error(ms, Xn, R64, 0)
    assert abs(r - rr) <= 0.02 * rr
    if mode == 0:  # 2-bit at this lr: the joint stage beats round-to-nearest
        assert rr < r0
    for i in range(3):
        packed, h16, f32 = m.harden_pack(i)
        st = ms.weights()[i]
        lev_ref = oracle_mod.harden(mode, st.logits, st.i0)
        lev = oracle_mod.unpack(mode, packed.reshape(st.N, -1), st.K)
        assert (lev == lev_ref).mean() > 0.99
    m.close()


def test_mlp_run_equals_step_loop_bit_exact(g):
    T, H, F = SHAPES[1]
    Xn, R, Wg, Wu, Wd = case(T, H, F, seed=31)
    taus = synth.tau_schedule(1.0, 0.1, 8)
    a = g.gsq_mlp_init(Xn, R, Wg, Wu, Wd, grid_mode=0, seed=4)
    b = g.gsq_mlp_init(Xn, R, Wg, Wu, Wd, grid_mode=0, seed=4)
    for tau in taus:
        a.step(float(tau), 1e-3)
    b.run(taus, 1e-3)
    assert a.last_loss() == b.last_loss()
    for i in range(3):
        for buf in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES):
            assert np.array_equal(a.get(i, buf), b.get(i, buf))
    a.close(); b.close()


def token_losses_vs_oracle(g, oracle_mod, m, Xn, R, tokens):
    """The step's loss per token from the GPU's output gradient (bf16 of
    2 (pred - R), H x T) against the oracle's MLP forward of that token with
    the GPU's own soft weights of the step (the loss is a sum over tokens)."""
    dpt = bits_to_f32(m.get(g.GSQ_MLP_STAGE, g.GSQ_MLP_DBG_DPT)).astype(np.float64)
    gpu = ((dpt / 2.0) ** 2).sum(0)
    assert gpu.sum() == pytest.approx(m.last_loss(), rel=1e-2)
    Wh = [bits_to_f32(m.get(i, g.GSQ_DBG_WHAT)) for i in range(3)]
    for t in tokens:
        ref = oracle_mod.mlp_forward_backward(Xn[t:t + 1], R[t:t + 1], *Wh)[0]
        assert gpu[t] == pytest.approx(ref, rel=1e-2), t


def test_mlp_full_70b_shape(g, oracle_mod):
    """The 70B block MLP (H 8192, F 28672) on 8 x 2048 tokens in the bench's
    launch configuration: GEMM identities on sampled entries; each step's loss
    on sampled tokens against the oracle, after the first step and after a
    fused run."""
    import torch
    cfg = synth.MLP_STAGE["c5_70b_mlp"]
    T, H, F = cfg["T"], cfg["H"], cfg["F"]
    Xn, Wg, Wu, Wd = synth.make_mlp_stage(T, H, F)
    R = synth.random_target(T, H, 0.05)
    dev = lambda x: torch.from_numpy(x).cuda().to(torch.bfloat16)
    m = g.gsq_mlp_init(dev(Xn), torch.from_numpy(R).cuda(), dev(Wg), dev(Wu), dev(Wd),
                       grid_mode=cfg["grid"], seed=0)
    taus = synth.tau_schedule(1.0, 0.05, cfg["steps"])
    m.step(float(taus[0]), 1e-3)
    token_losses_vs_oracle(g, oracle_mod, m, Xn, R, [0, 5000, T - 1])
    m.run(taus[1:3], 1e-3)
    token_losses_vs_oracle(g, oracle_mod, m, Xn, R, [1, 12345])
    rng = np.random.default_rng(0)
    for i in range(3):
        assert np.isfinite(bits_to_f32(m.get(i, g.GSQ_DBG_WHAT))).all()
    # GEMM identity on sampled entries: a^T[f, t] = sum_k G[f, k] Xn[t, k]
    aT = m.get(g.GSQ_MLP_STAGE, g.GSQ_MLP_DBG_AT)
    G = bits_to_f32(m.get(0, g.GSQ_DBG_WHAT))
    for f, t in zip(rng.integers(0, F, 8), rng.integers(0, T, 8)):
        ref = float(np.dot(G[f].astype(np.float64), Xn[t].astype(np.float64)))
        assert abs(aT[f, t] - ref) <= 1e-3 * (abs(ref) + 1e-2)
    m.close()


def test_mlp_full_70b_shape_first_soft_weights(g, oracle_mod):
    """Step-0 soft weights of the 70B MLP shapes on sampled rows equal the
    oracle's (within the soft-weight contract)."""
    import torch
    cfg = synth.MLP_STAGE["c5_70b_mlp"]
    T, H, F = 64, cfg["H"], cfg["F"]  # token count does not enter the soft weights
    Xn, Wg, Wu, Wd = synth.make_mlp_stage(T, H, F)
    R = synth.random_target(T, H, 0.05)
    dev = lambda x: torch.from_numpy(x).cuda().to(torch.bfloat16)
    m = g.gsq_mlp_init(dev(Xn), torch.from_numpy(R).cuda(), dev(Wg), dev(Wu), dev(Wd),
                       grid_mode=cfg["grid"], seed=0)
    m.step(1.0, 0.0)  # lr 0: the step's soft weights stay in What
    rng = np.random.default_rng(1)
    for i, W in enumerate((Wg, Wu, Wd)):
        what = bits_to_f32(m.get(i, g.GSQ_DBG_WHAT))
        for n in rng.integers(0, W.shape[0], size=3):
            st = oracle_mod.init(cfg["grid"], W[n:n + 1], seed=oracle_mod.weight_seed(0, i),
                                 row0=int(n))
            _, _, w, wb = oracle_mod.soft_weight(st, 1.0, t=0)
            floor = np.repeat(st.s, 128, 1) * 1.5
            half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(w), 1e-30))) - 8)
            assert np.all(np.abs(what[n] - w[0]) <= 1e-5 * (np.abs(w[0]) + floor[0]) + half_ulp[0])
    m.close()

"""Parity of the bf16-state mode (gsq_init_bf16_state: logits and Lion momenta
stored as bf16, the logits rounded stochastically after each Lion update with
thresholds from the next step's Philox words, the momenta to nearest) with
the oracle's state16 mode, through the C ABI.  Needs a B200.

Tolerances as in test_gpu_parity: init bit-exact; logit and scale gradients
at 1e-5 given identical dW and state; the stored logits and momenta
identical wherever the oracle's momentum blend is not a near-tie (the
stochastic rounding is a deterministic function of the fp32 update and the
Philox word, so it adds no tolerance of its own); per-step loss 1e-2 and the
final hard error within 2% over trajectories; gsq_run equal to a loop of
gsq_step bit for bit; checkpoints bit-exact."""
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


def bits(x):
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def f32(b):
    return (np.asarray(b).astype(np.uint32) << 16).view(np.float32)


def case(mode, N, K, T, number=91):
    cfg = synth.small_config(N, K, T, mode, number=number, outlier_cols=4, outlier_scale=10.0)
    return synth.make_weight(cfg), synth.make_calib(cfg)


def layer(g, W, X, mode, seed):
    import torch
    return g.gsq_init(torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda(), 128, mode,
                      seed=seed, state_bf16=True)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_init_bit_exact(g, oracle_mod, mode):
    W, X = case(mode, 200, 384, 136)
    lay = layer(g, W, X, mode, seed=5)
    st = oracle_mod.init(mode, W, seed=5, state16=True)
    assert np.array_equal(lay.get(g.GSQ_DBG_LOGITS), bits(st.logits))
    assert np.array_equal(lay.get(g.GSQ_DBG_MOM), bits(st.mom))
    assert np.array_equal(lay.get(g.GSQ_DBG_SCALES), st.s)
    lay.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_backward_lion_given_identical_dw(g, oracle_mod, mode):
    N, K, T = 256, 512, 128
    W, X = case(mode, N, K, T)
    lay = layer(g, W, X, mode, seed=21)
    st = oracle_mod.init(mode, W, seed=21, state16=True)
    logits = f32(bits(synth.random_logits(st.logits.shape, 8, ties=False)))
    mom = f32(bits(synth.random_grad(st.logits.shape, 9, scale=1e-3)))
    st.logits[:] = logits
    st.mom[:] = mom
    lay.set(g.GSQ_DBG_LOGITS, bits(logits))
    lay.set(g.GSQ_DBG_MOM, bits(mom))
    dW = synth.random_grad((N, K), 10, scale=1.0)
    lay.set(g.GSQ_DBG_DW, dW)
    tau, lr = 0.4, 1e-3
    lay.backward(tau, lr)
    s0 = st.s.copy()
    dl_ref, ds_ref = oracle_mod.backward_lion(st, dW, tau, lr)
    a = np.abs(np.repeat(s0, 128, 1) * dW) / tau
    assert np.all(np.abs(lay.get(g.GSQ_DBG_DL) - dl_ref) <= 1e-5 * (np.abs(dl_ref) + a[None]))
    c = 0.9 * mom.astype(np.float64) + 0.1 * dl_ref
    clear = np.abs(c) > 0.1 * 1e-5 * (np.abs(dl_ref) + a[None]) + 1e-12
    assert clear.mean() > 0.99
    new_l = f32(lay.get(g.GSQ_DBG_LOGITS))
    assert np.array_equal(new_l[clear], st.logits[clear])
    # stored values are bf16: the stochastic rounding moved some logits by a
    # whole bf16 unit although lr is far below half a unit for most of them
    assert np.mean(new_l != logits) > 0.05
    new_m = f32(lay.get(g.GSQ_DBG_MOM))
    # momenta: the fp32 blend within (1 - beta2) times the gradient tolerance,
    # then the same nearest bf16 unless that lands on a rounding boundary
    assert np.mean(new_m == st.mom) > 0.999
    lay.close()


@pytest.mark.parametrize("mode,shape", [(0, (256, 512, 256)), (1, (200, 384, 200)),
                                        (2, (136, 256, 72))])
def test_trajectory_matches_oracle(g, oracle_mod, mode, shape):
    N, K, T = shape
    W, X = case(mode, N, K, T)
    steps = 20
    taus = synth.tau_schedule(1.0, 0.05, steps)
    lay = layer(g, W, X, mode, seed=0)
    st = oracle_mod.init(mode, W, seed=0, state16=True)
    Y = oracle_mod.reference_output(W, X)
    for i in range(steps):
        lay.step(float(taus[i]), 1e-3)
        loss_gpu = lay.last_loss()
        loss = oracle_mod.step(st, X, Y, float(taus[i]), 1e-3)
        assert abs(loss_gpu - loss) <= 1e-2 * loss, i
    _, r = g.gsq_recon_error(lay, 0)
    _, rr = oracle_mod.recon_error(st, X, Y, 0)
    assert abs(r - rr) <= 0.02 * rr
    agree = (f32(lay.get(g.GSQ_DBG_LOGITS)) == st.logits).mean()
    assert agree > 0.99
    packed, _, _ = g.gsq_harden_pack(lay)
    lev = oracle_mod.unpack(mode, packed.reshape(N, -1), K)
    assert (lev == oracle_mod.harden(mode, st.logits, st.i0)).mean() > 0.99
    lay.close()


@pytest.mark.parametrize("mode", [0, 2])
def test_run_equals_step_loop_and_checkpoint(g, mode):
    W, X = case(mode, 256, 512, 128)
    taus = synth.tau_schedule(1.0, 0.05, 10)
    a = layer(g, W, X, mode, seed=3)
    b = layer(g, W, X, mode, seed=3)
    for tau in taus:
        a.step(float(tau), 1e-3)
    b.run(taus[:4], 1e-3)
    buf = g.gsq_export_state(b)
    c = layer(g, W, X, mode, seed=3)
    g.gsq_import_state(c, buf)
    b.run(taus[4:], 1e-3)
    c.run(taus[4:], 1e-3)
    for which in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES, g.GSQ_DBG_SMOM):
        assert np.array_equal(a.get(which), b.get(which))
        assert np.array_equal(b.get(which), c.get(which))
    # half the state bytes of the fp32 mode
    import torch
    d = g.gsq_init(torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda(), 128, mode, seed=3)
    n32, n16 = len(g.gsq_export_state(d)), len(buf)
    L = 5 if mode == 2 else 4
    assert n32 - n16 == 2 * L * 256 * 512 * 2
    for lay in (a, b, c, d):
        lay.close()


def test_full_size_q_proj_row_slices(g, oracle_mod):
    """The q_proj-shaped layer in the benchmark's launch configuration, the
    oracle on a few rows."""
    import torch
    cfg = synth.CONFIGS["c2_qproj_4096x4096"]
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    lay = g.gsq_init(torch.from_numpy(W).cuda().to(torch.bfloat16),
                     torch.from_numpy(X).cuda().to(torch.bfloat16), 128, cfg.grid, seed=0,
                     state_bf16=True)
    taus = synth.tau_schedule(cfg.tau0, cfg.tau1, cfg.steps)[:2]
    lay.run(taus, cfg.lr)
    logits = f32(lay.get(g.GSQ_DBG_LOGITS))
    lay.close()
    for r in (0, 2051, cfg.N - 1):
        st = oracle_mod.init(cfg.grid, W[r:r + 1], seed=0, row0=r, state16=True)
        Y = oracle_mod.reference_output(W[r:r + 1], X)
        for tau in taus:
            oracle_mod.step(st, X, Y, float(tau), cfg.lr)
        assert (logits[:, r] == st.logits[:, 0]).mean() > 0.995, r

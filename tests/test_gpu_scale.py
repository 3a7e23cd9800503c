"""Parity of the scale-only step (assignments frozen at the hard choice of
the logits, only the group scales trained; agihunt.info summary,
optimisation paragraph) with the oracle, through the C ABI.  Needs a B200.

Tolerances as in test_gpu_parity: hard codes bit-exact (checked through the
weight, which is then exact given identical scales); scale gradient
|d ds| <= 1e-5 sum |dW c| given identical dW; Lion identical wherever the
momentum blend is not a near-tie; loss 1e-2 relative."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

pytestmark = pytest.mark.gpu

LEVELS = {0: np.array([-1.5, -0.5, 0.5, 1.5]), 1: np.array([-1.0, 0.0, 1.0]),
          2: np.arange(8) - 3.5}


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


def make(g, mode, N=256, K=512, T=256, seed=3):
    import torch
    cfg = synth.small_config(N, K, T, mode, number=95)
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    lay = g.gsq_init(torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda(), 128, mode,
                     seed=seed)
    return lay, W, X


def oracle_state(g, oracle_mod, lay, W, mode, seed=3):
    """The oracle state with the GPU context's current parameters."""
    st = oracle_mod.init(mode, W, seed=seed)
    st.logits[:] = lay.get(g.GSQ_DBG_LOGITS)
    st.mom[:] = lay.get(g.GSQ_DBG_MOM)
    st.s[:] = lay.get(g.GSQ_DBG_SCALES)
    st.ms[:] = lay.get(g.GSQ_DBG_SMOM)
    return st


def warm(lay, steps=4):
    for tau in synth.tau_schedule(1.0, 0.3, steps):
        lay.step(float(tau), 2e-3)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_scale_backward_given_identical_dw(g, oracle_mod, mode):
    lay, W, X = make(g, mode)
    warm(lay)
    st = oracle_state(g, oracle_mod, lay, W, mode)
    N, K = W.shape
    dW = synth.random_grad((N, K), 31, scale=1.0)
    lay.set(g.GSQ_DBG_DW, dW)
    lr = 1e-3
    ms0 = st.ms.astype(np.float64)
    lay.debug_scale_backward(lr)
    ds_ref = oracle_mod.scale_backward_lion(st, dW, lr)
    ds = lay.get(g.GSQ_DBG_DS)
    lev = oracle_mod.harden(mode, st.logits, st.i0)
    bound = np.abs(dW.astype(np.float64) * LEVELS[mode][lev]).reshape(N, -1, 128).sum(-1)
    assert np.all(np.abs(ds - ds_ref) <= 1e-5 * bound)
    # Lion: both sides start from the same s and ms, so the update is the same
    # wherever the sign of the blend c = b1 m + (1 - b1) ds is decided beyond
    # the gradient tolerance
    c = 0.9 * ms0 + 0.1 * ds_ref.astype(np.float64)
    clear = np.abs(c) > 0.1 * 1e-5 * bound + 1e-12
    assert clear.mean() > 0.99
    s_gpu = lay.get(g.GSQ_DBG_SCALES)
    assert np.array_equal(s_gpu[clear], st.s[clear])
    assert np.all(np.abs(s_gpu - st.s) <= 2 * lr + 1e-7)
    mtol = 0.01 * 1e-5 * bound + 2.0 ** -22 * np.abs(st.ms)
    assert np.all(np.abs(lay.get(g.GSQ_DBG_SMOM) - st.ms) <= mtol)
    lay.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_scale_steps_match_oracle(g, oracle_mod, mode):
    lay, W, X = make(g, mode, seed=5)
    warm(lay)
    st = oracle_state(g, oracle_mod, lay, W, mode, seed=5)
    Y = oracle_mod.reference_output(W, X)
    logits0, mom0 = lay.get(g.GSQ_DBG_LOGITS), lay.get(g.GSQ_DBG_MOM)
    lr = 5e-4
    for i in range(6):
        lay.scale_step(lr)
        loss, d = oracle_mod.scale_step(st, X, Y, lr, dumps=True)
        assert abs(lay.last_loss() - loss) <= 1e-2 * loss, i
        if i == 0:
            # the first hard weight: bit-exact up to double rounding of s c
            wb = bits_to_f32(lay.get(g.GSQ_DBG_WHAT))
            assert (wb != d["w"]).mean() < 1e-3
    s_gpu = lay.get(g.GSQ_DBG_SCALES)
    assert (s_gpu == st.s).mean() > 0.98
    assert np.all(np.abs(s_gpu - st.s) <= 6 * 2 * lr + 1e-6)
    # the assignments and their state stay frozen
    assert np.array_equal(lay.get(g.GSQ_DBG_LOGITS), logits0)
    assert np.array_equal(lay.get(g.GSQ_DBG_MOM), mom0)
    _, r_gpu = g.gsq_recon_error(lay, g.GSQ_RECON_HARD)
    _, r_ref = oracle_mod.recon_error(st, X, Y)
    assert abs(r_gpu - r_ref) <= 0.02 * r_ref
    lay.close()


def test_scale_run_equals_step_loop_bit_exact(g):
    a, W, X = make(g, 0, seed=7)
    b, _, _ = make(g, 0, seed=7)
    for lay in (a, b):
        warm(lay, 3)
    for _ in range(5):
        a.scale_step(1e-3)
    b.scale_run(5, 1e-3)
    assert a.last_loss() == b.last_loss()
    assert np.array_equal(a.get(g.GSQ_DBG_SCALES), b.get(g.GSQ_DBG_SCALES))
    assert np.array_equal(a.get(g.GSQ_DBG_SMOM), b.get(g.GSQ_DBG_SMOM))
    a.close(); b.close()


def test_codes_follow_the_logits(g, oracle_mod):
    """The frozen codes are recomputed after GSQ steps move the logits."""
    lay, W, X = make(g, 2, seed=9)
    lay.scale_step(1e-3)
    warm(lay, 3)
    st = oracle_state(g, oracle_mod, lay, W, 2, seed=9)
    lay.scale_step(1e-3)
    lev = oracle_mod.harden(2, st.logits, st.i0)
    wb = bits_to_f32(lay.get(g.GSQ_DBG_WHAT)).astype(np.float64)
    ref = np.repeat(st.s.astype(np.float64), 128, 1) * LEVELS[2][lev]
    assert np.all(np.abs(wb - ref) <= 2.0 ** -8 * np.abs(ref))
    lay.close()


def test_scale_step_bad_arguments(g):
    lay, _, _ = make(g, 0)
    for args in [(-1e-3, 0.9, 0.99), (1e-3, 1.0, 0.99), (1e-3, 0.9, -0.1)]:
        with pytest.raises(g.GSQError):
            lay.scale_step(*args)
    with pytest.raises(g.GSQError):
        lay.scale_run(0, 1e-3)
    lay.close()


def test_full_size_scale_step_row_slices(g, oracle_mod):
    """The q_proj-shaped layer in the benchmark's launch configuration: one
    scale-only step after init, against the oracle on a slice of rows (the
    loss decomposes over rows)."""
    import torch
    cfg = synth.CONFIGS["c2_qproj_4096x4096"]
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    lay = g.gsq_init(torch.from_numpy(W).cuda().to(torch.bfloat16),
                     torch.from_numpy(X).cuda().to(torch.bfloat16), 128, cfg.grid, seed=0)
    lay.scale_run(2, 1e-3)
    scales = lay.get(g.GSQ_DBG_SCALES)
    assert np.isfinite(lay.last_loss())
    lay.close()
    for r in [0, 7, cfg.N // 2 + 1, cfg.N - 1]:
        Wr = W[r:r + 1]
        st = oracle_mod.init(cfg.grid, Wr, seed=0, row0=r)
        Y = oracle_mod.reference_output(Wr, X)
        for _ in range(2):
            oracle_mod.scale_step(st, X, Y, 1e-3)
        assert (scales[r] == st.s[0]).mean() > 0.9, r
        assert np.allclose(scales[r], st.s[0], rtol=0, atol=4e-3 + 1e-7)

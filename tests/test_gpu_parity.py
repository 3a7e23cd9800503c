"""Parity of the CUDA path (through the C ABI) with the oracle, phase by phase
and over whole trajectories, on seeded synthetic layers.  Needs a B200.

Tolerances (the floating-point contract of the step):
  * Philox uniforms, initial levels, logit init, hard levels, packed codes,
    scale export: bit-exact;
  * soft weight before rounding: |dw| <= 1e-5 (|w| + s c_max);
  * logit gradients: |d dl| <= 1e-5 (|dl| + |a| / tau); scale gradients:
    |d ds| <= 1e-5 sum |dW v| (given identical dW and parameters);
  * loss: 1e-2 relative (bf16 operands, fp32 accumulation); weight gradient:
    1e-2 normwise; reference output: 1e-5 normwise;
  * Lion: identical updates wherever the oracle's momentum blend c is not a
    near-tie (|c| above the gradient tolerance);
  * final hard reconstruction error after the trajectory: within 2%.
"""
import numpy as np
import pytest

import oracle as orc
from post_weight_quantization_philox_b200 import synth

pytestmark = pytest.mark.gpu

LEVEL_MAX = {0: 1.5, 1: 1.0, 2: 3.5}


@pytest.fixture(scope="module")
def g():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    return gsq


def bf16_bits(x):
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def make_case(mode, N, K, T, w_bf16=True, number=90, **kw):
    cfg = synth.small_config(N, K, T, mode, number=number, w_bf16=w_bf16,
                             x_bf16=w_bf16, **kw)
    return cfg, synth.make_weight(cfg), synth.make_calib(cfg)


def gpu_layer(g, W, X, mode, seed=0, init_idx=None, device=True):
    import torch
    if device:
        Wt = torch.from_numpy(W).cuda()
        Xt = torch.from_numpy(X).cuda()
        return g.gsq_init(Wt, Xt, 128, mode, init_idx=init_idx, seed=seed)
    return g.gsq_init(W, X, 128, mode, init_idx=init_idx, seed=seed)


SHAPES = [(256, 512, 256), (200, 384, 200), (136, 256, 72)]


# ------------------------------------------------------------ Philox, init

@pytest.mark.parametrize("mode", [0, 1, 2])
def test_uniforms_bit_exact(g, oracle_mod, mode):
    cfg, W, X = make_case(mode, 8, 128, 8)
    lay = gpu_layer(g, W, X, mode, seed=0xDEADBEEF12345678)
    for t, c0 in [(0, 0), (3, 12345), (77, (1 << 32) - 100)]:
        gpu = lay.uniforms(t, c0, 4096)
        ref = oracle_mod.uniforms(mode, 0xDEADBEEF12345678, t, c0, 4096)
        assert np.array_equal(gpu.view(np.uint32), ref.view(np.uint32))
    lay.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES)
def test_init_bit_exact(g, oracle_mod, mode, shape):
    N, K, T = shape
    cfg, W, X = make_case(mode, N, K, T, w_bf16=(mode != 0))
    W[1, :128] = 0.0  # an all-zero group
    lay = gpu_layer(g, W, X, mode)
    st = oracle_mod.init(mode, W)
    assert np.array_equal(lay.get(g.GSQ_DBG_SCALES), st.s)
    assert np.array_equal(lay.get(g.GSQ_DBG_I0), st.i0)
    assert np.array_equal(lay.get(g.GSQ_DBG_LOGITS), st.logits)
    assert not lay.get(g.GSQ_DBG_MOM).any() and not lay.get(g.GSQ_DBG_SMOM).any()
    # reference output (transposed, padded to a multiple of 64 tokens)
    Y = oracle_mod.reference_output(W, X)
    YT = lay.get(g.GSQ_DBG_YREFT)
    assert not YT[:, T:].any()
    err = np.linalg.norm(YT[:, :T].T - Y) / np.linalg.norm(Y)
    assert err < 1e-5
    lay.close()


def test_init_from_given_levels(g, oracle_mod):
    cfg, W, X = make_case(2, 64, 256, 64)
    idx = np.random.default_rng(1).integers(0, 8, size=W.shape).astype(np.int8)
    lay = gpu_layer(g, W, X, 2, init_idx=idx)
    st = oracle_mod.init(2, W, init_idx=idx)
    assert np.array_equal(lay.get(g.GSQ_DBG_I0), idx)
    assert np.array_equal(lay.get(g.GSQ_DBG_LOGITS), st.logits)
    lay.close()
    bad = idx.copy()
    bad[3, 5] = 9
    with pytest.raises(g.GSQError) as e:
        gpu_layer(g, W, X, 2, init_idx=bad)
    assert e.value.status == g.GSQ_ERR_INVALID_ARG


def test_host_and_device_inputs_agree(g, oracle_mod):
    cfg, W, X = make_case(0, 128, 256, 64)
    a = gpu_layer(g, W, X, 0, device=True)
    b = gpu_layer(g, W, X, 0, device=False)
    for which in (g.GSQ_DBG_SCALES, g.GSQ_DBG_LOGITS, g.GSQ_DBG_YREFT):
        assert np.array_equal(a.get(which), b.get(which))
    a.close(); b.close()


def test_nonfinite_input_is_reported(g):
    cfg, W, X = make_case(0, 128, 256, 64)
    X[3, 7] = np.nan
    with pytest.raises(g.GSQError) as e:
        gpu_layer(g, W, X, 0)
    assert e.value.status == g.GSQ_ERR_NONFINITE


# ---------------------------------------------------------- soft weight

@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES[:2])
def test_soft_weight(g, oracle_mod, mode, shape):
    N, K, T = shape
    cfg, W, X = make_case(mode, N, K, T)
    lay = gpu_layer(g, W, X, mode, seed=11)
    st = oracle_mod.init(mode, W, seed=11)
    logits = synth.random_logits(st.logits.shape, 5, ties=False)
    st.logits[:] = logits
    lay.set(g.GSQ_DBG_LOGITS, logits)
    for tau in (1.0, 0.3, 0.05):
        lay.soft_weight(tau)
        w_gpu = lay.get(g.GSQ_DBG_WSOFT32).astype(np.float64)
        _, _, w, wb = oracle_mod.soft_weight(st, tau)
        floor = np.repeat(st.s, 128, 1) * LEVEL_MAX[mode]
        assert np.all(np.abs(w_gpu - w) <= 1e-5 * (np.abs(w) + floor))
        wb_gpu = bits_to_f32(lay.get(g.GSQ_DBG_WHAT))
        mism = wb_gpu != wb
        assert mism.mean() < 1e-3  # rounding-boundary cases only
        # every GPU bf16 value is the rounding of a value within the fp32
        # tolerance of the oracle's exact soft weight
        if mism.any():
            mag = np.maximum(np.abs(wb[mism]), np.abs(wb_gpu[mism])).astype(np.float64)
            half_ulp = 2.0 ** (np.floor(np.log2(mag)) - 8)
            tol = 1e-5 * (np.abs(w[mism]) + floor[mism]) + half_ulp
            assert np.all(np.abs(wb_gpu[mism] - w[mism]) <= tol * (1 + 1e-9))
    lay.close()


# --------------------------------------------------------------- GEMMs

@pytest.mark.parametrize("shape", [(401, 552, 200), (128, 256, 64), (300, 1000, 4160)])
def test_gemm_entry_matches_oracle(g, oracle_mod, shape):
    import torch
    M, N, Kc = shape
    rng = np.random.default_rng(M + N)
    A = synth.bf16_values(rng.normal(size=(M, Kc)).astype(np.float32))
    B = synth.bf16_values(rng.normal(size=(N, Kc)).astype(np.float32))
    C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    g.gsq_gemm_bf16_abt(torch.from_numpy(A).cuda().to(torch.bfloat16),
                        torch.from_numpy(B).cuda().to(torch.bfloat16), C)
    ref = oracle_mod.gemm_abt(A, B)
    got = C.cpu().numpy().astype(np.float64)
    # fp32 accumulation: error grows like sqrt(Kc) * 2^-24 relative
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 2e-7 * np.sqrt(Kc)
    assert np.max(np.abs(got - ref)) < 1e-4 * np.sqrt(Kc)


@pytest.mark.parametrize("shape", SHAPES)
def test_forward_loss_and_dy(g, oracle_mod, shape):
    N, K, T = shape
    cfg, W, X = make_case(0, N, K, T)
    lay = gpu_layer(g, W, X, 0)
    st = oracle_mod.init(0, W)
    Y = oracle_mod.reference_output(W, X)
    _, _, w, wb = oracle_mod.soft_weight(st, 0.5)
    lay.set(g.GSQ_DBG_WHAT, bf16_bits(wb))
    loss_gpu = lay.forward()
    loss, dY = oracle_mod.forward(X, wb, Y)
    assert abs(loss_gpu - loss) <= 1e-2 * loss
    dYT = bits_to_f32(lay.get(g.GSQ_DBG_DYT))
    assert not dYT[:, T:].any()
    d = dYT[:, :T].T
    assert np.linalg.norm(d - dY) / np.linalg.norm(dY) < 1e-2
    lay.close()


@pytest.mark.parametrize("shape", SHAPES)
def test_weight_gradient(g, oracle_mod, shape):
    N, K, T = shape
    cfg, W, X = make_case(0, N, K, T)
    lay = gpu_layer(g, W, X, 0)
    rng = np.random.default_rng(3)
    dY = synth.bf16_values(rng.normal(0, 0.1, size=(T, N)).astype(np.float32))
    dYT = np.zeros((N, lay.Tp), np.float32)
    dYT[:, :T] = dY.T
    lay.set(g.GSQ_DBG_DYT, bf16_bits(dYT))
    lay.weight_grad()
    dW = lay.get(g.GSQ_DBG_DW)
    ref = oracle_mod.weight_grad(dY, X)
    assert np.linalg.norm(dW - ref) / np.linalg.norm(ref) < 1e-2
    assert np.linalg.norm(dW - ref) / np.linalg.norm(ref) < 1e-5  # fp32 accumulate
    lay.close()


# ------------------------------------------------------ backward + Lion

@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES[:2])
def test_backward_lion_given_identical_dw(g, oracle_mod, mode, shape):
    N, K, T = shape
    cfg, W, X = make_case(mode, N, K, T)
    lay = gpu_layer(g, W, X, mode, seed=21)
    st = oracle_mod.init(mode, W, seed=21)
    logits = synth.random_logits(st.logits.shape, 8, ties=False)
    st.logits[:] = logits
    lay.set(g.GSQ_DBG_LOGITS, logits)
    mom = synth.random_grad(st.logits.shape, 9, scale=1e-3)
    st.mom[:] = mom
    lay.set(g.GSQ_DBG_MOM, mom)
    dW = synth.random_grad((N, K), 10, scale=1.0)
    lay.set(g.GSQ_DBG_DW, dW)
    tau, lr = 0.4, 1e-3
    lay.backward(tau, lr)
    s0 = st.s.copy()
    dl_ref, ds_ref = oracle_mod.backward_lion(st, dW, tau, lr)
    dl = lay.get(g.GSQ_DBG_DL)
    ds = lay.get(g.GSQ_DBG_DS)
    a = np.abs(np.repeat(s0, 128, 1) * dW) / tau
    assert np.all(np.abs(dl - dl_ref) <= 1e-5 * (np.abs(dl_ref) + a[None]))
    y, v, _, _ = oracle_mod.soft_weight(oracle_mod.State(
        mode, N, K, 128, logits, mom, s0, st.ms, st.i0, seed=21), tau)
    bound = (np.abs(dW.astype(np.float64) * v)).reshape(N, -1, 128).sum(-1)
    assert np.all(np.abs(ds - ds_ref) <= 1e-5 * bound)
    # Lion: identical wherever the sign of c is decided beyond the tolerance
    c = 0.9 * mom.astype(np.float64) + 0.1 * dl_ref
    clear = np.abs(c) > 0.1 * 1e-5 * (np.abs(dl_ref) + a[None]) + 1e-12
    new_l = lay.get(g.GSQ_DBG_LOGITS)
    assert clear.mean() > 0.99
    assert np.array_equal(new_l[clear], st.logits[clear])
    # momenta: (1 - beta2) times the gradient tolerance, plus fp32 rounding
    mtol = 0.01 * 1e-5 * (np.abs(dl_ref) + a[None]) + 2.0**-22 * np.abs(st.mom)
    assert np.all(np.abs(lay.get(g.GSQ_DBG_MOM) - st.mom) <= mtol)
    cs = 0.1 * ds_ref.astype(np.float64)
    sclear = np.abs(cs) > 1e-5 * bound * 0.1
    assert np.array_equal(lay.get(g.GSQ_DBG_SCALES)[sclear], st.s[sclear])
    lay.close()


# ---------------------------------------------------------- harden/pack

@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("shape", SHAPES[:2])
def test_harden_pack_bit_exact(g, oracle_mod, mode, shape):
    N, K, T = shape
    cfg, W, X = make_case(mode, N, K, T)
    lay = gpu_layer(g, W, X, mode)
    L = oracle_mod.NUM_LOGITS[mode]
    logits = synth.random_logits((L, N, K), 31 + mode, ties=True)
    lay.set(g.GSQ_DBG_LOGITS, logits)
    i0 = lay.get(g.GSQ_DBG_I0)
    packed, h16, f32 = g.gsq_harden_pack(lay)
    lev = oracle_mod.harden(mode, logits, i0)
    ref = oracle_mod.pack(mode, lev)
    assert np.array_equal(packed.reshape(N, -1), ref)
    s = lay.get(g.GSQ_DBG_SCALES)
    assert np.array_equal(f32, s)
    assert np.array_equal(h16, oracle_mod.f16_bits(s).reshape(s.shape))
    # device output buffers
    import torch
    pd = torch.zeros(packed.size, dtype=torch.int32, device="cuda")
    hd = torch.zeros(s.shape, dtype=torch.int16, device="cuda")
    g.gsq_harden_pack(lay, pd, hd, None)
    assert np.array_equal(pd.cpu().numpy().view(np.uint32), packed)
    assert np.array_equal(hd.cpu().numpy().view(np.uint16), h16)
    lay.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_recon_error(g, oracle_mod, mode):
    cfg, W, X = make_case(mode, 200, 384, 200)
    lay = gpu_layer(g, W, X, mode)
    st = oracle_mod.init(mode, W)
    logits = synth.random_logits(st.logits.shape, 41, ties=False)
    st.logits[:] = logits
    lay.set(g.GSQ_DBG_LOGITS, logits)
    Y = oracle_mod.reference_output(W, X)
    for emode, tau in ((0, 1.0), (1, 0.3)):
        a, r = g.gsq_recon_error(lay, emode, tau)
        ra, rr = oracle_mod.recon_error(st, X, Y, emode, tau)
        assert abs(a - ra) <= 1e-3 * ra and abs(r - rr) <= 1e-3 * rr
    lay.close()


# ---------------------------------------------------------- trajectories

@pytest.mark.parametrize("mode,shape", [(0, (256, 512, 256)), (1, (200, 384, 200)),
                                        (2, (136, 256, 72))])
def test_trajectory_matches_oracle(g, oracle_mod, mode, shape):
    """Whole steps: per-step loss within 1e-2, final hard recon error within 2%."""
    N, K, T = shape
    cfg, W, X = make_case(mode, N, K, T, w_bf16=(mode != 0), outlier_cols=4,
                          outlier_scale=10.0)
    steps = 20
    taus = synth.tau_schedule(1.0, 0.05, steps)
    lay = gpu_layer(g, W, X, mode, seed=0)
    st = oracle_mod.init(mode, W, seed=0)
    Y = oracle_mod.reference_output(W, X)
    for i in range(steps):
        lay.step(float(taus[i]), 1e-3)
        loss_gpu = lay.last_loss()
        loss = oracle_mod.step(st, X, Y, float(taus[i]), 1e-3)
        assert abs(loss_gpu - loss) <= 1e-2 * loss, i
    a, r = g.gsq_recon_error(lay, 0)
    ra, rr = oracle_mod.recon_error(st, X, Y, 0)
    assert abs(r - rr) <= 0.02 * rr
    # the state mostly agrees exactly (Lion sign ties may flip a few)
    agree = (lay.get(g.GSQ_DBG_LOGITS) == st.logits).mean()
    assert agree > 0.99
    lay.close()


def test_first_config_full_trajectory(g, oracle_mod):
    """Single 256x512 fp32 layer, 4 outlier channels x10, 2-bit, 20 steps."""
    cfg = synth.CONFIGS["c1_small_256x512"]
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    taus = synth.tau_schedule(cfg.tau0, cfg.tau1, cfg.steps)
    lay = g.gsq_init(W, X, 128, cfg.grid, seed=0)
    st = oracle_mod.init(cfg.grid, W, seed=0)
    Y = oracle_mod.reference_output(W, X)
    losses, ref = [], []
    for tau in taus:
        lay.step(float(tau), cfg.lr)
        losses.append(lay.last_loss())
        ref.append(oracle_mod.step(st, X, Y, float(tau), cfg.lr))
    assert np.all(np.abs(np.array(losses) - ref) <= 1e-2 * np.array(ref))
    a, r = g.gsq_recon_error(lay, 0)
    ra, rr = oracle_mod.recon_error(st, X, Y, 0)
    assert abs(r - rr) <= 0.02 * rr
    packed, h16, f32 = g.gsq_harden_pack(lay)
    lev_ref = oracle_mod.harden(cfg.grid, st.logits, st.i0)
    lev_gpu = oracle_mod.unpack(cfg.grid, packed.reshape(cfg.N, -1), cfg.K)
    assert (lev_gpu == lev_ref).mean() > 0.99
    lay.close()


@pytest.mark.parametrize("mode,shape", [(0, (256, 512, 256)), (1, (200, 384, 200)),
                                        (2, (136, 256, 72))])
def test_run_equals_step_loop_bit_exact(g, mode, shape):
    """gsq_run fuses each step's backward with the next step's soft weight;
    the state and losses must equal those of separate gsq_step calls bit for
    bit (same arithmetic, different kernel boundaries)."""
    N, K, T = shape
    cfg, W, X = make_case(mode, N, K, T)
    taus = synth.tau_schedule(1.0, 0.05, 12)
    a = gpu_layer(g, W, X, mode, seed=3)
    b = gpu_layer(g, W, X, mode, seed=3)
    la = []
    for tau in taus:
        a.step(float(tau), 1e-3)
        la.append(a.last_loss())
    b.run(taus[:5], 1e-3)
    b.run(taus[5:], 1e-3)
    hist = np.zeros(12)
    g._check(g.lib().gsq_loss_history(b.ctx, 0, 12, hist.ctypes.data), "hist")
    assert list(hist) == la
    for which in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES, g.GSQ_DBG_SMOM):
        assert np.array_equal(a.get(which), b.get(which))
    a.close(); b.close()


def test_checkpoint_resume_bit_exact(g):
    cfg, W, X = make_case(2, 136, 256, 72)
    taus = synth.tau_schedule(1.0, 0.1, 10)
    a = gpu_layer(g, W, X, 2, seed=4)
    for i in range(5):
        a.step(float(taus[i]), 1e-3)
    snap = g.gsq_export_state(a)
    for i in range(5, 10):
        a.step(float(taus[i]), 1e-3)
    b = gpu_layer(g, W, X, 2, seed=4)
    g.gsq_import_state(b, snap)
    assert g.gsq_get_step(b) == 5
    for i in range(5, 10):
        b.step(float(taus[i]), 1e-3)
    for which in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES, g.GSQ_DBG_SMOM):
        assert np.array_equal(a.get(which), b.get(which))
    assert a.last_loss() == b.last_loss()
    a.close(); b.close()


def test_deterministic_reruns(g):
    cfg, W, X = make_case(1, 200, 384, 200)
    outs = []
    for _ in range(2):
        lay = gpu_layer(g, W, X, 1, seed=9)
        for tau in synth.tau_schedule(1.0, 0.2, 4):
            lay.step(float(tau), 1e-3)
        outs.append((lay.last_loss(), lay.get(g.GSQ_DBG_LOGITS)))
        lay.close()
    assert outs[0][0] == outs[1][0]
    assert np.array_equal(outs[0][1], outs[1][1])


def test_bad_step_arguments(g):
    cfg, W, X = make_case(0, 128, 128, 64)
    lay = gpu_layer(g, W, X, 0)
    for args in [(0.0, 1e-3, 0.9, 0.99), (-1.0, 1e-3, 0.9, 0.99),
                 (1.0, -1.0, 0.9, 0.99), (1.0, 1e-3, 1.0, 0.99),
                 (float("nan"), 1e-3, 0.9, 0.99)]:
        with pytest.raises(g.GSQError) as e:
            g.gsq_step(lay, *args)
        assert e.value.status == g.GSQ_ERR_INVALID_ARG
    with pytest.raises(g.GSQError) as e:
        g.gsq_last_loss(lay)  # no step yet
    assert e.value.status == g.GSQ_ERR_STATE
    lay.close()


# ------------------------------------------- full-size row-slice parity

@pytest.mark.parametrize("name", ["c2_qproj_4096x4096", "c3_downproj_4096x14336",
                                  "c4_gateproj_14336x4096"])
def test_full_size_row_slices(g, oracle_mod, name):
    """Full layers in the benchmark's launch configuration; the oracle follows
    a slice of rows (the loss decomposes over rows and the noise is keyed by
    the global coordinate)."""
    import torch
    cfg = synth.CONFIGS[name]
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    lay = g.gsq_init(torch.from_numpy(W).cuda().to(torch.bfloat16),
                     torch.from_numpy(X).cuda().to(torch.bfloat16), 128, cfg.grid, seed=0)
    steps = 2
    taus = synth.tau_schedule(cfg.tau0, cfg.tau1, cfg.steps)[:steps]
    for tau in taus:
        lay.step(float(tau), cfg.lr)
    loss_gpu = lay.last_loss()
    logits = lay.get(g.GSQ_DBG_LOGITS)
    scales = lay.get(g.GSQ_DBG_SCALES)
    lay.close()
    rows = [0, 1, cfg.N // 2 + 3, cfg.N - 1]
    for r in rows:
        Wr = W[r:r + 1]
        st = oracle_mod.init(cfg.grid, Wr, seed=0, row0=r)
        Y = oracle_mod.reference_output(Wr, X)
        for tau in taus:
            oracle_mod.step(st, X, Y, float(tau), cfg.lr)
        agree = (logits[:, r] == st.logits[:, 0]).mean()
        assert agree > 0.995, (r, agree)
        assert np.allclose(scales[r], st.s[0], rtol=0, atol=3 * cfg.lr * steps)
    assert np.isfinite(loss_gpu) and loss_gpu > 0

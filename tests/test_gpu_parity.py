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


def test_noise_log2_every_uniform(g):
    """The logarithm inside every step's noise, log2(u) for each of the 2^23
    uniforms u = (m + 1/2) 2^-23, against fp64: relative error within 1.5e-7
    everywhere, in particular next to u = 1 where log2(u) is tiny and a
    logarithm with an absolute error (the hardware lg2) is off by up to 86%.
    The Gumbel noise -ln(-ln u) takes log2 of -log2(u), so its absolute error
    is this relative error over ln 2."""
    cfg, W, X = make_case(0, 8, 128, 8)
    lay = gpu_layer(g, W, X, 0)
    n = 1 << 23
    got = np.concatenate([lay.noise_log2(m0, 1 << 21) for m0 in range(0, n, 1 << 21)])
    u = (np.arange(n, dtype=np.float64) + 0.5) * 2.0 ** -23
    ref = np.log2(u)
    rel = np.abs(got.astype(np.float64) - ref) / np.abs(ref)
    assert rel.max() <= 1.5e-7, (rel.max(), int(rel.argmax()))
    assert np.all(got < 0)
    # the last uniform below 1: log2(1 - 2^-24) = -8.6e-8, relatively exact
    assert abs(got[-1] / ref[-1] - 1) <= 1.5e-7
    with pytest.raises(g.GSQError):
        lay.noise_log2(n - 10, 11)
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


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("state16", [False, True])
def test_row_shards_equal_whole_layer(g, oracle_mod, mode, state16):
    """gsq_init_rows: the shards [0, 256) and [256, 456) of a layer, each
    keyed by its global row offset, follow the whole layer's trajectory bit
    for bit (every output row of the GEMMs is the same dot products in the
    same order whatever the row tile), and their losses add up to the
    layer's; the shard's noise equals the oracle's at the global coordinates."""
    import torch
    N, K, T = 456, 640, 200
    cfg, W, X = make_case(mode, N, K, T)
    Xd = torch.from_numpy(X).cuda()
    full = g.gsq_init(torch.from_numpy(W).cuda(), Xd, 128, mode, seed=31, state_bf16=state16)
    bands = [(0, 256), (256, N - 256)]
    shards = [g.gsq_init(torch.from_numpy(np.ascontiguousarray(W[r0:r0 + n])).cuda(), Xd, 128,
                         mode, seed=31, state_bf16=state16, row0=r0) for r0, n in bands]
    taus = np.array([1.0, 0.6, 0.3, 0.15], np.float32)
    full.run(taus, 1e-3)
    for sh in shards:
        sh.run(taus, 1e-3)
    for which in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES, g.GSQ_DBG_SMOM,
                  g.GSQ_DBG_WHAT, g.GSQ_DBG_DW):
        whole = full.get(which)
        axis = 1 if which in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM) else 0
        parts = np.concatenate([sh.get(which) for sh in shards], axis=axis)
        assert np.array_equal(parts.view(np.uint8), whole.view(np.uint8)), which
    assert sum(sh.last_loss() for sh in shards) == pytest.approx(full.last_loss(), rel=1e-12)
    # the soft weight of the second shard at step 4 from the oracle's noise at
    # the global coordinates (the oracle state takes row0 likewise)
    st = oracle_mod.State(mode, N - 256, K, 128, shards[1].get(g.GSQ_DBG_LOGITS).astype(np.float32),
                          shards[1].get(g.GSQ_DBG_MOM).astype(np.float32),
                          shards[1].get(g.GSQ_DBG_SCALES), shards[1].get(g.GSQ_DBG_SMOM),
                          shards[1].get(g.GSQ_DBG_I0), row0=256, seed=31, t=4)
    if not state16:
        shards[1].soft_weight(0.2)
        _, _, w, _ = oracle_mod.soft_weight(st, 0.2)
        w_gpu = shards[1].get(g.GSQ_DBG_WSOFT32).astype(np.float64)
        floor = np.repeat(st.s, 128, 1) * LEVEL_MAX[mode]
        assert np.all(np.abs(w_gpu - w) <= 1e-5 * (np.abs(w) + floor))
    full.close()
    for sh in shards:
        sh.close()


def test_row_offset_rejected_on_host(g):
    cfg, W, X = make_case(0, 8, 128, 8)
    import ctypes as C
    ctx = C.c_void_p()
    rc = g.lib().gsq_init_rows(C.byref(ctx), W.ctypes.data, g.GSQ_F32, X.ctypes.data, g.GSQ_F32,
                               8, 128, 8, 128, 0, None, 0, -1, 0, None)
    assert rc == g.GSQ_ERR_INVALID_ARG and not ctx.value
    rc = g.lib().gsq_init_rows(C.byref(ctx), W.ctypes.data, g.GSQ_F32, X.ctypes.data, g.GSQ_F32,
                               8, 128, 8, 128, 0, None, 0, 0, 2, None)
    assert rc == g.GSQ_ERR_INVALID_ARG and not ctx.value


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


@pytest.mark.parametrize("shape", [(401, 552, 200), (300, 1000, 4160), (4096, 3968, 768)])
def test_subtracting_gemm_entry(g, oracle_mod, shape):
    """C -= A B^T in place (the epilogue of GPTQ's tensor-core updates): ragged
    tiles, a deep K, and the q_proj column-block shape; C's old values and the
    product of the library's GEMM entry both come back exactly as fp32 sums."""
    import torch
    M, N, Kc = shape
    rng = np.random.default_rng(M + 7 * N)
    A = synth.bf16_values(rng.normal(size=(M, Kc)).astype(np.float32))
    B = synth.bf16_values(rng.normal(size=(N, Kc)).astype(np.float32))
    C0 = rng.normal(0, 10, size=(M, N)).astype(np.float32)
    C = torch.from_numpy(C0).cuda()
    Ad = torch.from_numpy(A).cuda().to(torch.bfloat16)
    Bd = torch.from_numpy(B).cuda().to(torch.bfloat16)
    g.gsq_gemm_bf16_abt_sub(Ad, Bd, C)
    ref = C0.astype(np.float64) - oracle_mod.gemm_abt(A, B)
    got = C.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref)) < 1e-4 * np.sqrt(Kc)
    # the same product from the storing entry, subtracted in fp32 on the host
    P = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    g.gsq_gemm_bf16_abt(Ad, Bd, P)
    assert np.array_equal(got.astype(np.float32), C0 - P.cpu().numpy())


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


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_step_next_loop_equals_run(g, mode):
    """A caller-driven loop of gsq_step_next(tau_t, tau_{t+1}) (the backward
    forms the next soft weight, the next call skips it) equals gsq_run bit
    for bit; a call at another temperature than the one announced recomputes
    the soft weight, as gsq_step would."""
    cfg, W, X = make_case(mode, 200, 384, 136)
    taus = synth.tau_schedule(1.0, 0.05, 9)
    a = gpu_layer(g, W, X, mode, seed=6)
    b = gpu_layer(g, W, X, mode, seed=6)
    c = gpu_layer(g, W, X, mode, seed=6)
    for i, tau in enumerate(taus):
        nxt = float(taus[i + 1]) if i + 1 < len(taus) else None
        a.step(float(tau), 1e-3, tau_next=nxt)
        # c announces a wrong next temperature every time
        c.step(float(tau), 1e-3, tau_next=0.77)
    b.run(taus, 1e-3)
    assert a.last_loss() == b.last_loss() == c.last_loss()
    for which in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES, g.GSQ_DBG_SMOM):
        assert np.array_equal(a.get(which), b.get(which))
        assert np.array_equal(c.get(which), b.get(which))
    st = g.lib().gsq_step_next(a.ctx, 0.5, 0.0, 1e-3, 0.9, 0.99)
    assert st == g.GSQ_ERR_INVALID_ARG
    a.close(); b.close(); c.close()


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

def _row_state(oracle_mod, mode, arrays, r, t):
    """The oracle state of row r from the GPU's buffers (identical values)."""
    logits, mom, s, ms, i0 = arrays
    return oracle_mod.State(mode, 1, logits.shape[2], 128,
                            np.ascontiguousarray(logits[:, r:r + 1], np.float32),
                            np.ascontiguousarray(mom[:, r:r + 1], np.float32),
                            np.ascontiguousarray(s[r:r + 1]), np.ascontiguousarray(ms[r:r + 1]),
                            np.ascontiguousarray(i0[r:r + 1]), row0=r, seed=0, t=t)


@pytest.mark.parametrize("name", ["c2_qproj_4096x4096", "c3_downproj_4096x14336",
                                  "c4_gateproj_14336x4096"])
def test_full_size_fused_run_against_oracle_rows(g, oracle_mod, name):
    """Full layers in the benchmark's launch configuration (gsq_run: every
    backward but a run's last also forms the next step's soft weight).

    1. gsq_run over 5 steps equals a loop of gsq_step bit for bit, all
       buffers of the whole layer (the fused path computes what the unfused
       one does, at full size and in every GEMM wave);
    2. on sampled rows (first, last, both sides of a 256-row tile edge, the
       last row tile) the state after 5 fused steps follows the oracle's own
       5-step trajectory of those rows (Lion near-ties aside);
    3. one more step from the GPU's exact state, row by row against the
       oracle: the soft weight (fp32 contract, then bf16 rounding), each
       row's loss from the GPU's output gradient at 1e-2, the dW rows at
       1e-2, and -- given the GPU's own dW -- the fused backward: logits and
       scales bit-identical wherever Lion's blend is not a near-tie, momenta
       within their bound.
    The loss decomposes over rows and the noise is keyed by the global
    coordinate, so each row is an independent oracle problem."""
    import torch
    cfg = synth.CONFIGS[name]
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    Wd = torch.from_numpy(W).cuda().to(torch.bfloat16)
    Xd = torch.from_numpy(X).cuda().to(torch.bfloat16)
    taus = np.array([1.0, 0.6, 0.35, 0.2, 0.1, 0.05], np.float32)
    lr = cfg.lr
    N, K, T, mode = cfg.N, cfg.K, cfg.T, cfg.grid
    lay = g.gsq_init(Wd, Xd, 128, mode, seed=0)
    lay.run(taus[:5], lr)
    bufs = (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES, g.GSQ_DBG_SMOM, g.GSQ_DBG_I0)
    s5 = [lay.get(b) for b in bufs]
    # 1. the same five steps one gsq_step at a time
    ref = g.gsq_init(Wd, Xd, 128, mode, seed=0)
    for tau in taus[:5]:
        ref.step(float(tau), lr)
    for b, a in zip(bufs, s5):
        assert np.array_equal(ref.get(b).view(np.uint8), a.view(np.uint8)), b
    assert ref.last_loss() == lay.last_loss()
    ref.close()
    # step 5 on the GPU
    lay.run(taus[5:6], lr)
    w5 = bits_to_f32(lay.get(g.GSQ_DBG_WHAT))
    dW5 = lay.get(g.GSQ_DBG_DW)
    dyt = lay.get(g.GSQ_DBG_DYT)[:, :T]
    s6 = [lay.get(b) for b in bufs[:4]]
    loss5 = lay.last_loss()
    lay.close()
    E = bits_to_f32(dyt).astype(np.float64) / 2.0
    row_loss_gpu = (E * E).sum(1)
    assert row_loss_gpu.sum() == pytest.approx(loss5, rel=1e-2)
    rows = sorted({0, 1, 255, 256, N // 2 + 3, N - 257, N - 200, N - 1})
    agree = []
    for r in rows:
        Wr = np.ascontiguousarray(W[r:r + 1])
        Y = oracle_mod.reference_output(Wr, X)
        # 2. the oracle's own trajectory of this row
        tr = oracle_mod.init(mode, Wr, seed=0, row0=r)
        for tau in taus[:5]:
            oracle_mod.step(tr, X, Y, float(tau), lr)
        agree.append((tr.logits[:, 0] == s5[0][:, r]).mean())
        # 3. step 5 from the GPU's state of the row
        st = _row_state(oracle_mod, mode, s5, r, 5)
        _, v, w, wb = oracle_mod.soft_weight(st, float(taus[5]))
        floor = np.repeat(st.s, 128, 1) * LEVEL_MAX[mode]
        half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(w5[r:r + 1]), 1e-30))) - 8)
        assert np.all(np.abs(w5[r:r + 1] - w) <= 1e-5 * (np.abs(w) + floor) + half_ulp), r
        assert (w5[r:r + 1] != wb).mean() < 1e-2, r
        loss_r, dY = oracle_mod.forward(X, wb, Y)
        assert row_loss_gpu[r] == pytest.approx(loss_r, rel=1e-2), r
        dW_ref = oracle_mod.weight_grad(dY, X)
        assert np.linalg.norm(dW5[r] - dW_ref[0]) <= 1e-2 * np.linalg.norm(dW_ref[0]), r
        # the fused backward given the GPU's dW of the row
        dWr = np.ascontiguousarray(dW5[r:r + 1])
        m_before = st.mom.copy()
        dl_ref, ds_ref = oracle_mod.backward_lion(st, dWr, float(taus[5]), lr)
        a = np.abs(np.repeat(s5[2][r:r + 1], 128, 1) * dWr) / float(taus[5])
        c = 0.9 * m_before.astype(np.float64) + 0.1 * dl_ref
        clear = np.abs(c) > 0.1 * 1e-5 * (np.abs(dl_ref) + a[None]) + 1e-12
        # at tau = 0.05 many probabilities are saturated, so |dl| << |a| / tau
        # and the tolerance floor leaves a few percent of the blends unclear
        assert clear.mean() > 0.9, (r, clear.mean())
        assert np.array_equal(s6[0][:, r:r + 1][clear], st.logits[clear]), r
        mtol = 0.01 * 1e-5 * (np.abs(dl_ref) + a[None]) + 2.0 ** -22 * np.abs(st.mom)
        assert np.all(np.abs(s6[1][:, r:r + 1] - st.mom) <= mtol), r
        bound = np.abs(dWr.astype(np.float64) * v).reshape(1, -1, 128).sum(-1)
        sclear = np.abs(0.9 * s5[3][r:r + 1].astype(np.float64) + 0.1 * ds_ref) > 1e-6 * bound
        assert sclear.mean() > 0.9, r
        assert np.array_equal(s6[2][r:r + 1][sclear], st.s[sclear]), r
    assert min(agree) > 0.99, agree



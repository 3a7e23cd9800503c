"""Parity of GSQ on GGUF K-Quant formats (gsq_kq_*) with the oracle
(oracle/kquant.py), through the C ABI.  Needs a B200.

Tolerances as for the GSQ grids: the start (blocks, sub-block parameters,
codes, logits), the export of an unmoved state and the dequantisation
bit-exact (every integer decision taken in fp32 without contraction on both
sides); soft weight |dw| <= 1e-5 (|w| + |a| c_max + |b|); logit gradients
|d dl| <= 1e-5 (|dl| + |a dw| c_span / tau), sub-block gradients
<= 1e-5 sum |dw| (|v| + 1) given identical dW; Lion identical away from
near-ties; per-step loss 1e-2 and the exported blocks' reconstruction error
within 2% over a trajectory."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

pytestmark = pytest.mark.gpu
FMTS = [0, 1]


@pytest.fixture(scope="module")
def g():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    return gsq


@pytest.fixture(scope="module")
def KQ(oracle_mod):
    from oracle import kquant
    return kquant


def case(N, K, T, number=93):
    cfg = synth.small_config(N, K, T, 0, number=number, outlier_cols=4, outlier_scale=10.0)
    return synth.make_weight(cfg), synth.make_calib(cfg)


def layer(g, W, X, fmt, seed=0, start=None):
    import torch
    return g.gsq_kq_init(torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda(), fmt,
                         start_blocks=start, seed=seed)


@pytest.mark.parametrize("fmt", FMTS)
def test_start_and_state_bit_exact(g, KQ, fmt):
    N, K, T = 64, 768, 64
    W, X = case(N, K, T)
    lay = layer(g, W, X, fmt, seed=1)
    blk = KQ.start(fmt, W)
    assert np.array_equal(lay.start_blocks(), blk.reshape(-1))
    st = KQ.init_state(fmt, blk, N, K, seed=1)
    assert np.array_equal(lay.get(g.GSQ_KQ_DBG_A), st.a)
    assert np.array_equal(lay.get(g.GSQ_KQ_DBG_B), st.b)
    assert np.array_equal(lay.get(g.GSQ_KQ_DBG_Q0).astype(np.int64), st.q0)
    assert np.array_equal(lay.get(g.GSQ_KQ_DBG_LOGITS), st.logits)
    lay.close()


@pytest.mark.parametrize("fmt", FMTS)
def test_given_start_and_unmoved_export(g, KQ, fmt):
    """Caller-given blocks with every sub-block code range reached: the state
    decodes them exactly and exporting before any step gives them back."""
    N, K, T = 16, 512, 64
    W, X = case(N, K, T)
    rng = np.random.default_rng(3 + fmt)
    nb = N * K // 256
    q = rng.integers(KQ.QMIN[fmt], KQ.QMAX[fmt] + 1, (nb, 256))
    if fmt == 0:
        sc, m = rng.integers(0, 16, (nb, 16)), rng.integers(0, 16, (nb, 16))
        sc[:, 0], m[:, 1] = 15, 15
        dmin = rng.uniform(1e-4, 2e-3, nb)
    else:
        sc, m = np.clip(rng.integers(-32, 32, (nb, 16)), -31, 31), np.zeros((nb, 16), np.int64)
        sc[:, 0] = 31
        dmin = np.zeros(nb)
    blk = KQ.encode(fmt, q, sc, m, rng.uniform(1e-4, 2e-3, nb), dmin)
    lay = layer(g, W, X, fmt, start=blk.reshape(-1))
    st = KQ.init_state(fmt, blk, N, K)
    assert np.array_equal(lay.get(g.GSQ_KQ_DBG_A), st.a)
    assert np.array_equal(lay.export(), blk.reshape(-1))
    assert np.array_equal(KQ.export(st), blk)
    lay.close()


@pytest.mark.parametrize("fmt", FMTS)
def test_dequant_bit_exact(g, KQ, fmt):
    import torch
    import gguf
    from gguf import GGMLQuantizationType as G
    W, _ = case(32, 1024, 8)
    blk = KQ.start(fmt, W)
    out = g.gsq_kq_dequant(fmt, blk.reshape(-1), 32, 1024)
    ref32 = gguf.quants.dequantize(blk, G.Q2_K if fmt == 0 else G.Q3_K).reshape(32, 1024)
    ref = torch.from_numpy(ref32).to(torch.bfloat16)
    assert torch.equal(out.cpu(), ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_soft_weight(g, KQ, fmt):
    N, K, T = 64, 512, 64
    W, X = case(N, K, T)
    lay = layer(g, W, X, fmt, seed=5)
    st = KQ.init_state(fmt, KQ.start(fmt, W), N, K, seed=5)
    lg = synth.random_logits(st.logits.shape, 4, ties=False)
    st.logits[:] = lg
    lay.set(g.GSQ_KQ_DBG_LOGITS, lg)
    for tau in (1.0, 0.1):
        lay.soft_weight(tau)
        w = lay.get(g.GSQ_KQ_DBG_WSOFT32)
        _, _, wr, _ = KQ.soft_weight(st, tau)
        A = np.abs(np.repeat(st.a, 16, 1)).astype(np.float64)
        B = np.abs(np.repeat(st.b, 16, 1)).astype(np.float64)
        assert np.all(np.abs(w - wr) <= 1e-5 * (np.abs(wr) + 4 * A + B)), tau
    lay.close()


@pytest.mark.parametrize("fmt", FMTS)
def test_backward_lion_given_identical_dw(g, KQ, fmt):
    N, K, T = 64, 512, 64
    W, X = case(N, K, T)
    lay = layer(g, W, X, fmt, seed=7)
    st = KQ.init_state(fmt, KQ.start(fmt, W), N, K, seed=7)
    lg = synth.random_logits(st.logits.shape, 8, ties=False)
    mom = synth.random_grad(st.logits.shape, 9, scale=1e-3)
    st.logits[:], st.mom[:] = lg, mom
    lay.set(g.GSQ_KQ_DBG_LOGITS, lg)
    lay.set(g.GSQ_KQ_DBG_MOM, mom)
    dW = synth.random_grad((N, K), 10, scale=1.0)
    lay.set(g.GSQ_KQ_DBG_DW, dW)
    tau, lr = 0.4, 1e-3
    y, u, _, _ = KQ.soft_weight(st, tau)
    dl_ref, da_ref, db_ref = KQ.gradients(st, y, u, dW, tau)
    a0 = st.a.copy()
    lay.backward(tau, lr)
    A = np.abs(np.repeat(a0, 16, 1)).astype(np.float64)
    span = 7.0 if fmt else 3.0
    tol = 1e-5 * (np.abs(dl_ref) + (A * np.abs(dW) * span / tau)[None])
    assert np.all(np.abs(lay.get(g.GSQ_KQ_DBG_DL) - dl_ref) <= tol)
    bound = (np.abs(dW.astype(np.float64)) * (np.abs(u) + 1)).reshape(N, -1, 16).sum(-1)
    assert np.all(np.abs(lay.get(g.GSQ_KQ_DBG_DA) - da_ref) <= 1e-5 * bound)
    if fmt == 0:
        assert np.all(np.abs(lay.get(g.GSQ_KQ_DBG_DB) - db_ref) <= 1e-5 * bound)
    # Lion on the logits and a: identical wherever the blend's sign is clear
    KQ._lion(st.logits, st.mom, dl_ref, lr, 0.9, 0.99)
    KQ._lion(st.a, st.ma, da_ref, lr, 0.9, 0.99)
    c = 0.9 * mom.astype(np.float64) + 0.1 * dl_ref
    clear = np.abs(c) > 0.1 * tol + 1e-12
    assert clear.mean() > 0.99
    assert np.array_equal(lay.get(g.GSQ_KQ_DBG_LOGITS)[clear], st.logits[clear])
    sclear = np.abs(0.1 * da_ref) > 1e-5 * bound * 0.1
    assert np.array_equal(lay.get(g.GSQ_KQ_DBG_A)[sclear], st.a[sclear])
    lay.close()


@pytest.mark.parametrize("fmt", FMTS)
def test_trajectory(g, KQ, fmt):
    N, K, T = 128, 512, 128
    W, X = case(N, K, T)
    lay = layer(g, W, X, fmt, seed=0)
    st = KQ.init_state(fmt, KQ.start(fmt, W), N, K, seed=0)
    Y = KQ.reference_output(W, X)
    taus = synth.tau_schedule(1.0, 0.05, 20)
    for i, tau in enumerate(taus):
        lay.step(float(tau), 1e-4)
        loss = KQ.step(st, X, Y, float(tau), 1e-4)
        assert abs(lay.last_loss() - loss) <= 1e-2 * loss, i
    e_gpu = lay.recon_error(0)[1]
    e_ref = KQ.recon_error(fmt, KQ.export(st), X, Y, N, K)[1]
    assert abs(e_gpu - e_ref) <= 0.02 * e_ref
    e_start = lay.recon_error(1)[1]
    assert abs(e_start - KQ.recon_error(fmt, KQ.start(fmt, W), X, Y, N, K)[1]) <= 1e-2 * e_start
    ex, er = lay.export(), KQ.export(st).reshape(-1)
    assert (ex == er).mean() > 0.98
    lay.close()


def test_full_size_q_proj_row_slices(g, KQ):
    """The q_proj-shaped layer (4096 x 4096, T 4096) in Q2_K, the bench's
    launch configuration; the oracle follows a few rows."""
    import torch
    cfg = synth.CONFIGS["c2_qproj_4096x4096"]
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    lay = g.gsq_kq_init(torch.from_numpy(W).cuda().to(torch.bfloat16),
                        torch.from_numpy(X).cuda().to(torch.bfloat16), 0, seed=0)
    taus = synth.tau_schedule(1.0, 0.05, 300)[:2]
    lay.run(taus, 1e-4)
    logits = lay.get(g.GSQ_KQ_DBG_LOGITS)
    a = lay.get(g.GSQ_KQ_DBG_A)
    start = lay.start_blocks().reshape(cfg.N, -1)
    lay.close()
    for r in (0, 1777, cfg.N - 1):
        blk = KQ.start(0, W[r:r + 1])
        assert np.array_equal(start[r], blk.reshape(-1))
        st = KQ.init_state(0, blk, 1, cfg.K, seed=0, row0=r)
        Y = KQ.reference_output(W[r:r + 1], X)
        for tau in taus:
            KQ.step(st, X, Y, float(tau), 1e-4)
        assert (logits[:, r] == st.logits[:, 0]).mean() > 0.995, r
        assert np.allclose(a[r], st.a[0], rtol=0, atol=3e-4)


@pytest.mark.parametrize("fmt", FMTS)
def test_run_equals_step_loop(g, fmt):
    """gsq_kq_run forms each next step's soft weight inside the backward;
    a loop of gsq_kq_step forms it in a soft-weight pass of its own.  The two
    must agree bit for bit, also after the debug entry points and the
    reconstruction error (which reuse the soft-weight buffer) intervene."""
    N, K, T = 136, 512, 120
    W, X = case(N, K, T, number=97)
    taus = synth.tau_schedule(1.0, 0.05, 12)
    a, b = layer(g, W, X, fmt, seed=4), layer(g, W, X, fmt, seed=4)
    for tau in taus[:6]:
        a.step(float(tau), 1e-4)
    b.run(taus[:6], 1e-4)
    b.recon_error(1)
    a.run(taus[6:], 1e-4)
    for tau in taus[6:]:
        b.step(float(tau), 1e-4)
    for which in (g.GSQ_KQ_DBG_LOGITS, g.GSQ_KQ_DBG_MOM, g.GSQ_KQ_DBG_A, g.GSQ_KQ_DBG_MA,
                  g.GSQ_KQ_DBG_B, g.GSQ_KQ_DBG_MB):
        assert np.array_equal(a.get(which), b.get(which)), which
    assert a.last_loss() == b.last_loss()
    assert np.array_equal(a.export(), b.export())
    a.close()
    b.close()

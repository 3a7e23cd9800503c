"""Parity of the attention V/O block stage (value and output quantized
jointly, attention probabilities fixed from the frozen query/key weights)
with the oracle, through the C ABI.  Needs a B200."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

pytestmark = pytest.mark.gpu

DIMS = dict(nseq=2, S=128, nh=4, nkv=2, d=128)


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


def case(seed=0, nseq=2, S=128, nh=4, nkv=2, d=128):
    Xa, Wq, Wk, Wv, Wo = synth.make_attn_stage(nseq, S, nh, nkv, d, seed=seed)
    return Xa, Wq, Wk, Wv, Wo


def fp_target(oracle_mod, Xa, Wq, Wk, Wv, Wo, dims):
    """Full-precision attention output (exact fp64) as the stage's target."""
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **dims, round_bf16=False)
    nseq, S, nh, nkv, d = dims["nseq"], dims["S"], dims["nh"], dims["nkv"], dims["d"]
    X = Xa.astype(np.float64)
    V = (X @ Wv.T.astype(np.float64)).reshape(nseq, S, nkv, d)
    o = np.zeros((nseq * S, nh * d))
    for s in range(nseq):
        for h in range(nh):
            o[s * S:(s + 1) * S, h * d:(h + 1) * d] = P[s, h].astype(np.float64) @ V[s, :, h // (nh // nkv)]
    return (o @ Wo.T.astype(np.float64)).astype(np.float32)


def make(g, Xa, R, Wq, Wk, Wv, Wo, mode=0, seed=0, dims=DIMS):
    return g.gsq_attn_init(Xa, R, Wq, Wk, Wv, Wo, dims["nseq"], dims["S"], dims["nh"],
                           dims["nkv"], dims["d"], grid_mode=mode, seed=seed)


def test_probabilities(g, oracle_mod):
    Xa, Wq, Wk, Wv, Wo = case()
    R = fp_target(oracle_mod, Xa, Wq, Wk, Wv, Wo, DIMS)
    a = make(g, Xa, R, Wq, Wk, Wv, Wo)
    P = bits_to_f32(a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_P)).astype(np.float64)
    ref = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS).astype(np.float64)
    S = DIMS["S"]
    iu = np.triu_indices(S, 1)
    assert np.all(P[..., iu[0], iu[1]] == 0)
    # both sides round the probabilities to bf16 (8 significant bits); the
    # operands Q, K are bf16 GEMM results on both sides, and fp32 against
    # fp64 accumulation may put one of them a unit apart, which moves a
    # probability by about one more unit: at most two bf16 units (2^-6
    # relative covers two units anywhere in a binade)
    assert np.all(np.abs(P - ref) <= 2.0 ** -6 * ref + 2.0 ** -16)
    assert np.abs(P - ref).mean() < 2e-6
    # a row of bf16 probabilities sums to 1 within its accumulated rounding
    assert np.allclose(P.sum(-1), 1.0, atol=2.0 ** -8)
    # the transposed copy holds the same values
    PT = a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_PT).reshape(DIMS["nseq"], DIMS["nkv"], S,
                                                             DIMS["nh"] // DIMS["nkv"], S)
    Pb = a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_P)
    grp = DIMS["nh"] // DIMS["nkv"]
    for h in range(DIMS["nh"]):
        assert np.array_equal(PT[:, h // grp, :, h % grp, :], np.swapaxes(Pb[:, h], 1, 2))
    a.close()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_one_step(g, oracle_mod, mode):
    Xa, Wq, Wk, Wv, Wo = case(seed=1)
    R = fp_target(oracle_mod, Xa, Wq, Wk, Wv, Wo, DIMS)
    a = make(g, Xa, R, Wq, Wk, Wv, Wo, mode=mode, seed=5)
    at = oracle_mod.attn_init(mode, Wv, Wo, seed=5)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS)
    for i, st in enumerate(at.weights()):
        assert np.array_equal(a.get(i, g.GSQ_DBG_SCALES), st.s)
        assert np.array_equal(a.get(i, g.GSQ_DBG_LOGITS), st.logits)
    tau, lr = 0.6, 1e-3
    a.step(tau, lr)
    dims = tuple(DIMS.values())
    loss, d = oracle_mod.attn_step(at, Xa, P, R.astype(np.float64), dims, tau, lr, dumps=True)
    assert abs(a.last_loss() - loss) <= 1e-2 * loss
    for i in range(2):
        wb = bits_to_f32(a.get(i, g.GSQ_DBG_WHAT))
        assert (wb != d["w"][i]).mean() < 1e-3
        dW = a.get(i, g.GSQ_DBG_DW)
        assert np.linalg.norm(dW - d["dW"][i]) / np.linalg.norm(d["dW"][i]) < 2e-2
        agree = (a.get(i, g.GSQ_DBG_LOGITS) == at.weights()[i].logits).mean()
        assert agree > 0.99
    a.close()


DIMS_CAUSAL = dict(nseq=2, S=512, nh=4, nkv=2, d=128)


def test_one_step_causal_tiles(g, oracle_mod):
    """S a multiple of 256: the batched products skip the zero half of P."""
    dims = DIMS_CAUSAL
    Xa, Wq, Wk, Wv, Wo = case(seed=7, **dims)
    R = fp_target(oracle_mod, Xa, Wq, Wk, Wv, Wo, dims)
    a = make(g, Xa, R, Wq, Wk, Wv, Wo, mode=0, seed=9, dims=dims)
    at = oracle_mod.attn_init(0, Wv, Wo, seed=9)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **dims)
    tau, lr = 0.7, 1e-3
    a.step(tau, lr)
    loss, d = oracle_mod.attn_step(at, Xa, P, R.astype(np.float64), tuple(dims.values()),
                                   tau, lr, dumps=True)
    assert abs(a.last_loss() - loss) <= 1e-2 * loss
    for i in range(2):
        dW = a.get(i, g.GSQ_DBG_DW)
        assert np.linalg.norm(dW - d["dW"][i]) / np.linalg.norm(d["dW"][i]) < 2e-2
        assert (a.get(i, g.GSQ_DBG_LOGITS) == at.weights()[i].logits).mean() > 0.99
    a.close()


def test_trajectory(g, oracle_mod):
    Xa, Wq, Wk, Wv, Wo = case(seed=2)
    R = fp_target(oracle_mod, Xa, Wq, Wk, Wv, Wo, DIMS)
    a = make(g, Xa, R, Wq, Wk, Wv, Wo, mode=0, seed=0)
    at = oracle_mod.attn_init(0, Wv, Wo, seed=0)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS)
    dims = tuple(DIMS.values())
    R64 = R.astype(np.float64)
    r0 = oracle_mod.attn_recon_error(at, Xa, P, R64, dims)[1]
    for tau in synth.tau_schedule(1.0, 0.05, 12):
        a.step(float(tau), 2e-3)
        loss = oracle_mod.attn_step(at, Xa, P, R64, dims, float(tau), 2e-3)
        assert abs(a.last_loss() - loss) <= 1e-2 * loss
    _, r = a.recon_error(g.GSQ_RECON_HARD)
    _, rr = oracle_mod.attn_recon_error(at, Xa, P, R64, dims)
    assert abs(r - rr) <= 0.02 * rr
    assert rr < r0
    for i in range(2):
        packed, _, _ = a.harden_pack(i)
        st = at.weights()[i]
        lev = oracle_mod.unpack(0, packed.reshape(st.N, -1), st.K)
        assert (lev == oracle_mod.harden(0, st.logits, st.i0)).mean() > 0.99
    a.close()


def test_run_equals_step_loop_bit_exact(g, oracle_mod):
    Xa, Wq, Wk, Wv, Wo = case(seed=3)
    R = fp_target(oracle_mod, Xa, Wq, Wk, Wv, Wo, DIMS)
    taus = synth.tau_schedule(1.0, 0.1, 6)
    a = make(g, Xa, R, Wq, Wk, Wv, Wo, seed=4)
    b = make(g, Xa, R, Wq, Wk, Wv, Wo, seed=4)
    for tau in taus:
        a.step(float(tau), 1e-3)
    b.run(taus, 1e-3)
    assert a.last_loss() == b.last_loss()
    for i in range(2):
        for buf in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES):
            assert np.array_equal(a.get(i, buf), b.get(i, buf))
    a.close(); b.close()


def test_full_70b_shape(g, oracle_mod):
    """The 70B attention shape (64 query / 8 value heads of 128, 8 x 2048
    tokens) in the bench's launch configuration: sampled probability rows
    against the oracle; after one step, sampled entries of V, of the
    attention outputs o = P V and of the value gradient dV = sum P^T do
    recomputed on the host from the step's own bf16 operands; a short run
    with finite losses."""
    import torch
    cfg = synth.ATTN_STAGE["c5_70b_attn"]
    dims = dict(nseq=cfg["nseq"], S=cfg["S"], nh=cfg["nh"], nkv=cfg["nkv"], d=cfg["d"])
    nseq, S, nh, nkv, d = (dims[k] for k in ("nseq", "S", "nh", "nkv", "d"))
    grp = nh // nkv
    Xa, Wq, Wk, Wv, Wo = synth.make_attn_stage(**dims)
    T, H = Xa.shape
    R = synth.random_target(T, H, 0.05)
    dev = lambda x: torch.from_numpy(x).cuda().to(torch.bfloat16)
    a = g.gsq_attn_init(dev(Xa), torch.from_numpy(R).cuda(), dev(Wq), dev(Wk), dev(Wv),
                        dev(Wo), nseq, S, nh, nkv, d, grid_mode=cfg["grid"], seed=0)
    P = a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_P)
    for s, h, q in [(0, 0, 5), (3, 17, 1000), (7, 63, 2047)]:
        row = bits_to_f32(P[s, h, q]).astype(np.float64)
        ref = oracle_mod.attn_prob_row(Xa, Wq, Wk, nseq, S, nh, nkv, s, h, q).astype(np.float64)
        assert np.all(row[q + 1:] == 0)
        assert np.all(np.abs(row - ref) <= 2.0 ** -6 * ref + 2.0 ** -16), (s, h, q)
        assert abs(row.sum() - 1.0) < 2.0 ** -8
    s_chk = 5
    Ps = bits_to_f32(P[s_chk]).astype(np.float64)  # nh x S x S
    del P

    def prefix_loss_vs_oracle(n=64):
        """The step's loss over the first n tokens of sequence s_chk from the
        GPU's output gradient, against the oracle's V/O forward of that prefix
        with the GPU's probabilities and soft weights of the step (causal: the
        prefix's outputs need no later token)."""
        dpt = bits_to_f32(a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_DPT)).astype(np.float64)
        gpu_tok = ((dpt / 2.0) ** 2).sum(0)
        assert gpu_tok.sum() == pytest.approx(a.last_loss(), rel=1e-2)
        lo = s_chk * S
        Wv_h = bits_to_f32(a.get(0, g.GSQ_DBG_WHAT))
        Wo_h = bits_to_f32(a.get(1, g.GSQ_DBG_WHAT))
        Pp = np.ascontiguousarray(Ps[None, :, :n, :n], np.float32)
        ref = oracle_mod.attn_vo_forward_backward(Xa[lo:lo + n], Pp, R[lo:lo + n], Wv_h, Wo_h,
                                                  1, n, nh, nkv, d)[0]
        assert gpu_tok[lo:lo + n].sum() == pytest.approx(ref, rel=1e-2)

    a.step(1.0, 1e-3)
    prefix_loss_vs_oracle()
    rows = slice(s_chk * S, (s_chk + 1) * S)
    VT = bits_to_f32(a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_VT)).astype(np.float64)  # Hk x T
    Wv_hat = bits_to_f32(a.get(0, g.GSQ_DBG_WHAT)).astype(np.float64)
    # V = bf16(Xa Wv^T): sampled rows within one bf16 rounding
    for j in (0, 517, nkv * d - 1):
        ref = Xa[rows].astype(np.float64) @ Wv_hat[j]
        mag = np.abs(Xa[rows].astype(np.float64)) @ np.abs(Wv_hat[j])
        assert np.all(np.abs(VT[j, rows] - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * mag)
    # o = P V for sampled (head, query) rows of one sequence
    O = bits_to_f32(a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_O)).astype(np.float64)  # T x H
    for h, q in [(0, 0), (9, 255), (9, 256), (40, 1500), (63, 2047)]:
        gq = h // grp
        ref = Ps[h, q] @ VT[gq * d:(gq + 1) * d, rows].T
        mag = Ps[h, q] @ np.abs(VT[gq * d:(gq + 1) * d, rows]).T
        got = O[s_chk * S + q, h * d:(h + 1) * d]
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * mag), (h, q)
    del O
    # dV = sum over the group's heads of P^T do, do = bf16(dp Wo) (sampled keys)
    dpT = bits_to_f32(a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_DPT))  # H x T
    Wo_hat = bits_to_f32(a.get(1, g.GSQ_DBG_WHAT))
    dV = bits_to_f32(a.get(g.GSQ_ATTN_STAGE, g.GSQ_ATTN_DBG_DV)).reshape(T, nkv * d)
    gk = 3
    dp_s = torch.from_numpy(np.ascontiguousarray(dpT[:, rows].T)).double()
    do = (dp_s @ torch.from_numpy(Wo_hat[:, gk * grp * d:(gk + 1) * grp * d]).double())
    do = do.float().to(torch.bfloat16).double().numpy()  # S x (grp d)
    for key in (0, 255, 256, 1024, 2047):
        ref = np.zeros(d)
        for hig in range(grp):
            h = gk * grp + hig
            ref += Ps[h, :, key] @ do[:, hig * d:(hig + 1) * d]
        got = dV[s_chk * S + key, gk * d:(gk + 1) * d].astype(np.float64)
        assert np.linalg.norm(got - ref) <= 1e-2 * np.linalg.norm(ref) + 1e-12, key
    taus = synth.tau_schedule(1.0, 0.05, cfg["steps"])
    a.run(taus[1:3], 1e-3)
    prefix_loss_vs_oracle()
    a.close()

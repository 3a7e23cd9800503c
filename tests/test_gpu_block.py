"""Parity of the staged block pipeline (gsq_dequant, gsq_block_forward,
gsq_block_quantize) with the oracle (oracle/block.py), through the C ABI.
Needs a B200.

GSQ quantizes the blocks of a model in order, each from the quantized
prefix's output; inside a block Q and K, then V with O, then the MLP on the
block output (agihunt.info summary, optimisation paragraph).

Tolerances: dequantization bit-exact (the same fp32 product and rounding as
the stages' hard weight); the block forward 2^-7 relative on each sublayer's
contribution, per row and normwise.  Both sides round the same GEMM operands
to bf16 (xa, Q, K, P, V, o, xm, silu(a) b), but the GPU accumulates in fp32
and the oracle in fp64, so an operand that sits near a rounding boundary can
land one bf16 unit (2^-8 relative) apart; a sublayer whose operands all
moved by one unit would be off by about 2^-8, and the bound allows twice
that.  (Measured: attention rows 1e-6 without such a flip, up to 3e-3 with;
MLP rows about 1e-3, where the attention's difference moves the bf16
rounding of RMSNorm(h).)  The pipeline's first-step losses of
every stage 1e-2 (the loss contract), final hard errors within 2%, and the
block output equal to the oracle's block forward with the GPU's own hard
weights at the forward tolerance."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

pytestmark = pytest.mark.gpu

FWD_TOL = 2.0 ** -7


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
def B(oracle_mod):
    from oracle import block
    return block


def weights(B, dm, seed, qk_scale=0.02):
    r = np.random.default_rng(seed)
    out = {}
    for n, shp in B.weight_shapes(dm).items():
        sc = qk_scale if n in ("q", "k") else 0.02
        out[n] = synth.bf16_values(r.normal(0, sc, shp))
    return out


def bf16_bits(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy()


def rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_dequant_is_the_hard_weight(g, oracle_mod, mode):
    import torch
    N, K, T = 192, 384, 128
    cfg = synth.small_config(N, K, T, mode, number=97)
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    lay = g.gsq_init(torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda(), 128, mode, seed=4)
    lay.run(synth.tau_schedule(1.0, 0.2, 4), 5e-2)
    packed, _, s32 = g.gsq_harden_pack(lay)
    Wd = g.gsq_dequant(mode, packed, s32, N, K)
    g.gsq_recon_error(lay, g.GSQ_RECON_HARD)   # leaves the hard weight in What
    what = lay.get(g.GSQ_DBG_WHAT)
    assert np.array_equal(bf16_bits(Wd).view(np.uint16), np.asarray(what).view(np.uint16))
    # the codes are the oracle's unpacking of the same stream
    lev = oracle_mod.unpack(mode, np.asarray(packed).reshape(N, -1), K)
    from oracle import block as B
    ref = oracle_mod.bf16_round(np.repeat(s32.astype(np.float64), 128, axis=1)
                                * B.LEVEL_VALUES[mode][lev])
    got = Wd.float().cpu().numpy()
    assert np.mean(got == ref) > 0.9999
    lay.close()


def test_block_forward_matches_oracle(g, B):
    import torch
    dm = B.BlockDims(nseq=2, S=256, nh=8, nkv=2, d=128, F=2816)
    W = weights(B, dm, 31, qk_scale=0.06)
    x = np.random.default_rng(32).normal(0, 1, (dm.T, dm.H))
    h, y = g.gsq_block_forward(torch.from_numpy(x).float().cuda(), W, dm.nseq, dm.S, dm.nh,
                               dm.nkv, dm.d, dm.F)
    h, y = h.cpu().numpy().astype(np.float64), y.cpu().numpy().astype(np.float64)
    f = B.block_forward(np.float32(x), W, dm)
    xs = np.float32(x).astype(np.float64)
    assert rel(h - xs, f["h"] - xs) < FWD_TOL
    assert rel(y - h, f["y"] - f["h"]) < FWD_TOL
    rows_a = (np.linalg.norm((h - xs) - (f["h"] - xs), axis=1)
              / np.linalg.norm(f["h"] - xs, axis=1))
    rows_m = (np.linalg.norm((y - h) - (f["y"] - f["h"]), axis=1)
              / np.linalg.norm(f["y"] - f["h"], axis=1))
    assert rows_a.max() < FWD_TOL and rows_m.max() < FWD_TOL
    # the first query of every sequence attends to itself only: no
    # probability rounding, so the attention rows agree to fp32 accumulation
    assert rows_a[0] < 1e-4 and rows_a[dm.S] < 1e-4


def test_block_forward_full_70b_shape_sampled_rows(g, B):
    """The 70B block (hidden 8192, 64 / 8 heads of 128, MLP 28672) on 8 x 2048
    tokens, the launch configuration of the pipeline bench; rows computed
    one by one by the oracle from the causal prefix of their sequence."""
    import torch
    dm = B.BlockDims(nseq=8, S=2048, nh=64, nkv=8, d=128, F=28672)
    gen = torch.Generator(device="cuda").manual_seed(41)
    x = torch.randn((dm.T, dm.H), generator=gen, device="cuda")
    Wt = {n: (torch.randn(shp, generator=gen, device="cuda") * 0.02).to(torch.bfloat16)
          for n, shp in B.weight_shapes(dm).items()}
    _, y = g.gsq_block_forward(x, Wt, dm.nseq, dm.S, dm.nh, dm.nkv, dm.d, dm.F)
    s, pos = 5, [0, 1, 37, 90]
    xs = x[s * dm.S:s * dm.S + max(pos) + 1].cpu().numpy()
    Wn = {n: w.float().cpu().numpy() for n, w in Wt.items()}
    xpad = np.zeros((dm.S, dm.H), np.float32)
    xpad[:xs.shape[0]] = xs
    dm1 = B.BlockDims(nseq=1, S=dm.S, nh=dm.nh, nkv=dm.nkv, d=dm.d, F=dm.F)
    ref = B.block_forward_rows(xpad, Wn, dm1, 0, pos)
    got = y[[s * dm.S + p for p in pos]].cpu().numpy().astype(np.float64)
    xr = xs[pos].astype(np.float64)
    for i in range(len(pos)):
        assert rel(got[i] - xr[i], ref[i] - xr[i]) < FWD_TOL, pos[i]
    del Wt


STACK = dict(nseq=2, S=128, nh=2, nkv=1, d=128, F=256)


@pytest.fixture(scope="module")
def stacks(g, B):
    """A two-block stack, 6 steps per stage, quantized by both sides."""
    import torch
    dm = B.BlockDims(**STACK)
    x0 = np.random.default_rng(7).normal(0, 1, (dm.T, dm.H)).astype(np.float32)
    taus = [synth.tau_schedule(1.0, 0.05, 6)] * 4
    blocks = [weights(B, dm, 20, 0.06), weights(B, dm, 21, 0.06)]
    ref = B.quantize_stack(x0, blocks, dm, 0, taus, 1e-4, [7, 8])
    gpu, x = [], torch.from_numpy(x0).cuda()
    for Wb, seed in zip(blocks, [7, 8]):
        r = g.gsq_block_quantize(x, Wb, dm.nseq, dm.S, dm.nh, dm.nkv, dm.d, dm.F, taus, 1e-4,
                                 seed=seed)
        r["x_in"] = x.cpu().numpy().astype(np.float64)
        gpu.append(r)
        x = r["x_out"]
    return dm, blocks, ref, gpu


def test_pipeline_stage_losses_match_oracle(stacks):
    _, _, ref, gpu = stacks
    for b, (o, r) in enumerate(zip(ref, gpu)):
        for stage in ("q", "k", "vo", "mlp"):
            first = o["stats"][stage]["losses"][0]
            assert abs(r["stats"][stage]["first_loss"] - first) <= 1e-2 * first, (b, stage)
            ro, rg = o["stats"][stage]["recon"][1], r["stats"][stage]["recon"][1]
            assert abs(rg - ro) <= 0.02 * ro, (b, stage, rg, ro)
            assert r["stats"][stage]["ms"] > 0


def test_pipeline_output_is_the_forward_of_its_hard_weights(g, stacks, B, oracle_mod):
    dm, _, ref, gpu = stacks
    shapes = B.weight_shapes(dm)
    for b, r in enumerate(gpu):
        hard = {}
        for name in B.WEIGHTS:
            N, K = shapes[name]
            lev = oracle_mod.unpack(0, r["packed"][name].cpu().numpy().view(np.uint32)
                                    .reshape(N, -1), K)
            s = r["scales"][name].cpu().numpy().astype(np.float64)
            hard[name] = oracle_mod.bf16_round(np.repeat(s, 128, axis=1)
                                               * B.LEVEL_VALUES[0][lev]).astype(np.float32)
        f = B.block_forward(r["x_in"], hard, dm)
        xo = r["x_out"].cpu().numpy().astype(np.float64)
        assert rel(xo - r["x_in"], f["y"] - r["x_in"]) < FWD_TOL, b
        # the GPU's quantized block is about as far from the full-precision
        # block as the oracle's
        e_gpu = np.sum((xo - ref[b]["y_fp"]) ** 2) if b == 0 else None
        if e_gpu is not None:
            e_ref = np.sum((ref[b]["x_out"] - ref[b]["y_fp"]) ** 2)
            assert abs(e_gpu - e_ref) <= 0.05 * e_ref


def test_pipeline_next_block_sees_quantized_prefix(stacks):
    _, _, _, gpu = stacks
    x1 = gpu[1]["x_in"]
    assert np.array_equal(x1, gpu[0]["x_out"].cpu().numpy().astype(np.float64))


def test_block_quantize_bad_arguments(g, B):
    """Rejected on the host before any buffer is touched."""
    import ctypes as C
    import torch
    dm = B.BlockDims(**STACK)
    W = weights(B, dm, 50)
    keep = [torch.from_numpy(W[n]).to(torch.bfloat16).cuda() for n in B.WEIGHTS]
    arr = (C.c_void_p * 7)(*[w.data_ptr() for w in keep])
    x = torch.zeros((dm.T, dm.H), device="cuda")
    y = torch.zeros((dm.T, dm.H), device="cuda")
    L = g.lib()
    # n_heads not a multiple of n_kv_heads
    assert L.gsq_block_forward(x.data_ptr(), arr, dm.nseq, dm.S, 3, 2, dm.d, dm.F, 5e5, 1e-5,
                               None, y.data_ptr(), None) == g.GSQ_ERR_INVALID_ARG
    # seq_len not a multiple of 128, head_dim other than 128
    assert L.gsq_block_forward(x.data_ptr(), arr, 2, 100, dm.nh, dm.nkv, dm.d, dm.F, 5e5, 1e-5,
                               None, y.data_ptr(), None) == g.GSQ_ERR_UNSUPPORTED
    assert L.gsq_block_forward(x.data_ptr(), arr, dm.nseq, dm.S, 4, 2, 64, dm.F, 5e5, 1e-5,
                               None, y.data_ptr(), None) == g.GSQ_ERR_UNSUPPORTED
    # a null weight
    arr2 = (C.c_void_p * 7)(*([None] + [w.data_ptr() for w in keep[1:]]))
    assert L.gsq_block_forward(x.data_ptr(), arr2, dm.nseq, dm.S, dm.nh, dm.nkv, dm.d, dm.F,
                               5e5, 1e-5, None, y.data_ptr(), None) == g.GSQ_ERR_INVALID_ARG
    # a non-positive temperature
    with pytest.raises(g.GSQError) as e:
        g.gsq_block_quantize(x, W, dm.nseq, dm.S, dm.nh, dm.nkv, dm.d, dm.F,
                             [np.array([1.0, -1.0], np.float32)] * 4, 1e-3)
    assert e.value.status == g.GSQ_ERR_INVALID_ARG
    # the binding checks shapes before the call
    with pytest.raises(ValueError):
        g.gsq_block_forward(x, W, dm.nseq, dm.S, dm.nh * 2, dm.nkv, dm.d, dm.F)
    del keep

"""Pins of the oracle's staged block pipeline (oracle/block.py): GSQ quantizes
the blocks of a model in order, each from the output of the quantized prefix,
and inside a block Q and K first, then V with O, then the MLP on the block
output (agihunt.info summary, optimisation paragraph).  CPU only.

* the block forward against an independent torch fp64 formulation (complex
  rotation for the rotary embedding, torch's scaled-dot-product attention
  with a causal mask, grouped heads by repetition);
* causality and independence of sequences, exactly;
* output rows computed alone (for sampled checks of large layers) equal the
  rows of the full forward;
* weights already on the grid with lr = 0: every stage ends with zero hard
  error and the quantized block reproduces the full-precision block;
* the V/O stage's hard loss equals the error of the quantized attention
  sublayer, and the MLP stage's equals the block-output error
  ||x_out - y_fp||^2 (the MLP is trained on the block output);
* a stack equals the block forward applied in order with the hard weights
  (the next block sees the quantized prefix, not the full-precision one);
* the stages reduce the Q / K errors from the round-to-nearest start.
Planted mistakes in copies of oracle/block.py are each caught by one pin."""
import importlib.util
import os
import sys

import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SMALL = dict(nseq=2, S=8, nh=4, nkv=2, d=16, F=48)
STACK = dict(nseq=2, S=128, nh=2, nkv=1, d=128, F=256)


def weights(B, dm, seed, scale=0.02):
    r = np.random.default_rng(seed)
    return {n: synth.bf16_values(r.normal(0, scale, shp))
            for n, shp in B.weight_shapes(dm).items()}


def torch_block(x, W, dm, theta=500000.0, eps=1e-5):
    """The same block written with torch fp64 library routines."""
    import torch
    import torch.nn.functional as F
    t = lambda a: torch.as_tensor(np.asarray(a, np.float64))  # noqa: E731
    x = t(x)
    Wt = {k: t(v) for k, v in W.items()}

    def rms(v):
        return v * torch.rsqrt(v.pow(2).mean(-1, keepdim=True) + eps)

    def heads(v, n):
        return v.view(dm.nseq, dm.S, n, dm.d).transpose(1, 2)

    def rope(v):
        half = dm.d // 2
        pos = torch.arange(dm.S, dtype=torch.float64)
        inv = theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / dm.d)
        rot = torch.polar(torch.ones(dm.S, half, dtype=torch.float64), pos[:, None] * inv)
        z = torch.complex(v[..., :half], v[..., half:]) * rot
        return torch.cat([z.real, z.imag], dim=-1)

    xa = rms(x)
    q = rope(heads(xa @ Wt["q"].T, dm.nh))
    k = rope(heads(xa @ Wt["k"].T, dm.nkv))
    v = heads(xa @ Wt["v"].T, dm.nkv)
    grp = dm.nh // dm.nkv
    k, v = k.repeat_interleave(grp, dim=1), v.repeat_interleave(grp, dim=1)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
    o = o.transpose(1, 2).reshape(dm.T, dm.H)
    h = x + o @ Wt["o"].T
    xm = rms(h)
    y = h + (F.silu(xm @ Wt["gate"].T) * (xm @ Wt["up"].T)) @ Wt["down"].T
    return h.numpy(), y.numpy()


# ------------------------------------------------------------------ pins

def pin_forward_matches_torch(B):
    dm = B.BlockDims(**SMALL)
    W = weights(B, dm, 1, scale=0.2)
    x = np.random.default_rng(2).normal(0, 1, (dm.T, dm.H))
    f = B.block_forward(x, W, dm, round_bf16=False)
    h, y = torch_block(x, W, dm)

    # the oracle's probability routine takes fp32 inputs and returns fp32
    # probabilities (relative 6e-8 per entry): sublayer outputs normwise 1e-6
    def close(a, b):
        return np.linalg.norm(a - b) <= 1e-6 * np.linalg.norm(b)
    assert close(f["h"] - x, h - x)
    assert close(f["y"] - f["h"], y - h)
    # the bf16-mirroring mode is a small perturbation of the exact block
    fr = B.block_forward(x, W, dm, round_bf16=True)
    assert np.linalg.norm(fr["y"] - y) < 2e-2 * np.linalg.norm(y - x)


def pin_causal_and_sequences_independent(B):
    dm = B.BlockDims(**SMALL)
    W = weights(B, dm, 3, scale=0.2)
    x = np.random.default_rng(4).normal(0, 1, (dm.T, dm.H))
    y = B.block_forward(x, W, dm)["y"]
    x2 = x.copy()
    x2[dm.S - 1] += 1.0          # last token of sequence 0
    y2 = B.block_forward(x2, W, dm)["y"]
    assert np.array_equal(np.delete(y, dm.S - 1, 0), np.delete(y2, dm.S - 1, 0))
    x3 = x.copy()
    x3[dm.S + 2] -= 1.0          # token 2 of sequence 1
    y3 = B.block_forward(x3, W, dm)["y"]
    assert np.array_equal(y[:dm.S + 2], y3[:dm.S + 2])
    assert not np.array_equal(y[dm.S + 3:], y3[dm.S + 3:])


def pin_rows_alone_equal_full_forward(B):
    dm = B.BlockDims(**SMALL)
    W = weights(B, dm, 12, scale=0.2)
    x = np.random.default_rng(13).normal(0, 1, (dm.T, dm.H))
    y = B.block_forward(x, W, dm)["y"]
    for s, pos in ((0, [0, 3]), (1, [7, 2, 5])):
        rows = B.block_forward_rows(x, W, dm, s, pos)
        assert np.allclose(rows, y[[s * dm.S + p for p in pos]], rtol=0, atol=1e-12), (s, pos)


def on_grid_weights(B, dm, seed):
    """Weights on the 2-bit grid with scale 2^-6 and a +-1.5 level in every
    group, so round-to-nearest from absmax / 1.5 recovers them exactly."""
    r = np.random.default_rng(seed)
    out = {}
    for n, (N, K) in B.weight_shapes(dm).items():
        lev = r.integers(0, 4, (N, K))
        lev[:, ::128] = 3
        out[n] = (np.array([-1.5, -0.5, 0.5, 1.5])[lev] * 2.0 ** -6).astype(np.float32)
    return out


def pin_on_grid_block_reproduced(B):
    dm = B.BlockDims(nseq=1, S=128, nh=1, nkv=1, d=128, F=128)
    W = on_grid_weights(B, dm, 5)
    x = np.random.default_rng(6).normal(0, 1, (dm.T, dm.H))
    taus = [synth.tau_schedule(1.0, 0.5, 2)] * 4
    r = B.quantize_block(x, W, dm, 0, taus, 0.0, seed=9)
    for name in B.WEIGHTS:
        assert np.array_equal(r["hard"][name], W[name]), name
    for stage in ("q", "k", "vo"):
        assert r["stats"][stage]["recon"][0] == 0.0, stage
    # the MLP target y_fp - h is a difference of fp64 sums taken in another
    # order than the stage's own forward: zero up to fp64 rounding
    assert r["stats"]["mlp"]["recon"][1] < 1e-24
    assert np.array_equal(r["x_out"], r["y_fp"])


def make_stack(B):
    dm = B.BlockDims(**STACK)
    x0 = np.random.default_rng(7).normal(0, 1, (dm.T, dm.H))
    taus = [synth.tau_schedule(1.0, 0.05, 6)] * 4
    blocks = [weights(B, dm, 20), weights(B, dm, 21)]
    return dm, x0, blocks, B.quantize_stack(x0, blocks, dm, 0, taus, 1e-4, [7, 8])


def pin_stage_losses_are_block_errors(B, stack):
    _, _, _, out = stack
    for r in out:
        ea = float(((r["h"] - r["x_in"] - r["attn_fp"]) ** 2).sum())
        assert abs(r["stats"]["vo"]["recon"][0] - ea) <= 1e-6 * ea
        e = float(((r["x_out"] - r["y_fp"]) ** 2).sum())
        assert e > 0
        assert abs(r["stats"]["mlp"]["recon"][0] - e) <= 1e-9 * e


def pin_stack_is_quantized_prefix_forward(B, stack):
    dm, x0, blocks, out = stack
    x = np.asarray(x0, np.float64)
    for r in out:
        assert np.array_equal(r["x_in"], x)
        f = B.block_forward(x, r["hard"], dm)
        assert np.allclose(f["y"], r["x_out"], rtol=0, atol=1e-12 * np.abs(x).max())
        x = f["y"]
    # block 1 started from the quantized output of block 0, not the full-precision one
    fp0 = B.block_forward(x0, blocks[0], dm)["y"]
    assert np.linalg.norm(out[1]["x_in"] - fp0) > 1e-3 * np.linalg.norm(fp0)


# ----------------------------------------------------------------- tests

@pytest.fixture(scope="module")
def B(oracle_mod):
    from oracle import block
    return block


@pytest.fixture(scope="module")
def stack(B):
    return make_stack(B)


def test_block_forward_matches_torch(B):
    pin_forward_matches_torch(B)


def test_causal_and_sequences_independent(B):
    pin_causal_and_sequences_independent(B)


def test_rows_computed_alone_equal_full_forward(B):
    pin_rows_alone_equal_full_forward(B)


def test_on_grid_block_reproduced_exactly(B):
    pin_on_grid_block_reproduced(B)


def test_stage_losses_are_block_errors(B, stack):
    pin_stage_losses_are_block_errors(B, stack)


def test_stack_is_the_quantized_prefix_forward(B, stack):
    pin_stack_is_quantized_prefix_forward(B, stack)


def test_stages_improve_on_round_to_nearest(B, stack, oracle_mod):
    dm, x0, blocks, out = stack
    r = out[0]
    xa = np.ascontiguousarray(r["xa"], np.float32)
    for name in ("q", "k"):
        st = oracle_mod.init(0, blocks[0][name])
        Y = oracle_mod.reference_output(blocks[0][name], xa)
        rtn = oracle_mod.recon_error(st, xa, Y)[0]
        assert r["stats"][name]["recon"][0] < rtn, name


# ------------------------------------------------------- planted mistakes

MUTATIONS = [
    ("residual_dropped", "    h = x + attn\n", "    h = attn\n",
     lambda B: pin_forward_matches_torch(B)),
    ("rmsnorm_axis", "np.mean(x * x, axis=1, keepdims=True)",
     "np.mean(x * x, axis=0, keepdims=True)", lambda B: pin_forward_matches_torch(B)),
    ("value_head_group", "g = h // grp", "g = h % dm.nkv",
     lambda B: pin_forward_matches_torch(B)),
    ("silu_missing_input", "hh = _r(a / (1.0 + np.exp(-a)) * b, round_bf16)",
     "hh = _r(1.0 / (1.0 + np.exp(-a)) * b, round_bf16)",
     lambda B: pin_forward_matches_torch(B)),
    ("mlp_target_own_output", 'Rm = fp["y"] - h',
     'Rm = mlp_out(xm, W["gate"], W["up"], W["down"], True)',
     lambda B: pin_stage_losses_are_block_errors(B, make_stack(B))),
    ("vo_probs_full_precision", 'P = attn_probs(xa, hard["q"], hard["k"],',
     'P = attn_probs(xa, W["q"], W["k"],',
     lambda B: pin_stage_losses_are_block_errors(B, make_stack(B))),
    ("prefix_full_precision", '        x = r["x_out"]', '        x = r["y_fp"]',
     lambda B: pin_stack_is_quantized_prefix_forward(B, make_stack(B))),
    ("rows_value_head_group", "V[:p + 1, g * dm.d:(g + 1) * dm.d]",
     "V[:p + 1, h % dm.nkv * dm.d:(h % dm.nkv + 1) * dm.d]",
     lambda B: pin_rows_alone_equal_full_forward(B)),
    ("mlp_input_unnormalised", "xm = f32(bf16_round(rmsnorm(h, eps)))",
     "xm = f32(bf16_round(h))", lambda B: pin_on_grid_block_reproduced(B)),
]


def mutated(oracle_mod, name, old, new):
    src = open(os.path.join(ROOT, "oracle", "block.py")).read()
    assert src.count(old) == 1, name
    spec = importlib.util.spec_from_loader(f"oracle.block_mut_{name}", loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    sys.modules[spec.name] = mod  # dataclasses look their module up by name
    exec(compile(src.replace(old, new), f"block_mut_{name}", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(oracle_mod, name, old, new, pin):
    with pytest.raises(AssertionError):
        pin(mutated(oracle_mod, name, old, new))

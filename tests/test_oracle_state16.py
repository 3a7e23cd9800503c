"""Pins of the oracle's bf16 logit / momentum state (the reduced-memory mode
the pages' memory figure points at: per-coordinate logits take 2-5x the
weight memory, agihunt.info summary, limitations paragraph).  After the fp32
Lion update of step t the logits are rounded to bf16 stochastically, with a
9-bit threshold taken from the low 9 bits of the Philox word that gives the
same coordinate and logit its noise at step t + 1; the momenta are rounded to
the nearest bf16.  CPU only.

* stochastic rounding returns one of the two bf16 neighbours, keeps bf16
  values unchanged, and is unbiased to 2^-9 of a bf16 unit over its 512
  thresholds;
* the momenta equal torch's nearest-even bf16 conversion;
* the thresholds are the low 9 bits of the step-(t+1) Philox words (the
  Random123 known-answer-tested generator);
* under a constant Lion direction the stochastically rounded logits follow
  the fp32 trajectory on average, where rounding to nearest would stall."""
import numpy as np
import pytest


def _bf16_neighbours(x):
    """(toward zero, away from zero) bf16 neighbours of fp32 values."""
    b = np.asarray(x, np.float32).view(np.uint32)
    lo = (b & np.uint32(0xFFFF0000)).view(np.float32)
    hi = ((b & np.uint32(0xFFFF0000)) + np.uint32(0x10000)).view(np.float32)
    return lo, hi


def test_stochastic_rounding_brackets_and_is_unbiased(oracle_mod):
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.normal(0, 1, 40), rng.normal(0, 1e-3, 20),
                         [2.0, -0.375, 1.0 + 2.0 ** -9, -(3.0 + 2.0 ** -12)]]).astype(np.float32)
    for x in xs:
        lo, hi = _bf16_neighbours(x)
        ys = np.array([oracle_mod.bf16_sr(float(x), r) for r in range(512)], np.float32)
        if lo == x:
            assert np.all(ys == x)
            continue
        assert np.all((ys == lo) | (ys == hi)), x
        unit = abs(float(hi) - float(lo))
        assert abs(ys.astype(np.float64).mean() - float(x)) <= unit * 2.0 ** -9 + 1e-12, x


def _state(oracle_mod, mode, seed=3):
    from post_weight_quantization_philox_b200 import synth
    W = synth.make_weight(synth.small_config(4, 256, 8, mode, number=80))
    st = oracle_mod.init(mode, W, seed=seed, state16=True)
    rng = np.random.default_rng(9)
    st.logits[:] = rng.normal(0, 1, st.logits.shape).astype(np.float32)
    st.mom[:] = rng.normal(0, 1e-3, st.mom.shape).astype(np.float32)
    return st


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_momenta_round_to_nearest(oracle_mod, mode):
    import torch
    st = _state(oracle_mod, mode)
    before = st.mom.copy()
    oracle_mod.state16_store(st, 7)
    ref = torch.from_numpy(before).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(st.mom, ref)


@pytest.mark.parametrize("mode", [0, 2])
def test_thresholds_are_next_step_philox_words(oracle_mod, mode):
    st = _state(oracle_mod, mode, seed=0x1234_5678_9ABC)
    before = st.logits.copy()
    t_next = 11
    oracle_mod.state16_store(st, t_next)
    L, N, K = before.shape
    key = [st.seed & 0xFFFFFFFF, st.seed >> 32]
    for c in (0, 1, 300, N * K - 1):
        w = list(oracle_mod.philox4x32_10([c & 0xFFFFFFFF, c >> 32, t_next, 0], key))
        if L == 5:
            q = c - c % 4
            w.append(oracle_mod.philox4x32_10([q & 0xFFFFFFFF, q >> 32, t_next, 1], key)[c % 4])
        n, k = divmod(c, K)
        for p in range(L):
            x = before[p, n, k]
            lo, hi = _bf16_neighbours(x)
            low16 = int(np.float32(x).view(np.uint32)) & 0xFFFF
            up = low16 + ((int(w[p]) & 0x1FF) << 7) >= 0x10000
            assert st.logits[p, n, k] == (hi if up else lo), (c, p)


def test_rounding_follows_fp32_lion_on_average(oracle_mod):
    """Constant gradient sign, lr 1e-3, logits at +2 (bf16 unit 2^-6): after
    100 steps the fp32 logits are at 1.9; the stochastically rounded ones
    must average 1.9 too, where rounding to nearest would stay at 2."""
    n = 1 << 14
    st = oracle_mod.init(0, np.full((1, n), 0.01, np.float32), seed=4, state16=True)
    st.logits[:] = 2.0
    theta32 = st.logits.copy()
    m32 = np.zeros_like(theta32)
    grad = np.ones_like(theta32)
    for t in range(100):
        oracle_mod.lion(st.logits, st.mom, grad, 1e-3, 0.9, 0.99)
        oracle_mod.state16_store(st, t + 1)
        oracle_mod.lion(theta32, m32, grad, 1e-3, 0.9, 0.99)
    assert abs(float(theta32.mean()) - 1.9) < 1e-4
    assert abs(float(st.logits.astype(np.float64).mean()) - float(theta32.mean())) < 2e-3
    # every stored logit is a bf16 value
    assert np.array_equal(_bf16_neighbours(st.logits)[0], st.logits)
    # rounding to nearest instead would never leave 2 (a step of 1e-3 is
    # below half a bf16 unit there)
    rn = np.float32(2.0)
    for _ in range(100):
        rn = np.float32(oracle_mod.bf16_round(float(rn - np.float32(1e-3))))
    assert rn == 2.0

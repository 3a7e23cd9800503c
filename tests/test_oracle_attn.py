"""Pins of the oracle's attention V/O joint stage (GSQ staging: Q and K
first, then V and O jointly; agihunt.info summary, optimisation paragraph):
attention probabilities against torch (complex-number rotation and
scaled_dot_product_attention), the rotary embedding's relative-position
property, and the V/O loss and gradients against fp64 autograd.  CPU only."""
import numpy as np
import pytest

DIMS = dict(nseq=2, S=16, nh=4, nkv=2, d=128)


def _inputs(seed=0, nseq=2, S=16, nh=4, nkv=2, d=128):
    rng = np.random.default_rng(seed)
    H, Hk = nh * d, nkv * d
    Xa = rng.normal(0, 1, (nseq * S, H)).astype(np.float32)
    Wq = rng.normal(0, 0.03, (H, H)).astype(np.float32)
    Wk = rng.normal(0, 0.03, (Hk, H)).astype(np.float32)
    Wv = rng.normal(0, 0.03, (Hk, H)).astype(np.float32)
    Wo = rng.normal(0, 0.03, (H, H)).astype(np.float32)
    return Xa, Wq, Wk, Wv, Wo


def _torch_rotated(Xa, Wq, Wk, nseq, S, nh, nkv, d, theta=500000.0):
    """Rotated queries and (group-repeated) keys as [seq, head, pos, d]."""
    import torch
    X = torch.tensor(Xa, dtype=torch.float64)
    Q = (X @ torch.tensor(Wq, dtype=torch.float64).T).view(nseq, S, nh, d)
    K = (X @ torch.tensor(Wk, dtype=torch.float64).T).view(nseq, S, nkv, d)
    half = d // 2
    freq = theta ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
    ang = torch.arange(S, dtype=torch.float64)[:, None] * freq[None, :]
    rot = torch.polar(torch.ones_like(ang), ang)  # e^{i angle}

    def rope(x):  # pairs (i, i + d/2) as complex numbers
        z = torch.complex(x[..., :half], x[..., half:]) * rot[None, :, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    Q, K = rope(Q), rope(K)
    grp = nh // nkv
    K = K.repeat_interleave(grp, dim=2)
    return Q.permute(0, 2, 1, 3), K.permute(0, 2, 1, 3)


def _torch_probs(Xa, Wq, Wk, nseq, S, nh, nkv, d, theta=500000.0):
    import torch
    q, k = _torch_rotated(Xa, Wq, Wk, nseq, S, nh, nkv, d, theta)
    scores = (q @ k.transpose(-1, -2)) / np.sqrt(d)
    mask = torch.triu(torch.ones(S, S, dtype=torch.bool), 1)
    scores = scores.masked_fill(mask, float("-inf"))
    return torch.softmax(scores, dim=-1).numpy()


def test_probs_match_torch(oracle_mod):
    Xa, Wq, Wk, _, _ = _inputs()
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS, round_bf16=False)
    ref = _torch_probs(Xa, Wq, Wk, **DIMS)
    assert np.allclose(P, ref, rtol=1e-6, atol=1e-7)
    # and against torch's fused attention on those rotated inputs: with
    # V = identity per head the attention output equals P
    import torch
    q, k = _torch_rotated(Xa, Wq, Wk, **DIMS)
    eye = torch.eye(DIMS["S"], dtype=torch.float64)[None, None].expand(
        q.shape[0], q.shape[1], -1, -1)
    out = torch.nn.functional.scaled_dot_product_attention(q, k, eye, is_causal=True)
    assert np.allclose(P, out.numpy(), rtol=1e-6, atol=1e-7)


def test_probs_rows_causal_and_normalised(oracle_mod):
    Xa, Wq, Wk, _, _ = _inputs(seed=1)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS, round_bf16=False)
    S = DIMS["S"]
    assert np.allclose(P.sum(-1), 1.0, atol=1e-6)
    assert np.all(P[..., np.triu_indices(S, 1)[0], np.triu_indices(S, 1)[1]] == 0)
    assert np.all(P >= 0)


def test_rotary_relative_position_property(oracle_mod):
    """With the same input at every position, scores depend only on the
    offset key - query, so P[q+1, k+1] / P[q+1, k'+1] = P[q, k] / P[q, k']."""
    nseq, S, nh, nkv, d = 1, 12, 2, 1, 128
    rng = np.random.default_rng(2)
    row = rng.normal(0, 1, (1, nh * d)).astype(np.float32)
    Xa = np.repeat(row, nseq * S, axis=0)
    Wq = rng.normal(0, 0.05, (nh * d, nh * d)).astype(np.float32)
    Wk = rng.normal(0, 0.05, (nkv * d, nh * d)).astype(np.float32)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, nseq, S, nh, nkv, d, round_bf16=False)[0].astype(np.float64)
    for h in range(nh):
        for q in range(1, S - 1):
            for k in range(q):
                r1 = P[h, q, k] / P[h, q, q]
                r2 = P[h, q + 1, k + 1] / P[h, q + 1, q + 1]
                assert np.isclose(r1, r2, rtol=1e-5)


def _torch_vo(Xa, P, R, Wv, Wo, nseq, S, nh, nkv, d):
    import torch
    X = torch.tensor(Xa, dtype=torch.float64)
    Pt = torch.tensor(P, dtype=torch.float64)
    v = torch.tensor(Wv, dtype=torch.float64, requires_grad=True)
    o_w = torch.tensor(Wo, dtype=torch.float64, requires_grad=True)
    V = (X @ v.T).view(nseq, S, nkv, d).permute(0, 2, 1, 3)
    V = V.repeat_interleave(nh // nkv, dim=1)
    o = (Pt @ V).permute(0, 2, 1, 3).reshape(nseq * S, nh * d)
    pred = o @ o_w.T
    loss = ((pred - torch.tensor(R)) ** 2).sum()
    loss.backward()
    return loss.item(), v.grad.numpy(), o_w.grad.numpy()


def test_vo_matches_torch_autograd(oracle_mod):
    Xa, Wq, Wk, Wv, Wo = _inputs(seed=3)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS, round_bf16=False)
    R = np.random.default_rng(4).normal(0, 0.1, (Xa.shape[0], Wo.shape[0]))
    loss, dWv, dWo = oracle_mod.attn_vo_forward_backward(Xa, P, R, Wv, Wo, **DIMS,
                                                         round_bf16=False)
    tl, tv, to = _torch_vo(Xa, P, R, Wv, Wo, **DIMS)
    assert np.isclose(loss, tl, rtol=1e-10)
    assert np.allclose(dWv, tv, rtol=1e-5, atol=1e-6 * np.abs(tv).max())
    assert np.allclose(dWo, to, rtol=1e-5, atol=1e-6 * np.abs(to).max())


def test_vo_bf16_rounding_is_a_small_perturbation(oracle_mod):
    Xa, Wq, Wk, Wv, Wo = _inputs(seed=5)
    P0 = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS, round_bf16=False)
    P1 = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS, round_bf16=True)
    assert np.abs(P1 - P0).max() < 2e-2
    R = np.random.default_rng(6).normal(0, 0.1, (Xa.shape[0], Wo.shape[0]))
    l0, v0, o0 = oracle_mod.attn_vo_forward_backward(Xa, P0, R, Wv, Wo, **DIMS, round_bf16=False)
    l1, v1, o1 = oracle_mod.attn_vo_forward_backward(Xa, P1, R, Wv, Wo, **DIMS, round_bf16=True)
    assert abs(l1 - l0) <= 1e-2 * l0
    assert np.linalg.norm(v1 - v0) <= 3e-2 * np.linalg.norm(v0)


def test_vo_zero_loss_on_own_output(oracle_mod):
    Xa, Wq, Wk, Wv, Wo = _inputs(seed=7)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS, round_bf16=False)
    # target = the exact V/O output -> zero loss and zero gradients
    X = Xa.astype(np.float64)
    nseq, S, nh, nkv, d = DIMS.values()
    V = (X @ Wv.T.astype(np.float64)).reshape(nseq, S, nkv, d)
    o = np.zeros((nseq * S, nh * d))
    for s in range(nseq):
        for h in range(nh):
            o[s * S:(s + 1) * S, h * d:(h + 1) * d] = P[s, h].astype(np.float64) @ V[s, :, h // (nh // nkv)]
    R = o @ Wo.T.astype(np.float64)
    loss, dWv, dWo = oracle_mod.attn_vo_forward_backward(Xa, P, R, Wv, Wo, **DIMS, round_bf16=False)
    assert loss < 1e-18 and np.abs(dWv).max() < 1e-9 and np.abs(dWo).max() < 1e-9


def test_single_row_equals_full_probabilities(oracle_mod):
    Xa, Wq, Wk, _, _ = _inputs(seed=8)
    P = oracle_mod.attn_probs(Xa, Wq, Wk, **DIMS)
    for s, h, q in [(0, 0, 0), (1, 3, 9), (0, 2, 15)]:
        row = oracle_mod.attn_prob_row(Xa, Wq, Wk, DIMS["nseq"], DIMS["S"], DIMS["nh"],
                                       DIMS["nkv"], s, h, q)
        assert np.array_equal(row, P[s, h, q])

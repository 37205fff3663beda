"""Pins of the gradient oracle (``oracle/bwd_oracle.c``) against facts fixed outside it:
torch autograd in float64 through the attention definition, central finite differences
of the forward oracle, identities that hold for any input (value-gradient sum, key-gradient
sum), grouped heads against repeated heads, and the bf16 input path.

The pages state that FlashAttention recomputes attention in the backward pass instead of
storing it ("Flash Attention" page, section "Zentrale technische Innovationen"); what that
pass computes is the gradient of softmax(scale Q K^T [+ mask]) V.
"""
import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def torch_grads(q, k, v, do, scale, causal):
    """float64 autograd of the definition.  Causal masks align at the bottom right (query i
    sees key j iff j <= i + Nk - Nq); a query row with no admissible key has O = 0."""
    group = q.shape[1] // k.shape[1]
    Nq, Nk = q.shape[2], k.shape[2]
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    kk, vv = tk.repeat_interleave(group, 1), tv.repeat_interleave(group, 1)
    if Nq == Nk or not causal:
        o = torch.nn.functional.scaled_dot_product_attention(tq, kk, vv, is_causal=causal,
                                                             scale=scale)
    else:
        keep = torch.ones(Nq, Nk, dtype=torch.bool).tril(diagonal=Nk - Nq)
        s = (scale * tq @ kk.transpose(-1, -2)).masked_fill(~keep, -np.inf)
        m = s.amax(-1, keepdim=True).detach()
        e = torch.exp(s - torch.where(torch.isfinite(m), m, torch.zeros_like(m)))
        den = e.sum(-1, keepdim=True)
        o = (e / torch.where(den > 0, den, torch.ones_like(den))) @ vv
    o.backward(torch.tensor(do))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 2, 17, 17, 8), (2, 4, 1, 9, 9, 16), (1, 3, 3, 5, 23, 4),
                                   (1, 2, 1, 23, 5, 4)])
def test_matches_torch_autograd(shape, causal):
    B, Hq, Hkv, Nq, Nk, d = shape
    q, do = rnd((B, Hq, Nq, d), 1), rnd((B, Hq, Nq, d), 2)
    k, v = rnd((B, Hkv, Nk, d), 3), rnd((B, Hkv, Nk, d), 4)
    got = oracle.attention_bwd(q, k, v, do, 0.37, causal)
    ref = torch_grads(q, k, v, do, 0.37, causal)
    for g, r in zip(got, ref):
        assert np.abs(g - r).max() < 1e-12


@pytest.mark.parametrize("causal,nq,nk", [(False, 5, 5), (True, 5, 5), (True, 3, 6),
                                           (True, 6, 3), (False, 6, 3)])
def test_matches_finite_differences_of_the_forward_oracle(causal, nq, nk):
    """d/dx of L = sum(dO * O) by central differences of the forward oracle (whose causal
    mask is aligned at the bottom right when Nq != Nk)."""
    B, Hq, Hkv, d = 1, 2, 1, 3
    q, k, v = rnd((B, Hq, nq, d), 5), rnd((B, Hkv, nk, d), 6), rnd((B, Hkv, nk, d), 7)
    do = rnd((B, Hq, nq, d), 8)
    scale, h = 0.6, 1e-6
    got = dict(zip("qkv", oracle.attention_bwd(q, k, v, do, scale, causal)))

    def loss(q, k, v):
        return float((oracle.attention(q, k, v, scale, causal)[0] * do).sum())

    for name in "qkv":
        base = dict(q=q, k=k, v=v)
        arr = base[name]
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            lp = loss(**dict(base, **{name: plus}))
            lm = loss(**dict(base, **{name: minus}))
            assert abs((lp - lm) / (2 * h) - got[name][idx]) < 1e-7, (name, idx)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_identities(causal):
    """Rows of P sum to 1, so sum_j dV_j = sum_i dO_i and sum_j dS_ij = 0, which makes
    sum_j dK_j = 0 for every head."""
    B, Hq, Hkv, N, d = 2, 4, 2, 31, 8
    q, do = rnd((B, Hq, N, d), 9), rnd((B, Hq, N, d), 10)
    k, v = rnd((B, Hkv, N, d), 11), rnd((B, Hkv, N, d), 12)
    _, dk, dv = oracle.attention_bwd(q, k, v, do, 0.5, causal)
    dsum = do.reshape(B, Hkv, Hq // Hkv, N, d).sum(axis=(2, 3))
    assert np.abs(dv.sum(axis=2) - dsum).max() < 1e-11
    assert np.abs(dk.sum(axis=2)).max() < 1e-11


def test_grouped_heads_equal_repeated_heads_summed():
    B, Hq, Hkv, N, d = 1, 6, 2, 13, 4
    q, do = rnd((B, Hq, N, d), 13), rnd((B, Hq, N, d), 14)
    k, v = rnd((B, Hkv, N, d), 15), rnd((B, Hkv, N, d), 16)
    dq1, dk1, dv1 = oracle.attention_bwd(q, k, v, do, 0.4, True)
    dq2, dk2, dv2 = oracle.attention_bwd(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1),
                                         do, 0.4, True)
    assert np.abs(dq1 - dq2).max() < 1e-13
    assert np.abs(dk1 - dk2.reshape(B, Hkv, 3, N, d).sum(axis=2)).max() < 1e-12
    assert np.abs(dv1 - dv2.reshape(B, Hkv, 3, N, d).sum(axis=2)).max() < 1e-12


def test_bf16_inputs_decode_exactly():
    t = [torch.randn((1, 2, 11, 8)).to(torch.bfloat16) for _ in range(4)]
    a = oracle.attention_bwd(*t, 0.3, False)
    b = oracle.attention_bwd(*(x.double().numpy() for x in t), 0.3, False)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_causal_rows_without_keys_have_zero_gradient():
    """Causal with Nq = 7 > Nk = 3: query rows 0..3 see no key, so O is the constant 0 there;
    their dQ rows vanish and they add nothing to dK and dV (the gradients of K and V equal
    those of the problem restricted to rows 4..6, which is square and causal)."""
    q, do = rnd((1, 2, 7, 4), 40), rnd((1, 2, 7, 4), 41)
    k, v = rnd((1, 2, 3, 4), 42), rnd((1, 2, 3, 4), 43)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, 0.7, True)
    assert not dq[:, :, :4].any()
    dq2, dk2, dv2 = oracle.attention_bwd(q[:, :, 4:], k, v, do[:, :, 4:], 0.7, True)
    assert np.array_equal(dq[:, :, 4:], dq2)
    assert np.abs(dk - dk2).max() < 1e-14 and np.abs(dv - dv2).max() < 1e-14

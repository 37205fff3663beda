"""Pins for the fp64 CPU oracle, against facts that do not come from the oracle itself.

Each test fixes one property that the attention definition (page "FlashAttention (DE)",
section "Problematik der Standard-Attention": softmax(Q K^T / sqrt(d_k)) V) or plain
mathematics implies: closed forms, invariances, brute force on tiny inputs, a library
routine, and the tiled online-softmax restatement (same page, section
"Online-Softmax-Berechnung").  Together they are chosen so that a dropped term, a wrong
sign or index, a transposed operand or a wrong log base in the oracle fails one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ----------------------------------------------------------------------------- decoders

def test_bf16_decode_matches_torch_on_every_code():
    codes = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.decode_bf16(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.decode_e4m3(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_decode_closed_forms():
    # OCP E4M3: largest finite 448, smallest normal 2^-6, smallest subnormal 2^-9.
    assert oracle.decode_e4m3(0x7E) == 448.0
    assert oracle.decode_e4m3(0xFE) == -448.0
    assert oracle.decode_e4m3(0x08) == 2.0 ** -6
    assert oracle.decode_e4m3(0x01) == 2.0 ** -9
    assert oracle.decode_e4m3(0x38) == 1.0
    assert math.isnan(oracle.decode_e4m3(0x7F))


# ----------------------------------------------------------------------------- closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_constant_scores_give_mean_of_values(causal):
    # All key rows equal => s_ij does not depend on j => softmax is uniform over the
    # admissible keys: O_i = mean of those v_j, LSE_i = s_i0 + ln(#keys).
    B, H, N, d = 2, 3, 37, 8
    q = rnd((B, H, N, d), 1)
    k = np.broadcast_to(rnd((B, H, 1, d), 2), (B, H, N, d)).copy()
    v = rnd((B, H, N, d), 3)
    scale = 0.3
    o, lse = oracle.attention(q, k, v, scale, causal)
    for b in range(B):
        for h in range(H):
            s0 = scale * q[b, h] @ k[b, h, 0]
            for i in range(N):
                n = i + 1 if causal else N
                np.testing.assert_allclose(o[b, h, i], v[b, h, :n].mean(axis=0),
                                           rtol=0, atol=1e-13)
                assert abs(lse[b, h, i] - (s0[i] + math.log(n))) < 1e-12


def test_causal_row_zero_is_first_value_row():
    B, H, N, d = 2, 4, 19, 16
    q, k, v = rnd((B, H, N, d), 4), rnd((B, H, N, d), 5), rnd((B, H, N, d), 6)
    scale = 0.25
    o, lse = oracle.attention(q, k, v, scale, causal=True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], scale * np.einsum("bht,bht->bh", q[:, :, 0], k[:, :, 0]),
                               rtol=0, atol=1e-13)


def test_single_key_gives_that_value_row():
    # Nk = 1: every query attends only to key 0.
    q, k, v = rnd((1, 2, 9, 4), 7), rnd((1, 2, 1, 4), 8), rnd((1, 2, 1, 4), 9)
    o, lse = oracle.attention(q, k, v, 1.7, causal=False)
    np.testing.assert_array_equal(o, np.broadcast_to(v, o.shape))
    np.testing.assert_allclose(lse, 1.7 * np.einsum("bhit,bht->bhi", q, k[:, :, 0]), atol=1e-13)


def test_dominant_score_limit_and_bound():
    # Make key j0 align with query i0 so that s_{i0,j0} = alpha.  Then
    # |O_i0 - v_j0| <= sum_{j != j0} exp(s_j - s_j0) |v_j - v_j0|  (convexity bound),
    # which tends to 0 as alpha grows.
    N, d, scale = 64, 16, 0.125
    q, k, v = rnd((1, 1, N, d), 10), rnd((1, 1, N, d), 11), rnd((1, 1, N, d), 12)
    i0, j0 = 5, 41
    for alpha in (5.0, 20.0, 60.0):
        kk = k.copy()
        kk[0, 0, j0] = alpha * q[0, 0, i0] / (scale * (q[0, 0, i0] @ q[0, 0, i0]))
        o, _ = oracle.attention(q, kk, v, scale, causal=False)
        s = scale * kk[0, 0] @ q[0, 0, i0]
        assert abs(s[j0] - alpha) < 1e-9
        w = np.exp(s - s[j0])
        bound = sum(w[j] * np.abs(v[0, 0, j] - v[0, 0, j0]) for j in range(N) if j != j0)
        err = np.abs(o[0, 0, i0] - v[0, 0, j0])
        assert np.all(err <= bound + 1e-12)
        if alpha >= 60.0:
            assert err.max() < 1e-12


# ----------------------------------------------------------------------------- invariances

def test_key_value_permutation_invariance():
    B, H, N, d = 1, 3, 50, 12
    q, k, v = rnd((B, H, N, d), 13), rnd((B, H, N, d), 14), rnd((B, H, N, d), 15)
    perm = np.random.default_rng(16).permutation(N)
    o1, l1 = oracle.attention(q, k, v, 0.4, causal=False)
    o2, l2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], 0.4, causal=False)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_moves_lse_only(causal):
    # k_j -> k_j + c for all j adds scale*q_i.c to every score of row i: softmax
    # unchanged, LSE_i moves by exactly that amount.
    B, H, N, d = 1, 2, 33, 8
    q, k, v = rnd((B, H, N, d), 17), rnd((B, H, N, d), 18), rnd((B, H, N, d), 19)
    c = rnd((d,), 20)
    scale = 0.35
    o1, l1 = oracle.attention(q, k, v, scale, causal)
    o2, l2 = oracle.attention(q, k + c, v, scale, causal)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2 - l1, scale * q @ c, rtol=0, atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_mha_with_repeated_heads(causal):
    # Query head hq shares K/V head hq // (Hq/Hkv): identical to MHA on K/V whose heads
    # are repeated (Hq/Hkv) times each, in order.
    B, Hq, Hkv, N, d = 2, 8, 2, 21, 8
    q, k, v = rnd((B, Hq, N, d), 21), rnd((B, Hkv, N, d), 22), rnd((B, Hkv, N, d), 23)
    g = Hq // Hkv
    o1, l1 = oracle.attention(q, k, v, 0.3, causal)
    o2, l2 = oracle.attention(q, np.repeat(k, g, axis=1), np.repeat(v, g, axis=1), 0.3, causal)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


# ----------------------------------------------------------------------------- brute force

def _bruteforce(q, k, v, scale, causal):
    # Pure Python, exact-ish sums (math.fsum), no max subtraction.
    Nq, d = len(q), len(q[0])
    o, lse = [], []
    for i in range(Nq):
        keys = range(i + 1) if causal else range(len(k))
        e = [math.exp(scale * math.fsum(q[i][t] * k[j][t] for t in range(d))) for j in keys]
        z = math.fsum(e)
        lse.append(math.log(z))
        o.append([math.fsum(e[n] * v[j][t] for n, j in enumerate(keys)) / z for t in range(d)])
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (1, 1, 4, 3), (1, 2, 8, 4), (2, 1, 7, 2)])
def test_bruteforce_tiny(shape, causal):
    q, k, v = rnd(shape, 24), rnd(shape, 25), rnd(shape, 26)
    o, lse = oracle.attention(q, k, v, 0.7, causal)
    for b in range(shape[0]):
        for h in range(shape[1]):
            bo, bl = _bruteforce(q[b, h].tolist(), k[b, h].tolist(), v[b, h].tolist(), 0.7, causal)
            np.testing.assert_allclose(o[b, h], np.array(bo), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], np.array(bl), rtol=0, atol=1e-12)


def test_nonsquare_noncausal_bruteforce():
    q, k, v = rnd((1, 1, 3, 4), 27), rnd((1, 1, 7, 4), 28), rnd((1, 1, 7, 4), 29)
    o, lse = oracle.attention(q, k, v, 0.5, causal=False)
    bo, bl = _bruteforce(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), 0.5, False)
    np.testing.assert_allclose(o[0, 0], np.array(bo), atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], np.array(bl), atol=1e-12)


@pytest.mark.parametrize("nq,nk", [(3, 5), (5, 3), (4, 4), (1, 6)])
def test_bottom_right_causal_bruteforce(nq, nk):
    """Causal with Nq != Nk: query i sees keys j <= i + (Nk - Nq); a query with no key
    gets O = 0 and LSE = -inf."""
    q, k, v = rnd((1, 1, nq, 3), 33), rnd((1, 1, nk, 3), 34), rnd((1, 1, nk, 3), 35)
    o, lse = oracle.attention(q, k, v, 0.6, causal=True)
    for i in range(nq):
        keys = list(range(0, min(nk, i + 1 + nk - nq)))
        if not keys:
            assert np.all(o[0, 0, i] == 0.0) and lse[0, 0, i] == -np.inf
            continue
        e = [math.exp(0.6 * math.fsum(q[0, 0, i, t] * k[0, 0, j, t] for t in range(3)))
             for j in keys]
        z = math.fsum(e)
        assert abs(lse[0, 0, i] - math.log(z)) < 1e-12
        for t in range(3):
            assert abs(o[0, 0, i, t] - math.fsum(e[n] * v[0, 0, j, t] for n, j in enumerate(keys)) / z) < 1e-12


# ----------------------------------------------------------------------------- library routine

@pytest.mark.parametrize("nq,nk", [(20, 45), (45, 20)])
def test_bottom_right_causal_matches_torch_sdpa_with_explicit_mask(nq, nk):
    q, k, v = rnd((1, 2, nq, 8), 36), rnd((1, 2, nk, 8), 37), rnd((1, 2, nk, 8), 38)
    o, lse = oracle.attention(q, k, v, 0.3, causal=True)
    mask = torch.arange(nk)[None, :] <= torch.arange(nq)[:, None] + (nk - nq)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=mask,
        scale=0.3).numpy()
    rows = mask.any(dim=1).numpy()      # rows with at least one key
    np.testing.assert_allclose(o[:, :, rows], ref[:, :, rows], rtol=0, atol=1e-12)
    assert np.all(o[:, :, ~rows] == 0.0) and np.all(lse[:, :, ~rows] == -np.inf)

@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_float64(causal):
    B, H, N, d = 2, 3, 45, 16
    q, k, v = rnd((B, H, N, d), 30), rnd((B, H, N, d), 31), rnd((B, H, N, d), 32)
    scale = 0.2
    o, _ = oracle.attention(q, k, v, scale, causal)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        is_causal=causal, scale=scale).numpy()
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- online softmax

def _tiled_online(q, k, v, scale, causal, bn, tau):
    """Test-only restatement of the tiled online softmax (page "FlashAttention (DE)",
    section "Online-Softmax-Berechnung"): keys arrive in tiles of bn; a running maximum
    and a running sum of exponentials are kept; the accumulator is rescaled only when
    the tile maximum exceeds the maximum in use by more than tau (in log2 units), the
    lazy rescaling of page "FlashAttention 4: Praxisleitfaden ...", section "Intelligenteres
    Online-Softmax-Rescaling in FA4".  Works in the scaled base-2 domain like the GPU."""
    Nq, d = q.shape
    Nk = k.shape[0]
    c = scale / math.log(2.0)
    o = np.zeros((Nq, d))
    lse = np.zeros(Nq)
    for i in range(Nq):
        m_used, l, acc = -np.inf, 0.0, np.zeros(d)
        last = i + 1 if causal else Nk
        for j0 in range(0, last, bn):
            j1 = min(j0 + bn, last)
            x = (k[j0:j1] @ q[i]) * c
            xm = x.max()
            if xm > m_used + tau:
                alpha = 0.0 if m_used == -np.inf else 2.0 ** (m_used - xm)
                acc *= alpha
                l *= alpha
                m_used = xm
            p = 2.0 ** (x - m_used)
            l += p.sum()
            acc += p @ v[j0:j1]
        o[i] = acc / l
        lse[i] = (m_used + math.log2(l)) * math.log(2.0)
    return o, lse


@pytest.mark.parametrize("bn,tau", [(1, 0.0), (3, 0.0), (16, 3.0), (128, 8.0), (5, 8.0)])
@pytest.mark.parametrize("causal", [False, True])
def test_tiled_online_softmax_reaches_the_definition(bn, tau, causal):
    N, d = 150, 8
    q, k, v = rnd((1, 1, N, d), 33, 2.0), rnd((1, 1, N, d), 34, 2.0), rnd((1, 1, N, d), 35)
    o, lse = oracle.attention(q, k, v, 0.5, causal)
    to, tl = _tiled_online(q[0, 0], k[0, 0], v[0, 0], 0.5, causal, bn, tau)
    np.testing.assert_allclose(o[0, 0], to, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], tl, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- storage formats

@pytest.mark.parametrize("causal", [False, True])
def test_bf16_bits_path_equals_decoded_f64_path(causal):
    g = torch.Generator().manual_seed(36)
    q, k, v = (torch.randn((1, 4, 40, 16), generator=g).to(torch.bfloat16) for _ in range(3))
    o1, l1 = oracle.attention(q, k, v, 0.25, causal)
    o2, l2 = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), 0.25, causal)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_e4m3_path_applies_each_descale_to_its_own_tensor():
    g = torch.Generator().manual_seed(37)
    B, Hq, Hkv, N, d = 2, 4, 2, 24, 16
    q8 = (torch.randn((B, Hq, N, d), generator=g) * 30).clamp(-448, 448).to(torch.float8_e4m3fn)
    k8 = (torch.randn((B, Hkv, N, d), generator=g) * 30).clamp(-448, 448).to(torch.float8_e4m3fn)
    v8 = (torch.randn((B, Hkv, N, d), generator=g) * 30).clamp(-448, 448).to(torch.float8_e4m3fn)
    dq = torch.rand(B * Hq, generator=g, dtype=torch.float64) * 0.01 + 0.001
    dk = torch.rand(B * Hkv, generator=g, dtype=torch.float64) * 0.01 + 0.002
    dv = torch.rand(B * Hkv, generator=g, dtype=torch.float64) * 0.05 + 0.003
    o1, l1 = oracle.attention(q8, k8, v8, 0.125, False, descale_q=dq, descale_k=dk, descale_v=dv)
    qf = q8.double() * dq.reshape(B, Hq, 1, 1)
    kf = k8.double() * dk.reshape(B, Hkv, 1, 1)
    vf = v8.double() * dv.reshape(B, Hkv, 1, 1)
    o2, l2 = oracle.attention(qf.numpy(), kf.numpy(), vf.numpy(), 0.125, False)
    np.testing.assert_allclose(o1, o2, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-14, atol=1e-13)


def test_row_subset_equals_full_rows():
    q, k, v = rnd((2, 3, 30, 8), 38), rnd((2, 3, 30, 8), 39), rnd((2, 3, 30, 8), 40)
    o, lse = oracle.attention(q, k, v, 0.3, True)
    rows = np.array([0, 29, 30, 95, 179, 100])
    so, sl = oracle.attention_rows(q, k, v, 0.3, True, rows=rows)
    np.testing.assert_array_equal(so, o.reshape(-1, 8)[rows])
    np.testing.assert_array_equal(sl, lse.reshape(-1)[rows])


def test_invalid_arguments_are_rejected():
    q, k, v = rnd((1, 3, 4, 2), 41), rnd((1, 2, 4, 2), 42), rnd((1, 2, 4, 2), 43)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, 1.0)            # Hq % Hkv != 0
    q2 = rnd((1, 2, 4, 2), 44)
    with pytest.raises(ValueError):
        oracle.attention_rows(q2, k, v, 1.0, rows=[8])   # row out of range

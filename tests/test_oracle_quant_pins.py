"""Pins of the quantisation oracle (``oracle/quant_oracle.c``) against facts fixed outside
it: SciPy's Hadamard construction, the Hadamard identity H H^T = d I, torch's e4m3 cast,
closed forms for basis vectors, orthogonality (norms, inverse, Q K^T invariance through
the attention oracle), the rounding bound of the e4m3 format, and exact scaling laws.

The method is the incoherent processing of the page "FlashAttention-3 (DE)", section
"Niedrige Praezision (FP8) mit reduziertem Quantisierungsfehler": multiply Q and K by a
random orthogonal (Hadamard) matrix, then quantise to FP8.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle


def _signs(d, seed):
    return np.where(np.random.default_rng(seed).random(d) < 0.5, -1, 1).astype(np.int8)


def _e4m3_values():
    """All finite non-negative e4m3 values in code order, from torch's cast table."""
    return torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


# ------------------------------------------------------------------------- Hadamard matrix

@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_matches_scipy_sylvester_construction(d):
    assert np.array_equal(oracle.hadamard(d), scipy.linalg.hadamard(d).astype(np.float64))


@pytest.mark.parametrize("d", [64, 128])
def test_hadamard_rows_are_orthogonal(d):
    h = oracle.hadamard(d)
    assert np.array_equal(h @ h.T, d * np.eye(d))


@pytest.mark.parametrize("d", [0, 3, 12, 96])
def test_hadamard_rejects_orders_that_are_not_powers_of_two(d):
    with pytest.raises(ValueError):
        oracle.hadamard(d)


# ---------------------------------------------------------------------------- e4m3 encoder

def test_encoder_matches_torch_cast_on_values_midpoints_and_neighbours():
    # Probes are fp32 numbers: torch casts to fp8 from fp32, so an fp64 probe would be
    # rounded twice on torch's side.
    vals = _e4m3_values().astype(np.float32)
    mids = (vals[:-1] + vals[1:]) / 2           # exact ties: must go to the even code
    probes = np.concatenate([
        vals, mids, np.nextafter(mids, np.float32(np.inf)),
        np.nextafter(mids, np.float32(-np.inf)),
        np.random.default_rng(0).uniform(-448, 448, 4000).astype(np.float32),
        np.random.default_rng(1).uniform(-0.03, 0.03, 4000).astype(np.float32),
        np.array([0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10], np.float32)])
    probes = np.concatenate([probes, -probes])
    ref = torch.from_numpy(probes).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.encode_e4m3(float(v)) for v in probes], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_encoder_saturates_to_largest_finite_value():
    for v in (448.0001, 464.0, 479.0, 1e6, np.inf):
        assert oracle.encode_e4m3(v) == 0x7E
        assert oracle.encode_e4m3(-v) == 0xFE


# ------------------------------------------------------------------------------- rotation

def test_rotation_of_a_basis_vector_is_a_signed_hadamard_row():
    d = 128
    s = _signs(d, 2)
    h = scipy.linalg.hadamard(d)
    for t in (0, 1, 37, 127):
        x = np.zeros((1, 1, 1, d))
        x[0, 0, 0, t] = 1.0
        codes, descale, y = oracle.quantize_e4m3(x, s)
        assert np.allclose(y[0, 0, 0], s[t] * h[t] / math.sqrt(d), rtol=0, atol=1e-15)
        # every |y| equals amax, so every code is +-448
        expect = np.where(s[t] * h[t] > 0, 0x7E, 0xFE)
        assert np.array_equal(codes[0, 0, 0], expect)
        assert descale[0] == pytest.approx(1.0 / (448.0 * math.sqrt(d)), rel=1e-15)


def test_rotation_preserves_row_norms_and_inverts_with_its_transpose():
    d = 128
    s = _signs(d, 3)
    x = np.random.default_rng(4).standard_normal((2, 2, 9, d))
    _, _, y = oracle.quantize_e4m3(x, s)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    back = (y @ scipy.linalg.hadamard(d)) * s / math.sqrt(d)
    assert np.abs(back - x).max() < 1e-12


def test_rotation_leaves_attention_unchanged():
    """(Q R)(K R)^T = Q K^T, so attention over rotated Q and K equals attention over Q, K."""
    d = 64
    s = _signs(d, 5)
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((1, 2, 33, d)) for _ in range(3))
    _, _, qr = oracle.quantize_e4m3(q, s)
    _, _, kr = oracle.quantize_e4m3(k, s)
    for causal in (False, True):
        o1, l1 = oracle.attention(q, k, v, 0.125, causal)
        o2, l2 = oracle.attention(qr, kr, v, 0.125, causal)
        assert np.abs(o1 - o2).max() < 1e-12 and np.abs(l1 - l2).max() < 1e-12


def test_unrotated_path_keeps_values():
    x = torch.randn((1, 2, 7, 128)).to(torch.bfloat16)
    _, _, y = oracle.quantize_e4m3(x)
    assert np.array_equal(y, x.double().numpy())


# --------------------------------------------------------------------------- quantisation

@pytest.mark.parametrize("rotate", [False, True])
def test_codes_round_to_nearest_within_half_an_e4m3_step(rotate):
    d = 128
    rng = np.random.default_rng(7)
    x = rng.standard_normal((2, 3, 40, d))
    x[rng.random(x.shape) < 0.01] *= 50.0
    codes, descale, y = oracle.quantize_e4m3(x, _signs(d, 8) if rotate else None)
    u = y / descale.reshape(2, 3, 1, 1)           # the scaled value that was rounded
    deq = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    # half the spacing of e4m3 at |u|: 2^(floor(log2|u|) - 4) for normals (|u| >= 2^-6),
    # 2^-10 in the subnormal range
    e = np.floor(np.log2(np.maximum(np.abs(u), 2.0 ** -6)))
    half_step = 2.0 ** (e - 4)
    assert (np.abs(deq - u) <= half_step * (1 + 1e-12)).all()
    # the largest |y| of each slice maps to +-448 exactly, and descale = amax / 448
    amax = np.abs(y).reshape(6, -1).max(axis=1)
    assert np.allclose(descale, amax / 448.0, rtol=1e-15, atol=0)
    assert (np.abs(deq).reshape(6, -1).max(axis=1) == 448.0).all()


def test_zero_slice_gets_unit_descale_and_zero_codes():
    x = np.zeros((1, 2, 5, 128))
    x[0, 1] = np.random.default_rng(9).standard_normal((5, 128))
    codes, descale, _ = oracle.quantize_e4m3(x, _signs(128, 10))
    assert descale[0] == 1.0 and not codes[0, 0].any()
    assert descale[1] != 1.0 and codes[0, 1].any()


def test_power_of_two_scaling_changes_only_the_descale():
    d = 128
    s = _signs(d, 11)
    x = np.random.default_rng(12).standard_normal((1, 2, 16, d))
    c1, d1, _ = oracle.quantize_e4m3(x, s)
    c2, d2, _ = oracle.quantize_e4m3(x * 2.0 ** 7, s)
    assert np.array_equal(c1, c2) and np.array_equal(d2, d1 * 2.0 ** 7)


def test_incoherent_processing_lowers_score_error_for_channel_outliers():
    """The page's claim, on the oracle alone: when Q and K share a few large channels,
    the scores of the dequantised rotated vectors are closer to Q K^T than those of the
    plainly quantised ones."""
    d = 128
    rng = np.random.default_rng(13)
    q, k = rng.standard_normal((1, 1, 256, d)), rng.standard_normal((1, 1, 256, d))
    ch = rng.permutation(d)[:4]
    q[..., ch] *= 10.0
    k[..., ch] *= 10.0
    exact = q[0, 0] @ k[0, 0].T
    err = {}
    for rotate in (False, True):
        s = _signs(d, 14) if rotate else None
        cq, dq, _ = oracle.quantize_e4m3(q, s)
        ck, dk, _ = oracle.quantize_e4m3(k, s)
        deq = lambda c, ds: torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy() * ds
        sc = deq(cq, dq[0])[0, 0] @ deq(ck, dk[0])[0, 0].T
        err[rotate] = np.sqrt(np.mean((sc - exact) ** 2))
    assert err[True] < err[False] / 2

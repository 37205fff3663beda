"""The pins are not vacuous: each plausible mistake, planted in a copy of the oracle's C
sources (a dropped term, a wrong sign or index, a transposed operand, a wrong log base, a
mis-decoded format, a wrong rounding tie rule or scale, a dropped gradient term), makes at
least one pin fail,
while the real oracle passes them all.  The mistakes are planted on the CPU only, in
temporary builds."""
import math
import os
import shutil

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from oracle import build as oracle_build

SOURCES = oracle_build.SOURCES


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _bruteforce(q, k, v, scale, causal):
    Nq, d = len(q), len(q[0])
    o, lse = [], []
    for i in range(Nq):
        keys = range(i + 1) if causal else range(len(k))
        e = [math.exp(scale * math.fsum(q[i][t] * k[j][t] for t in range(d))) for j in keys]
        z = math.fsum(e)
        lse.append(math.log(z))
        o.append([math.fsum(e[n] * v[j][t] for n, j in enumerate(keys)) / z for t in range(d)])
    return np.array(o), np.array(lse)


# --------------------------------------------------------------- compact pins (lib -> None)

def pin_sdpa(lib):
    for causal in (False, True):
        q, k, v = rnd((1, 3, 21, 16), 1), rnd((1, 3, 21, 16), 2), rnd((1, 3, 21, 16), 3)
        o, _ = oracle.attention(q, k, v, 0.2, causal, _library=lib)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=causal,
            scale=0.2).numpy()
        assert np.abs(o - ref).max() < 1e-12


def pin_bruteforce_lse(lib):
    for causal in (False, True):
        q, k, v = rnd((1, 1, 6, 3), 4), rnd((1, 1, 6, 3), 5), rnd((1, 1, 6, 3), 6)
        o, lse = oracle.attention(q, k, v, 0.7, causal, _library=lib)
        bo, bl = _bruteforce(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), 0.7, causal)
        assert np.abs(o[0, 0] - bo).max() < 1e-12 and np.abs(lse[0, 0] - bl).max() < 1e-12


def pin_bottom_right(lib):
    q, k, v = rnd((1, 1, 4, 3), 10), rnd((1, 1, 7, 3), 11), rnd((1, 1, 7, 3), 12)
    o, _ = oracle.attention(q, k, v, 0.5, True, _library=lib)
    mask = torch.arange(7)[None, :] <= torch.arange(4)[:, None] + 3
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=mask,
        scale=0.5).numpy()
    assert np.abs(o - ref).max() < 1e-12


def pin_gqa(lib):
    q, k, v = rnd((1, 8, 9, 4), 7), rnd((1, 2, 9, 4), 8), rnd((1, 2, 9, 4), 9)
    o1, l1 = oracle.attention(q, k, v, 0.3, False, _library=lib)
    o2, l2 = oracle.attention(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), 0.3, False,
                              _library=lib)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_decoders(lib):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.decode_e4m3(int(c), _library=lib) for c in codes])
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    bcodes = np.array([0x3F80, 0x4000, 0xC1A0, 0x0001, 0x7F7F], dtype=np.uint16)
    bref = torch.from_numpy(bcodes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal([oracle.decode_bf16(int(c), _library=lib) for c in bcodes], bref)


def pin_e4m3_descales(lib):
    g = torch.Generator().manual_seed(10)
    q8, k8, v8 = ((torch.randn((1, 2, 12, 8), generator=g) * 20).to(torch.float8_e4m3fn)
                  for _ in range(3))
    dq = torch.tensor([0.01, 0.02], dtype=torch.float64)
    dk = torch.tensor([0.03, 0.005], dtype=torch.float64)
    dv = torch.tensor([0.07, 0.002], dtype=torch.float64)
    o1, l1 = oracle.attention(q8, k8, v8, 0.5, False, descale_q=dq, descale_k=dk, descale_v=dv,
                              _library=lib)
    f = lambda t, s: (t.double() * s.reshape(1, 2, 1, 1)).numpy()
    o2, l2 = oracle.attention(f(q8, dq), f(k8, dk), f(v8, dv), 0.5, False, _library=lib)
    assert np.abs(o1 - o2).max() < 1e-12 and np.abs(l1 - l2).max() < 1e-12


def _signs(d, seed):
    return np.where(np.random.default_rng(seed).random(d) < 0.5, -1, 1).astype(np.int8)


def pin_hadamard_scipy(lib):
    assert np.array_equal(oracle.hadamard(16, _library=lib), scipy.linalg.hadamard(16))


def pin_encoder_torch(lib):
    vals = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    probes = np.concatenate([vals, (vals[:-1] + vals[1:]) / 2, [500.0]]).astype(np.float32)
    probes = np.concatenate([probes[:-1], -probes[:-1]])
    ref = torch.from_numpy(probes).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = [oracle.encode_e4m3(float(v), _library=lib) for v in probes]
    assert np.array_equal(got, ref) and oracle.encode_e4m3(500.0, _library=lib) == 0x7E


def pin_rotation_basis_and_norm(lib):
    d, s = 32, _signs(32, 20)
    h = scipy.linalg.hadamard(d)
    x = np.zeros((1, 1, 2, d))
    x[0, 0, 0, 5] = 1.0
    x[0, 0, 1] = np.random.default_rng(21).standard_normal(d)
    _, _, y = oracle.quantize_e4m3(x, s, _library=lib)
    assert np.allclose(y[0, 0, 0], s[5] * h[5] / math.sqrt(d), atol=1e-15, rtol=0)
    assert abs(np.linalg.norm(y[0, 0, 1]) - np.linalg.norm(x[0, 0, 1])) < 1e-12


def pin_quantise_rounding_bound(lib):
    rng = np.random.default_rng(22)
    x = rng.standard_normal((1, 2, 8, 32))
    x[0, 0, 3, 4] = 40.0
    x[0, 1] *= -3.0
    x[0, 1, 2, 7] = -60.0
    codes, descale, y = oracle.quantize_e4m3(x, _signs(32, 23), _library=lib)
    u = y / descale.reshape(1, 2, 1, 1)
    deq = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    half = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(u), 2.0 ** -6))) - 4)
    assert (np.abs(deq - u) <= half * (1 + 1e-12)).all()
    assert np.allclose(descale, np.abs(y).reshape(2, -1).max(axis=1) / 448.0, rtol=1e-15)
    assert (np.abs(deq).reshape(2, -1).max(axis=1) == 448.0).all()
    z, dz, _ = oracle.quantize_e4m3(np.zeros((1, 1, 2, 32)), None, _library=lib)
    assert dz[0] == 1.0 and not z.any()


def pin_bwd_autograd(lib):
    for causal, nq, nk in ((False, 7, 7), (True, 7, 7), (True, 5, 9), (True, 9, 5)):
        q, do = rnd((1, 4, nq, 4), 30), rnd((1, 4, nq, 4), 31)
        k, v = rnd((1, 2, nk, 4), 32), rnd((1, 2, nk, 4), 33)
        got = oracle.attention_bwd(q, k, v, do, 0.45, causal, _library=lib)
        tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
        # bottom-right causal mask; rows with no admissible key have O = 0
        keep = torch.ones(nq, nk, dtype=torch.bool)
        if causal:
            keep = keep.tril(diagonal=nk - nq)
        s = (0.45 * tq @ tk.repeat_interleave(2, 1).transpose(-1, -2)).masked_fill(~keep, -np.inf)
        m = s.amax(-1, keepdim=True).detach()
        e = torch.exp(s - torch.where(torch.isfinite(m), m, torch.zeros_like(m)))
        den = e.sum(-1, keepdim=True)
        o = (e / torch.where(den > 0, den, torch.ones_like(den))) @ tv.repeat_interleave(2, 1)
        o.backward(torch.tensor(do))
        for g, r in zip(got, (tq.grad, tk.grad, tv.grad)):
            assert np.abs(g - r.numpy()).max() < 1e-12


def _np_block(counter, key):
    value = (sum(int(w) << (64 * n) for n, w in enumerate(counter)) - 1) % 2**256
    start = np.array([(value >> (64 * n)) & (2**64 - 1) for n in range(4)], dtype=np.uint64)
    return np.random.Philox(counter=start, key=np.array(key, dtype=np.uint64)).random_raw(4)


def pin_philox_numpy(lib):
    for ctr, key in (([6, 7, 9, 11], [3, 5]), ([0, 1, 2, 0], [2**63, 1])):
        assert np.array_equal(oracle.philox4x64(ctr, key, _library=lib), _np_block(ctr, key))


def pin_dropout_bruteforce(lib):
    q, k, v = rnd((1, 2, 5, 3), 40), rnd((1, 2, 40, 3), 41), rnd((1, 2, 40, 3), 42)
    thr, seed, off = 90, 7, 1
    for causal in (False, True):   # causal: bottom-right, query i sees keys j <= i + 35
        o, _ = oracle.attention_dropout_rows(q, k, v, 0.5, causal, thr, seed, off,
                                             _library=lib)
        o = o.reshape(2, 5, 3)
        for h in range(2):
            for i in range(5):
                adm = np.arange(40) <= (i + 35 if causal else 39)
                e = np.exp(0.5 * (k[0, h] @ q[0, h, i])) * adm
                keep = np.array([((int(_np_block([j // 32, i, h, 0], [seed, off])[(j % 32) // 8])
                                   >> (8 * (j % 8))) & 0xFF) >= thr for j in range(40)])
                ref = (e * keep) @ v[0, h] / e.sum() / (1 - thr / 256)
                assert np.abs(o[h, i] - ref).max() < 1e-12


PINS = [pin_sdpa, pin_bruteforce_lse, pin_bottom_right, pin_gqa, pin_decoders, pin_e4m3_descales,
        pin_hadamard_scipy, pin_encoder_torch, pin_rotation_basis_and_norm,
        pin_quantise_rounding_bound, pin_bwd_autograd, pin_philox_numpy, pin_dropout_bruteforce]

MUTANTS = {
    "scale_dropped": ("srow[j] = scale * dot;", "srow[j] = dot;"),
    "causal_off_by_one": ("if (causal && i + 1 + (Nk - Nq) < nkeys) nkeys = i + 1 + (Nk - Nq);",
                          "if (causal && i + 2 + (Nk - Nq) < nkeys) nkeys = i + 2 + (Nk - Nq);"),
    "causal_top_left_alignment": (
        "if (causal && i + 1 + (Nk - Nq) < nkeys) nkeys = i + 1 + (Nk - Nq);",
        "if (causal && i + 1 < nkeys) nkeys = i + 1;"),
    "gqa_head_mapping": ("const int64_t hk = hq / group;", "const int64_t hk = hq % Hkv;"),
    "lse_log_base": ("lse_out[r] = m + log(l);", "lse_out[r] = m + log2(l);"),
    "lse_max_dropped": ("lse_out[r] = m + log(l);", "lse_out[r] = log(l);"),
    "exp_sign": ("const double p = exp(srow[j] - m);", "const double p = exp(m - srow[j]);"),
    "keys_replaced_by_values": (
        "dot += qrow[t] * (load_elem(k, elem_type, kvoff + j * d + t) * dk);",
        "dot += qrow[t] * (load_elem(v, elem_type, kvoff + j * d + t) * dk);"),
    "key_tile_transposed": (
        "dot += qrow[t] * (load_elem(k, elem_type, kvoff + j * d + t) * dk);",
        "dot += qrow[t] * (load_elem(k, elem_type, kvoff + t * Nk + j) * dk);"),
    "normalisation_dropped": ("o_out[r * d + t] = acc[t] / l;", "o_out[r * d + t] = acc[t];"),
    "e4m3_bias": ("mag = ldexp(1.0 + (double)m / 8.0, e - 7);",
                  "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "bf16_shift": ("uint32_t u = ((uint32_t)h) << 16;", "uint32_t u = ((uint32_t)h) << 15;"),
    "descale_mixup": ("const double dv = descale_v ? descale_v[bhk] : 1.0;",
                      "const double dv = descale_k ? descale_k[bhk] : 1.0;"),
    # quantisation oracle
    "hadamard_lower_right_sign": ("out[(i + n) * d + (j + n)] = -h;",
                                  "out[(i + n) * d + (j + n)] = h;"),
    "rotation_norm_dropped": ("y[i * d + j] = acc / sqrt((double)d);", "y[i * d + j] = acc;"),
    "rotation_signs_ignored": ("* (double)signs[t] *", "*"),
    "rotation_wrong_operand": ("acc += load_x(x, elem_type, base + i * d + t)",
                               "acc += load_x(x, elem_type, base + i * d + j)"),
    "ties_to_odd": ("(err == best_err && (c & 1) == 0)", "(err == best_err && (c & 1) == 1)"),
    "amax_signed": ("if (fabs(y[e]) > amax) amax = fabs(y[e]);", "if (y[e] > amax) amax = y[e];"),
    "descale_inverted": ("descale[s] = amax > 0.0 ? amax / E4M3_MAX_FINITE : 1.0;",
                         "descale[s] = amax > 0.0 ? E4M3_MAX_FINITE / amax : 1.0;"),
    "zero_slice_descale": ("descale[s] = amax > 0.0 ? amax / E4M3_MAX_FINITE : 1.0;",
                           "descale[s] = amax > 0.0 ? amax / E4M3_MAX_FINITE : 0.0;"),
    "code_scale_wrong": ("oracle_encode_e4m3(y[e] * E4M3_MAX_FINITE / amax)",
                         "oracle_encode_e4m3(y[e] * 240.0 / amax)"),
    # gradient oracle
    "bwd_dq_row_term_dropped": ("acc += s[j] * (dp[j] - term) * ld(k, elem_type, kvoff + j * d + t);",
                                "acc += s[j] * dp[j] * ld(k, elem_type, kvoff + j * d + t);"),
    "bwd_dk_row_term_dropped": ("const double ds = p * (dpij - rowterm[gi]);",
                                "const double ds = p * dpij;"),
    "bwd_dq_scale_dropped": ("dq[qoff + t] = scale * acc;", "dq[qoff + t] = acc;"),
    "bwd_dv_reads_q": ("dvr[t] += p * ld(dout, elem_type, qoff + t);",
                       "dvr[t] += p * ld(q, elem_type, qoff + t);"),
    "bwd_causal_off_by_one": ("if (causal && j > i + (Nk - Nq)) continue;",
                              "if (causal && j >= i + (Nk - Nq)) continue;"),
    "bwd_key_pass_top_left": ("if (causal && j > i + (Nk - Nq)) continue;",
                              "if (causal && j > i) continue;"),
    "bwd_query_pass_top_left": ("const int64_t last = i + (Nk - Nq);", "const int64_t last = i;"),
    "dropout_causal_top_left": (
        "if (causal && i + 1 + (Nk - Nq) < n_adm) n_adm = i + 1 + (Nk - Nq);",
        "if (causal && i + 1 < n_adm) n_adm = i + 1;"),
    "bwd_row_without_keys_nonzero_dq": ("for (int64_t t = 0; t < d; ++t) dq[qoff + t] = 0.0;",
                                        "for (int64_t t = 0; t < d; ++t) dq[qoff + t] = 1.0;"),
    "bwd_lse_without_sum": ("lse[gi] = m + log(l);", "lse[gi] = m;"),
    "bwd_dp_reads_k": ("dp[j] = dot_rows(dout, qoff, v, kvoff + j * d, elem_type, d);",
                       "dp[j] = dot_rows(dout, qoff, k, kvoff + j * d, elem_type, d);"),
    "bwd_dk_reads_dout": ("dkr[t] += scale * ds * ld(q, elem_type, qoff + t);",
                          "dkr[t] += scale * ds * ld(dout, elem_type, qoff + t);"),
    # dropout oracle
    "philox_key_dropped": ("c0 = hi1 ^ c1 ^ k0;", "c0 = hi1 ^ c1;"),
    "philox_weyl_wrong": ("k1 += W1;", "k1 += W0;"),
    "dropout_byte_order": ("return (uint8_t)(o[t >> 3] >> (8 * (t & 7)));",
                           "return (uint8_t)(o[t >> 3] >> (8 * (7 - (t & 7))));"),
    "dropout_counter_swapped": (
        "const uint64_t ctr[4] = {(uint64_t)(j >> 5), (uint64_t)i, (uint64_t)bh, 0};",
        "const uint64_t ctr[4] = {(uint64_t)(j >> 5), (uint64_t)bh, (uint64_t)i, 0};"),
    "dropout_keep_strict": ("if (oracle_dropout_byte(seed, offset, bh, i, j) >= thr)",
                            "if (oracle_dropout_byte(seed, offset, bh, i, j) > thr)"),
    "dropout_scale_dropped": ("o_out[r * d + t] = acc[t] * keep_scale / row_sum;",
                              "o_out[r * d + t] = acc[t] / row_sum;"),
}


# Mutant builds go to a git-ignored directory inside the repository, one per mutant,
# removed after the test.
BUILD_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), ".mutant_build")


@pytest.fixture
def build_dir(request):
    path = os.path.join(BUILD_DIR, request.node.callspec.id if hasattr(request.node,
                                                                       "callspec") else "x")
    os.makedirs(path, exist_ok=True)
    yield path
    shutil.rmtree(path, ignore_errors=True)


def _build_mutant(build_dir, name, old, new):
    hits = [src for src in SOURCES if open(src).read().count(old) == 1]
    assert len(hits) == 1 and sum(open(src).read().count(old) for src in SOURCES) == 1, \
        "mutation anchor not found exactly once: %s" % name
    sources = []
    for src in SOURCES:
        text = open(src).read()
        path = os.path.join(build_dir, os.path.basename(src))
        with open(path, "w") as f:
            f.write(text.replace(old, new) if src == hits[0] else text)
        sources.append(path)
    lib = os.path.join(build_dir, "lib" + name + ".so")
    oracle_build.compile_library(lib, sources, opt="-O1")
    return oracle.load_library(lib)


def test_real_oracle_passes_every_compact_pin():
    for pin in PINS:
        pin(None)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_is_caught(build_dir, name):
    lib = _build_mutant(build_dir, name, *MUTANTS[name])
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, "no pin caught the mutation %s" % name

"""The pins are not vacuous: each plausible mistake, planted in a copy of the oracle's C
source (a dropped term, a wrong sign or index, a transposed operand, a wrong log base, a
mis-decoded format), makes at least one pin fail, while the real oracle passes them all.
The mistakes are planted on the CPU only, in temporary builds."""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle import build as oracle_build

SRC = oracle_build.SRC


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


PINS = [pin_sdpa, pin_bruteforce_lse, pin_gqa, pin_decoders, pin_e4m3_descales]

MUTANTS = {
    "scale_dropped": ("srow[j] = scale * dot;", "srow[j] = dot;"),
    "causal_off_by_one": ("if (causal && i + 1 < nkeys) nkeys = i + 1;",
                          "if (causal && i + 2 < nkeys) nkeys = i + 2;"),
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
}


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found: %s" % name
    path = tmp_path / (name + ".c")
    path.write_text(src.replace(old, new))
    lib = tmp_path / ("lib" + name + ".so")
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(lib),
                    str(path), "-lm"], check=True)
    return oracle.load_library(str(lib))


def test_real_oracle_passes_every_compact_pin():
    for pin in PINS:
        pin(None)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_is_caught(tmp_path, name):
    lib = _build_mutant(tmp_path, name, *MUTANTS[name])
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, "no pin caught the mutation %s" % name

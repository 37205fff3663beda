"""The C-ABI library: it loads without a GPU, exports every entry point the header
declares, keeps the oracle out of the product, and rejects invalid arguments on the host
before any CUDA call (so these checks run on a CPU-only machine)."""
import os
import re

import pytest

import exact_attention_101_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_b200.h")

A = 0x10000          # a 16-byte-aligned fake address: never dereferenced by these calls
OK_ARGS = dict(B=1, Hq=4, Hkv=2, Nq=256, Nk=256, d=128, scale=0.088, causal=0)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_library_builds_and_loads():
    from exact_attention_101_b200 import build
    assert os.path.exists(build.build())
    assert fa.fa_version() == 100


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert set(names) == set(fa.C_SYMBOLS)
    L = fa.lib()
    for n in names:
        assert hasattr(L, n), n


def test_product_does_not_reference_the_oracle():
    L = fa.lib()
    for sym in ("oracle_attention_rows", "oracle_decode_bf16"):
        with pytest.raises(AttributeError):
            getattr(L, sym)
    pkg = os.path.join(ROOT, "exact_attention_101_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
                assert "attn_oracle" not in src and "liboracle" not in src, f


def call(**kw):
    a = dict(OK_ARGS)
    a.update(kw)
    ptrs = dict(q=A, k=A, v=A, o=A, lse=A)
    for p in list(ptrs):
        if p in a:
            ptrs[p] = a.pop(p)
    dtype = a.pop("dtype", fa.FA_BF16)
    return fa.fa_fwd(ptrs["q"], ptrs["k"], ptrs["v"], ptrs["o"], ptrs["lse"], a["B"], a["Hq"],
                     a["Hkv"], a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"], dtype, None)


@pytest.mark.parametrize("kw", [
    dict(q=0), dict(k=0), dict(v=0), dict(o=0), dict(lse=0),
    dict(q=A + 8), dict(o=A + 4), dict(lse=A + 2),
    dict(B=0), dict(Hq=0), dict(Hkv=0), dict(Nq=0), dict(Nk=0), dict(d=0), dict(Nk=-5),
    dict(Hq=3, Hkv=2), dict(causal=2), dict(scale=0.0), dict(scale=-1.0),
    dict(scale=float("nan")), dict(scale=float("inf")), dict(dtype=fa.FA_E4M3), dict(dtype=7),
    dict(B=1 << 20, Hq=1 << 12, Hkv=1 << 12),
])
def test_invalid_arguments(kw):
    assert call(**kw) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [
    dict(d=96), dict(d=512), dict(d=32),
])
def test_unsupported_configurations(kw):
    assert call(**kw) == fa.FA_ERR_UNSUPPORTED


HOST_OK = dict(qh=A, kh=A, vh=A, oh=A, lh=A, qd=A, kd=A, vd=A, od=A, ld=A, B=1, Hq=4, Hkv=2,
               Nq=256, Nk=256, d=128, scale=0.088, causal=0, dtype=fa.FA_BF16, chunks=0)


def host_call(**kw):
    a = dict(HOST_OK)
    a.update(kw)
    return fa.fa_fwd_host(*(a[n] for n in ("qh", "kh", "vh", "oh", "lh", "qd", "kd", "vd", "od",
                                          "ld", "B", "Hq", "Hkv", "Nq", "Nk", "d", "scale",
                                          "causal", "dtype", "chunks")), None)


@pytest.mark.parametrize("kw", [
    dict(qh=0), dict(kh=0), dict(vh=0), dict(oh=0), dict(lh=0), dict(chunks=-1),
    dict(qd=0), dict(od=A + 4), dict(ld=A + 2), dict(Hq=3), dict(scale=0.0),
    dict(dtype=fa.FA_E4M3), dict(B=0),
])
def test_host_entry_invalid_arguments(kw):
    assert host_call(**kw) == fa.FA_ERR_INVALID_ARG


def test_host_entry_unsupported_head_dim():
    assert host_call(d=96) == fa.FA_ERR_UNSUPPORTED


def test_fp8_entry_validation():
    args = (A, A, A, A, A, 1, 2, 2, 128, 128)
    # missing descales
    assert fa.fa_fwd_fp8(*args, 128, 0.1, 0, 0, A, A, None) == fa.FA_ERR_INVALID_ARG
    # misaligned descale
    assert fa.fa_fwd_fp8(*args, 128, 0.1, 0, A + 2, A, A, None) == fa.FA_ERR_INVALID_ARG
    # fp8 supports d = 128 only
    assert fa.fa_fwd_fp8(*args, 64, 0.1, 0, A, A, A, None) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_fp8(*args, 256, 0.1, 0, A, A, A, None) == fa.FA_ERR_UNSUPPORTED


def test_status_strings():
    for s in range(5):
        assert fa.fa_status_string(s)
    assert fa.fa_status_string(99) == "unknown status"


def test_selftest_rejects_out_of_range_timeout():
    assert fa.fa_selftest_bounded_wait(0, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_selftest_bounded_wait(2000000, None) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [
    dict(x=0), dict(x8=0), dict(descale=0), dict(x=A + 8), dict(x8=A + 4), dict(descale=A + 2),
    dict(B=0), dict(H=0), dict(N=0), dict(d=0), dict(N=-1),
])
def test_quantize_invalid_arguments(kw):
    a = dict(x=A, signs=A, x8=A, descale=A, B=1, H=2, N=64, d=128)
    a.update(kw)
    assert fa.fa_quantize_e4m3(a["x"], a["signs"], a["x8"], a["descale"], a["B"], a["H"],
                               a["N"], a["d"], None) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("d", [64, 256])
def test_quantize_supports_head_dim_128_only(d):
    assert fa.fa_quantize_e4m3(A, None, A, A, 1, 2, 64, d, None) == fa.FA_ERR_UNSUPPORTED


BWD_OK = dict(q=A, k=A, v=A, o=A, dout=A, lse=A, dq=A, dk=A, dv=A, B=1, Hq=4, Hkv=2, Nq=256,
              Nk=256, d=128, scale=0.088, causal=0)


def bwd_call(**kw):
    a = dict(BWD_OK)
    a.update(kw)
    return fa.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"],
                     a["dv"], a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"], a["scale"],
                     a["causal"], None)


@pytest.mark.parametrize("kw", [
    dict(q=0), dict(o=0), dict(dout=0), dict(lse=0), dict(dq=0), dict(dk=0), dict(dv=0),
    dict(dout=A + 8), dict(dq=A + 4), dict(lse=A + 2), dict(B=0), dict(Nq=0), dict(Nk=0),
    dict(Hq=3, Hkv=2), dict(causal=2), dict(scale=0.0), dict(scale=float("nan")),
])
def test_bwd_invalid_arguments(kw):
    assert bwd_call(**kw) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(d=32), dict(d=96), dict(d=256)])
def test_bwd_unsupported_configurations(kw):
    assert bwd_call(**kw) == fa.FA_ERR_UNSUPPORTED


def test_bwd_noalloc_validates_like_fa_bwd_and_rejects_oversize_scratch():
    a = dict(BWD_OK)
    args = lambda **kw: [dict(a, **kw)[n] for n in ("q", "k", "v", "o", "dout", "lse", "dq", "dk",
                                                    "dv", "B", "Hq", "Hkv", "Nq", "Nk", "d",
                                                    "scale", "causal")] + [None]
    assert fa.fa_bwd_noalloc(*args(q=0)) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_noalloc(*args(d=256)) == fa.FA_ERR_UNSUPPORTED
    # B*Hq*Nq*d*4 = 128 MiB of dQ accumulator: more than the fixed 64 MiB scratch
    assert fa.fa_bwd_noalloc(*args(Hq=16, Hkv=16, Nq=16384, Nk=16384)) == fa.FA_ERR_UNSUPPORTED


VL_OK = dict(q=A, k=A, v=A, o=A, lse=A, cq=A, ck=A, B=2, Hq=4, Hkv=2, tq=300, tk=300, maxq=200,
             d=128, scale=0.088, causal=0, dtype=fa.FA_BF16)


def varlen_call(**kw):
    a = dict(VL_OK)
    a.update(kw)
    return fa.fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cq"], a["ck"], a["B"],
                            a["Hq"], a["Hkv"], a["tq"], a["tk"], a["maxq"], a["d"], a["scale"],
                            a["causal"], a["dtype"], None)


@pytest.mark.parametrize("kw", [
    dict(q=0), dict(cq=0), dict(ck=0), dict(cq=A + 2), dict(o=A + 8), dict(B=0), dict(tq=0),
    dict(tk=0), dict(maxq=0), dict(Hq=3), dict(causal=3), dict(scale=-1.0),
    dict(dtype=fa.FA_E4M3),
])
def test_varlen_invalid_arguments(kw):
    assert varlen_call(**kw) == fa.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("d", [32, 96, 512])
def test_varlen_unsupported_head_dims(d):
    assert varlen_call(d=d) == fa.FA_ERR_UNSUPPORTED


@pytest.mark.parametrize("p", [-0.1, 1.0, 1.5, float("nan"), float("inf")])
def test_dropout_probability_range(p):
    assert fa.fa_fwd_dropout(A, A, A, A, A, 1, 2, 2, 128, 128, 128, 0.088, 0, p, 1, 0,
                             fa.FA_BF16, None) == fa.FA_ERR_INVALID_ARG


def test_dropout_dtypes():
    assert fa.fa_fwd_dropout(A, A, A, A, A, 1, 2, 2, 128, 128, 128, 0.088, 0, 0.1, 1, 0,
                             fa.FA_E4M3, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_dropout(A, A, A, A, A, 1, 2, 2, 128, 128, 96, 0.088, 0, 0.1, 1, 0,
                             fa.FA_BF16, None) == fa.FA_ERR_UNSUPPORTED

"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The CUDA library never uses it, and the two share no code.

The attention arithmetic lives in ``attn_oracle.c`` (plain C, IEEE binary64): for every requested
query row it materialises the full score row ``s_j = scale * q.k_j`` over the admissible
keys, takes its maximum ``m``, forms ``p_j = exp(s_j - m)``, ``l = sum_j p_j`` and
returns ``O = sum_j p_j v_j / l`` and ``LSE = m + ln l``.  That is the attention formula
``softmax(Q K^T / sqrt(d_k)) V`` of the page "FlashAttention (DE)", section
"Problematik der Standard-Attention", which the pages say FlashAttention reproduces
exactly.  ``dropout_oracle.c`` holds attention with dropout on the weights (Philox4x64 bytes),
``bwd_oracle.c`` the gradients of that formula (dQ, dK, dV for an upstream dO), and
``quant_oracle.c`` the per-head e4m3 quantisation with the random-sign
Hadamard rotation of the page "FlashAttention-3 (DE)", section "Niedrige Praezision
(FP8) mit reduziertem Quantisierungsfehler".  This module only marshals arrays into that
library.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F64, BF16, E4M3 = 0, 1, 2

_lib = None


def _bind(lib):
    """Declare the C signatures on a loaded oracle library."""
    lib.oracle_attention_rows.restype = ctypes.c_int
    lib.oracle_attention_rows.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_int64, ctypes.c_int64, ctypes.c_double, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int]
    lib.oracle_decode_bf16.restype = ctypes.c_double
    lib.oracle_decode_bf16.argtypes = [ctypes.c_uint16]
    lib.oracle_decode_e4m3.restype = ctypes.c_double
    lib.oracle_decode_e4m3.argtypes = [ctypes.c_uint8]
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    lib.oracle_hadamard.restype = ctypes.c_int
    lib.oracle_hadamard.argtypes = [ctypes.c_int64, ctypes.c_void_p]
    lib.oracle_encode_e4m3.restype = ctypes.c_uint8
    lib.oracle_encode_e4m3.argtypes = [ctypes.c_double]
    lib.oracle_attention_bwd.restype = ctypes.c_int
    lib.oracle_attention_bwd.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
        ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_int]
    lib.oracle_philox4x64.restype = None
    lib.oracle_philox4x64.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.oracle_dropout_byte.restype = ctypes.c_uint8
    lib.oracle_dropout_byte.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int64]
    lib.oracle_attention_dropout_rows.restype = ctypes.c_int
    lib.oracle_attention_dropout_rows.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
        ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
        ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.oracle_quantize_e4m3.restype = ctypes.c_int
    lib.oracle_quantize_e4m3.argtypes = [
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _as_numpy(x):
    """CPU numpy view of a numpy array or CPU torch tensor (bf16 -> uint16 bits,
    float8_e4m3fn -> uint8 bits)."""
    if isinstance(x, np.ndarray):
        return x
    import torch  # only for tensors handed in by the caller
    if x.dtype == torch.bfloat16:
        x = x.view(torch.uint16) if hasattr(torch, "uint16") else x.view(torch.int16)
    elif x.dtype == torch.float8_e4m3fn:
        x = x.view(torch.uint8)
    return x.detach().cpu().contiguous().numpy()


def _elem_type(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return F64
    if a.dtype in (np.uint16, np.int16):
        return BF16
    if a.dtype in (np.uint8, np.int8):
        return E4M3
    raise TypeError("oracle inputs must be float64, bf16 bits (uint16) or e4m3 bits "
                    "(uint8); got %s" % a.dtype)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def attention_rows(q, k, v, scale, causal=False, rows=None, descale_q=None,
                   descale_k=None, descale_v=None, nthreads=0, _library=None):
    """Exact attention for selected query rows.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] -- float64 values, bf16 bit patterns or
    e4m3 bit patterns (all three of one kind).  rows: flattened row indices
    ``(b*Hq + hq)*Nq + i`` or None for every row.  descale_*: per-(batch, head)
    multipliers for e4m3 inputs.  Returns (o [nrows, d] float64, lse [nrows] float64).
    """
    qa, ka, va = (np.ascontiguousarray(_as_numpy(t)) for t in (q, k, v))
    et = _elem_type(qa)
    if _elem_type(ka) != et or _elem_type(va) != et:
        raise TypeError("q, k and v must share one storage format")
    B, Hq, Nq, d = qa.shape
    Bk, Hkv, Nk, dk = ka.shape
    if va.shape != ka.shape or Bk != B or dk != d:
        raise ValueError("shape mismatch between q, k and v")
    if rows is None:
        nrows = B * Hq * Nq
        rows_arr = None
        rows_ptr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        nrows = rows_arr.size
        rows_ptr = rows_arr.ctypes.data
    o = np.empty((nrows, d), dtype=np.float64)
    lse = np.empty((nrows,), dtype=np.float64)
    ds = []
    for arr in (descale_q, descale_k, descale_v):
        ds.append(None if arr is None else
                  np.ascontiguousarray(np.asarray(_as_numpy(arr), dtype=np.float64).reshape(-1)))
    rc = (_library or _load()).oracle_attention_rows(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, et,
        None if ds[0] is None else ds[0].ctypes.data,
        None if ds[1] is None else ds[1].ctypes.data,
        None if ds[2] is None else ds[2].ctypes.data,
        B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
        rows_ptr, nrows, o.ctypes.data, lse.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_rows failed with code %d" % rc)
    return o, lse


def attention(q, k, v, scale, causal=False, **kw):
    """All rows: returns (o [B, Hq, Nq, d], lse [B, Hq, Nq]) in float64."""
    qa = _as_numpy(q)
    B, Hq, Nq, d = qa.shape
    o, lse = attention_rows(q, k, v, scale, causal, rows=None, **kw)
    return o.reshape(B, Hq, Nq, d), lse.reshape(B, Hq, Nq)


def decode_bf16(bits: int, _library=None) -> float:
    return float((_library or _load()).oracle_decode_bf16(int(bits)))


def decode_e4m3(code: int, _library=None) -> float:
    return float((_library or _load()).oracle_decode_e4m3(int(code)))


def attention_bwd(q, k, v, dout, scale, causal=False, nthreads=0, _library=None):
    """Gradients (dq, dk, dv) in float64 of O = softmax(scale Q K^T [+ causal mask]) V for
    the upstream gradient dout.  q, dout: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; float64
    or bf16 bits (all four of one kind)."""
    arrs = [np.ascontiguousarray(_as_numpy(t)) for t in (q, k, v, dout)]
    et = _elem_type(arrs[0])
    if et == E4M3 or any(_elem_type(a) != et for a in arrs):
        raise TypeError("q, k, v, dout must all be float64 or all bf16")
    qa, ka, va, da = arrs
    B, Hq, Nq, d = qa.shape
    Bk, Hkv, Nk, dk_ = ka.shape
    if va.shape != ka.shape or da.shape != qa.shape or Bk != B or dk_ != d:
        raise ValueError("shape mismatch")
    dq = np.empty(qa.shape, dtype=np.float64)
    dk = np.empty(ka.shape, dtype=np.float64)
    dv = np.empty(ka.shape, dtype=np.float64)
    rc = (_library or _load()).oracle_attention_bwd(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, da.ctypes.data, et, B, Hq, Hkv, Nq,
        Nk, d, float(scale), int(bool(causal)), dq.ctypes.data, dk.ctypes.data,
        dv.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_bwd failed with code %d" % rc)
    return dq, dk, dv


def philox4x64(counter, key, _library=None):
    """Philox4x64-10 block for a 4-word counter and a 2-word key (uint64 each)."""
    c = np.ascontiguousarray(np.asarray(counter, dtype=np.uint64).reshape(4))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint64).reshape(2))
    out = np.empty(4, dtype=np.uint64)
    (_library or _load()).oracle_philox4x64(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def dropout_byte(seed, offset, bh, i, j, _library=None) -> int:
    return int((_library or _load()).oracle_dropout_byte(int(seed), int(offset), int(bh),
                                                        int(i), int(j)))


def attention_dropout_rows(q, k, v, scale, causal, threshold, seed, offset, rows=None,
                           nthreads=0, _library=None):
    """Attention with dropout on the weights (keep key j iff its Philox byte >= threshold,
    kept weights scaled by 1 / (1 - threshold/256)) for selected query rows.  q: [B, Hq,
    Nq, d]; k, v: [B, Hkv, Nk, d]; float64 or bf16 bits.  Returns (o [nrows, d], lse)."""
    qa, ka, va = (np.ascontiguousarray(_as_numpy(t)) for t in (q, k, v))
    et = _elem_type(qa)
    if et == E4M3 or _elem_type(ka) != et or _elem_type(va) != et:
        raise TypeError("q, k and v must all be float64 or all bf16")
    B, Hq, Nq, d = qa.shape
    _, Hkv, Nk, _ = ka.shape
    if rows is None:
        nrows, rows_ptr = B * Hq * Nq, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
        nrows, rows_ptr = rows_arr.size, rows_arr.ctypes.data
    o = np.empty((nrows, d), dtype=np.float64)
    lse = np.empty((nrows,), dtype=np.float64)
    rc = (_library or _load()).oracle_attention_dropout_rows(
        qa.ctypes.data, ka.ctypes.data, va.ctypes.data, int(et == BF16), B, Hq, Hkv, Nq, Nk,
        d, float(scale), int(bool(causal)), int(threshold), int(seed), int(offset), rows_ptr,
        nrows, o.ctypes.data, lse.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attention_dropout_rows failed with code %d" % rc)
    return o, lse


def hadamard(d: int, _library=None) -> np.ndarray:
    """Sylvester's Hadamard matrix of order d (a power of two) as float64 [d, d]."""
    out = np.empty((d, d), dtype=np.float64)
    if (_library or _load()).oracle_hadamard(int(d), out.ctypes.data) != 0:
        raise ValueError("d must be a power of two >= 1, got %r" % (d,))
    return out


def encode_e4m3(value: float, _library=None) -> int:
    """Nearest finite OCP e4m3 code (ties to even, saturating at 448)."""
    return int((_library or _load()).oracle_encode_e4m3(float(value)))


def quantize_e4m3(x, signs=None, nthreads=0, _library=None):
    """Per-(batch, head) e4m3 quantisation of x [B, H, N, d] (float64 or bf16 bits),
    after the rotation y = x diag(signs) H / sqrt(d) when ``signs`` (d values of +1/-1)
    is given.  Returns (codes uint8 [B, H, N, d], descale float64 [B*H],
    y float64 [B, H, N, d])."""
    xa = np.ascontiguousarray(_as_numpy(x))
    et = _elem_type(xa)
    if et == E4M3:
        raise TypeError("quantize_e4m3 takes float64 or bf16 input")
    B, H, N, d = xa.shape
    sa = None
    if signs is not None:
        sa = np.ascontiguousarray(np.asarray(_as_numpy(signs)).astype(np.int8).reshape(-1))
        if sa.size != d:
            raise ValueError("signs must have d entries")
    codes = np.empty(xa.shape, dtype=np.uint8)
    descale = np.empty((B * H,), dtype=np.float64)
    y = np.empty(xa.shape, dtype=np.float64)
    rc = (_library or _load()).oracle_quantize_e4m3(
        xa.ctypes.data, et, None if sa is None else sa.ctypes.data, B * H, N, d,
        codes.ctypes.data, descale.ctypes.data, y.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_quantize_e4m3 failed with code %d" % rc)
    return codes, descale, y


def load_library(path):
    """Load another build of the oracle source (the tests use this to check that their
    pins catch deliberately broken copies)."""
    return _bind(ctypes.CDLL(path))

"""B200-native fused exact attention forward: Python binding of ``libfa_b200.so``.

The C ABI (``include/fa_b200.h``) is the product; this module only marshals arguments
into it.  The functions ``fa_fwd``, ``fa_fwd_dropout``, ``fa_fwd_varlen``, ``fa_fwd_fp8``, ``fa_bwd``, ``fa_quantize_e4m3``,
``fa_check_device_error`` and ``fa_status_string`` have the names and argument order of
the C entry points and take raw device pointers.  ``forward`` / ``forward_dropout`` / ``forward_varlen`` /
``forward_fp8`` / ``backward`` / ``quantize_e4m3`` are conveniences that take CUDA tensors (PyTorch provides device
memory and streams only), allocate the outputs and raise on a non-zero status.  Every step of the attention runs in the CUDA kernels; there
is no CPU or library fallback -- if the shared library is missing, importing a function
that needs it raises.
"""
import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_b200.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)
FA_BF16, FA_BF16_OUT_F32, FA_E4M3 = range(3)

# Exported C symbols, in the order of include/fa_b200.h.
C_SYMBOLS = ("fa_fwd", "fa_fwd_host", "fa_fwd_dropout", "fa_fwd_varlen", "fa_fwd_fp8", "fa_bwd", "fa_bwd_noalloc", "fa_quantize_e4m3",
             "fa_check_device_error", "fa_rescale_stats", "fa_selftest_bounded_wait",
             "fa_status_string", "fa_version")

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__("%s failed: %s (status %d)" % (what, fa_status_string(status), status))
        self.status = status


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libfa_b200.so not found at %s; build it with "
                              "`python -m exact_attention_101_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.fa_fwd.restype = i
        L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp]
        L.fa_fwd_host.restype = i
        L.fa_fwd_host.argtypes = [vp] * 10 + [i, i, i, i, i, i, f, i, i, i, vp]
        L.fa_fwd_dropout.restype = i
        L.fa_fwd_dropout.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, f,
                                     ctypes.c_uint64, ctypes.c_uint64, i, vp]
        L.fa_fwd_varlen.restype = i
        L.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, vp]
        L.fa_fwd_fp8.restype = i
        L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp, vp]
        L.fa_bwd.restype = i
        L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp]
        L.fa_bwd_noalloc.restype = i
        L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i,
                                     vp]
        L.fa_quantize_e4m3.restype = i
        L.fa_quantize_e4m3.argtypes = [vp, vp, vp, vp, i, i, i, i, vp]
        L.fa_check_device_error.restype = i
        L.fa_check_device_error.argtypes = [vp]
        u64p = ctypes.POINTER(ctypes.c_ulonglong)
        L.fa_rescale_stats.restype = i
        L.fa_rescale_stats.argtypes = [vp, u64p, u64p, u64p, i]
        L.fa_selftest_bounded_wait.restype = i
        L.fa_selftest_bounded_wait.argtypes = [i, vp]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_status_string.argtypes = [i]
        L.fa_version.restype = i
        L.fa_version.argtypes = []
        _lib = L
    return _lib


# ------------------------------------------------------------------ raw C-ABI mirrors

def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """Raw ``fa_fwd``: pointers are ints (device addresses), stream an int handle."""
    return lib().fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream)


def fa_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev, o_dev, lse_dev,
                B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, chunks, stream) -> int:
    """Raw ``fa_fwd_host``: host and device addresses as ints."""
    return lib().fa_fwd_host(q_host, k_host, v_host, o_host, lse_host, q_dev, k_dev, v_dev,
                             o_dev, lse_dev, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype,
                             int(chunks), stream)


def fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dropout_p, seed,
                   offset, dtype, stream) -> int:
    """Raw ``fa_fwd_dropout``."""
    return lib().fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                                float(dropout_p), int(seed), int(offset), dtype, stream)


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv, total_q, total_k,
                  max_seqlen_q, d, scale, causal, dtype, stream) -> int:
    """Raw ``fa_fwd_varlen``."""
    return lib().fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, Hq, Hkv,
                               total_q, total_k, max_seqlen_q, d, scale, causal, dtype, stream)


def fa_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
               descale_q, descale_k, descale_v, stream) -> int:
    """Raw ``fa_fwd_fp8``."""
    return lib().fa_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                            descale_q, descale_k, descale_v, stream)


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
           stream) -> int:
    """Raw ``fa_bwd``."""
    return lib().fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale,
                        causal, stream)


def fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                   stream) -> int:
    """Raw ``fa_bwd_noalloc`` (fa_bwd with the library's fixed per-device scratch)."""
    return lib().fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d,
                                scale, causal, stream)


def fa_quantize_e4m3(x, signs, x8, descale, B, H, N, d, stream) -> int:
    """Raw ``fa_quantize_e4m3`` (signs may be 0 / None for no rotation)."""
    return lib().fa_quantize_e4m3(x, signs, x8, descale, B, H, N, d, stream)


def fa_check_device_error(stream) -> int:
    return lib().fa_check_device_error(stream)


def fa_rescale_stats(stream, reset=False):
    """Raw ``fa_rescale_stats``: returns (status, steps, lazy, eager)."""
    st, lz, eg = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    r = lib().fa_rescale_stats(stream, ctypes.byref(st), ctypes.byref(lz), ctypes.byref(eg),
                               int(bool(reset)))
    return r, st.value, lz.value, eg.value


def rescale_stats(reset=False, stream=None):
    """(steps, lazy rescales, eager rescales) of the d = 128 bf16 forward since the last
    reset, on the current device; raises on a non-zero status."""
    r, steps, lazy, eager = fa_rescale_stats(_stream_handle(stream), reset)
    if r != FA_OK:
        raise FaError(r, "fa_rescale_stats")
    return steps, lazy, eager


def fa_selftest_bounded_wait(timeout_us, stream) -> int:
    """Raw ``fa_selftest_bounded_wait``: a wait that nothing completes runs out after
    timeout_us; the next fa_check_device_error reports FA_ERR_TIMEOUT."""
    return lib().fa_selftest_bounded_wait(int(timeout_us), stream)


def fa_status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def fa_version() -> int:
    return lib().fa_version()


# ------------------------------------------------------------------ tensor conveniences

def _stream_handle(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check_inputs(q, k, v):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError("%s must be a CUDA tensor" % name)
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous [B, H, N, d]" % name)
        if t.dim() != 4:
            raise ValueError("%s must have 4 dimensions [B, H, N, d]" % name)
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError("shape mismatch: q %s, k %s, v %s" % (tuple(q.shape), tuple(k.shape),
                                                               tuple(v.shape)))
    return B, Hq, Hkv, Nq, Nk, d


def forward(q, k, v, causal=False, scale=None, out_dtype=None, out=None, lse=None,
            stream=None):
    """Exact attention forward for bf16 CUDA tensors in [B, H, N, d] layout.

    Returns ``(o, lse)``: o in ``out_dtype`` (torch.bfloat16 default, or torch.float32),
    lse fp32 [B, Hq, Nq] (natural log).  ``scale`` defaults to 1/sqrt(d).
    """
    import torch
    B, Hq, Hkv, Nq, Nk, d = _check_inputs(q, k, v)
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise ValueError("forward() takes bf16 q, k, v; use forward_fp8() for e4m3")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    dtype = FA_BF16_OUT_F32 if out_dtype == torch.float32 else FA_BF16
    st = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), dtype, _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_fwd")
    return out, lse


def forward_host(q, k, v, causal=False, scale=None, out_dtype=None, out=None, lse=None,
                 device_buffers=None, chunks=0, device=None, stream=None):
    """``forward`` for bf16 [B, H, N, d] tensors in host memory (pinned memory lets the
    copies overlap the kernel).  Returns host ``(o, lse)``, pinned when q is.
    ``device_buffers`` = (q, k, v, o, lse) CUDA tensors of the right shapes to reuse;
    otherwise they are allocated on ``device`` (default: the current CUDA device)."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("%s must be a contiguous bf16 host tensor [B, H, N, d]" % name)
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or dk != d:
        raise ValueError("q, k, v shapes do not match")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    pin = q.is_pinned()
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=out_dtype, pin_memory=pin)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, pin_memory=pin)
    for name, t in (("out", out), ("lse", lse)):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous host tensor" % name)
    if device_buffers is None:
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        device_buffers = (torch.empty(q.shape, dtype=q.dtype, device=dev),
                          torch.empty(k.shape, dtype=k.dtype, device=dev),
                          torch.empty(v.shape, dtype=v.dtype, device=dev),
                          torch.empty(out.shape, dtype=out.dtype, device=dev),
                          torch.empty(lse.shape, dtype=lse.dtype, device=dev))
    qd, kd, vd, od, ld = device_buffers
    dtype = FA_BF16_OUT_F32 if out_dtype == torch.float32 else FA_BF16
    st = fa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), ld.data_ptr(),
                     B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), dtype, chunks,
                     _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_fwd_host")
    return out, lse


def forward_dropout(q, k, v, dropout_p, seed, offset=0, causal=False, scale=None,
                    out_dtype=None, out=None, lse=None, stream=None):
    """``forward`` with dropout on the attention weights (probability rounded to a multiple
    of 1/256; the mask is a function of (seed, offset, batch, head, query, key))."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _check_inputs(q, k, v)
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise ValueError("forward_dropout() takes bf16 q, k, v")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    dtype = FA_BF16_OUT_F32 if out_dtype == torch.float32 else FA_BF16
    st = fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                        lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)),
                        dropout_p, seed, offset, dtype, _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_fwd_dropout")
    return out, lse


def forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, causal=False,
                   scale=None, out_dtype=None, out=None, lse=None, stream=None):
    """Attention over packed sequences of different lengths: q [total_q, Hq, d], k, v
    [total_k, Hkv, d] bf16, cu_seqlens_* int32 CUDA tensors of B+1 offsets.  Returns
    ``(o [total_q, Hq, d], lse [Hq, total_q])``."""
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if (not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 3
                or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous bf16 CUDA tensor [tokens, H, d]" % name)
    total_q, Hq, d = q.shape
    total_k, Hkv, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or dk != d:
        raise ValueError("shape mismatch between q, k and v")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if not t.is_cuda or t.dtype != torch.int32 or t.dim() != 1 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous int32 CUDA tensor" % name)
    B = cu_seqlens_q.numel() - 1
    if cu_seqlens_k.numel() != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must have the same length")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((total_q, Hq, d), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    dtype = FA_BF16_OUT_F32 if out_dtype == torch.float32 else FA_BF16
    st = fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                       cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, Hq, Hkv, total_q,
                       total_k, int(max_seqlen_q), d, scale, int(bool(causal)), dtype,
                       _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_fwd_varlen")
    return out, lse


def forward_fp8(q, k, v, descale_q, descale_k, descale_v, causal=False, scale=None,
                out=None, lse=None, stream=None):
    """fp8-e4m3 attention forward with per-(batch, head) fp32 descales; bf16 output."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _check_inputs(q, k, v)
    for t in (q, k, v):
        if t.dtype != torch.float8_e4m3fn:
            raise ValueError("forward_fp8() takes torch.float8_e4m3fn q, k, v")
    for name, t, n in (("descale_q", descale_q, B * Hq), ("descale_k", descale_k, B * Hkv),
                       ("descale_v", descale_v, B * Hkv)):
        if not t.is_cuda or t.dtype != torch.float32 or t.numel() != n or not t.is_contiguous():
            raise ValueError("%s must be a contiguous CUDA fp32 tensor of %d entries" % (name, n))
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    st = fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                    B, Hq, Hkv, Nq, Nk, d, scale, int(bool(causal)), descale_q.data_ptr(),
                    descale_k.data_ptr(), descale_v.data_ptr(), _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_fwd_fp8")
    return out, lse


def backward(q, k, v, o, lse, dout, causal=False, scale=None, dq=None, dk=None, dv=None,
             stream=None):
    """Gradients (dq, dk, dv) of the bf16 forward for the upstream gradient ``dout``;
    ``o`` and ``lse`` are that forward's outputs.  All bf16 CUDA tensors in [B, H, N, d]
    layout (lse fp32 [B, Hq, Nq])."""
    import torch
    B, Hq, Hkv, Nq, Nk, d = _check_inputs(q, k, v)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous bf16 CUDA tensor" % name)
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("o and dout must have q's shape")
    if (lse.dtype != torch.float32 or not lse.is_cuda or not lse.is_contiguous()
            or tuple(lse.shape) != (B, Hq, Nq)):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor [B, Hq, Nq]")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    st = fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq,
                Nk, d, scale, int(bool(causal)), _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_bwd")
    return dq, dk, dv


def quantize_e4m3(x, signs=None, out=None, descale=None, stream=None):
    """Per-(batch, head) e4m3 quantisation of a bf16 CUDA tensor x [B, H, N, 128], after
    the random-sign Hadamard rotation when ``signs`` (int8 CUDA tensor of 128 entries,
    +1 / -1) is given.  Returns ``(codes, descale)``: torch.float8_e4m3fn [B, H, N, 128]
    and fp32 [B*H], ready for ``forward_fp8``."""
    import torch
    if not x.is_cuda or x.dtype != torch.bfloat16 or x.dim() != 4 or not x.is_contiguous():
        raise ValueError("x must be a contiguous bf16 CUDA tensor [B, H, N, d]")
    B, H, N, d = x.shape
    if signs is not None and (not signs.is_cuda or signs.dtype != torch.int8 or
                              signs.numel() != d or not signs.is_contiguous()):
        raise ValueError("signs must be a contiguous int8 CUDA tensor of d entries")
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.float8_e4m3fn, device=x.device)
    if descale is None:
        descale = torch.empty((B * H,), dtype=torch.float32, device=x.device)
    st = fa_quantize_e4m3(x.data_ptr(), None if signs is None else signs.data_ptr(),
                          out.data_ptr(), descale.data_ptr(), B, H, N, d,
                          _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_quantize_e4m3")
    return out, descale


def check_device_error(stream=None):
    """Raise FaError if a bounded device-side wait gave up since the last check."""
    st = fa_check_device_error(_stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "device")

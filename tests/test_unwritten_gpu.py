"""Every output element is written by the call that owns it.  Outputs are filled with NaN
before each call (a fresh allocation can hold the correct results of an earlier identical
call, which would hide a skipped work unit); afterwards every element must be finite,
except the LSE of rows that admit no key (causal with more queries than keys), which is
-inf.  The shapes span many more work units than SMs, so that units are claimed
dynamically by every CTA."""
import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
from workloads import random_bf16

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def nan(shape, dtype, pin=False, device=DEV):
    if device is None:
        return torch.full(shape, float("nan"), dtype=dtype).pin_memory() if pin else \
            torch.full(shape, float("nan"), dtype=dtype)
    return torch.full(shape, float("nan"), dtype=dtype, device=device)


def check_lse(lse, Nq, Nk, causal):
    lse = lse.float().cpu()
    if causal and Nq > Nk:
        assert torch.isneginf(lse[..., :Nq - Nk]).all()
        assert torch.isfinite(lse[..., Nq - Nk:]).all()
    else:
        assert torch.isfinite(lse).all()


@pytest.mark.parametrize("shape,causal,out_dtype", [
    ((2, 32, 8, 4096, 4096, 128), True, torch.bfloat16),    # 1024 units
    ((2, 32, 8, 4096, 4096, 128), False, torch.bfloat16),
    ((2, 6, 3, 385, 385, 64), False, torch.float32),
    ((16, 12, 12, 512, 512, 64), True, torch.bfloat16),     # 384 units
    ((1, 2, 2, 300, 1000, 256), True, torch.bfloat16),
    ((2, 16, 4, 2048, 2048, 256), False, torch.float32),   # 256 units on CTA pairs
    ((2, 4, 2, 513, 129, 256), True, torch.bfloat16),      # rows without keys, CTA pairs
    ((3, 4, 1, 513, 129, 128), True, torch.bfloat16),       # rows without keys
    ((1, 3, 3, 1, 1, 64), False, torch.float32),
])
def test_forward_writes_every_output(cuda_ok, shape, causal, out_dtype):
    B, Hq, Hkv, Nq, Nk, d = shape
    q = random_bf16((B, Hq, Nq, d), 900).to(DEV)
    k, v = random_bf16((B, Hkv, Nk, d), 901).to(DEV), random_bf16((B, Hkv, Nk, d), 902).to(DEV)
    for rep in range(2):
        o, lse = nan((B, Hq, Nq, d), out_dtype), nan((B, Hq, Nq), torch.float32)
        fa.forward(q, k, v, causal=causal, out_dtype=out_dtype, out=o, lse=lse)
        torch.cuda.synchronize()
        assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
        assert torch.isfinite(o.float()).all(), rep
        check_lse(lse, Nq, Nk, causal)


def test_dropout_writes_every_output(cuda_ok):
    B, H, N, d = 2, 16, 2048, 128
    q, k, v = (random_bf16((B, H, N, d), 910 + s).to(DEV) for s in range(3))
    o, lse = nan((B, H, N, d), torch.bfloat16), nan((B, H, N), torch.float32)
    fa.forward_dropout(q, k, v, 0.2, seed=3, offset=1, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_varlen_writes_every_output(cuda_ok):
    lengths = [4096, 17, 1, 2000, 777, 3000, 128, 129] * 4
    total, H, d = sum(lengths), 16, 128
    q, k, v = (random_bf16((total, H, d), 920 + s).to(DEV) for s in range(3))
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=DEV)
    for causal in (False, True):
        o, lse = nan((total, H, d), torch.bfloat16), nan((H, total), torch.float32)
        fa.forward_varlen(q, k, v, cu, cu, max(lengths), causal=causal, out=o, lse=lse)
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all(), causal


def test_fp8_writes_every_output(cuda_ok):
    B, H, N, d = 4, 16, 2048, 128
    q, k, v = (random_bf16((B, H, N, d), 930 + s).to(DEV) for s in range(3))
    codes, desc = [], []
    for t in (q, k, v):
        c = torch.empty(t.shape, dtype=torch.float8_e4m3fn, device=DEV)
        s = torch.empty((B * H,), dtype=torch.float32, device=DEV)
        fa.quantize_e4m3(t, None, out=c, descale=s)
        codes.append(c)
        desc.append(s)
    o, lse = nan((B, H, N, d), torch.bfloat16), nan((B, H, N), torch.float32)
    fa.forward_fp8(*codes, *desc, causal=True, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_writes_every_gradient(cuda_ok, d, causal):
    B, Hq, Hkv, N = 2, 16, 4, 2048
    q = random_bf16((B, Hq, N, d), 940).to(DEV)
    k, v = random_bf16((B, Hkv, N, d), 941).to(DEV), random_bf16((B, Hkv, N, d), 942).to(DEV)
    do = random_bf16((B, Hq, N, d), 943).to(DEV)
    o, lse = fa.forward(q, k, v, causal=causal)
    dq, dk, dv = (nan(t.shape, torch.bfloat16) for t in (q, k, v))
    fa.backward(q, k, v, o, lse, do, causal=causal, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert torch.isfinite(g.float()).all(), name


def test_host_path_writes_every_output(cuda_ok):
    B, Hq, Hkv, N, d = 2, 8, 4, 1500, 128
    q = random_bf16((B, Hq, N, d), 950).pin_memory()
    k = random_bf16((B, Hkv, N, d), 951).pin_memory()
    v = random_bf16((B, Hkv, N, d), 952).pin_memory()
    bufs = (nan(q.shape, torch.bfloat16), nan(k.shape, torch.bfloat16),
            nan(v.shape, torch.bfloat16), nan(q.shape, torch.bfloat16),
            nan((B, Hq, N), torch.float32))
    o = nan(q.shape, torch.bfloat16, pin=True, device=None)
    lse = nan((B, Hq, N), torch.float32, pin=True, device=None)
    fa.forward_host(q, k, v, causal=True, out=o, lse=lse, device_buffers=bufs, chunks=3)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()

"""fa_bwd_noalloc: the backward pass in the library's fixed per-device scratch gives what
fa_bwd (stream-ordered scratch) gives, on two calls in a row (the second call must not see
the first call's accumulator: the fixed buffer is cleared every call), and matches the
fp64 gradient oracle within the backward's bar."""
import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
import oracle
from workloads import random_bf16

pytestmark = pytest.mark.gpu


def _bwd(fn, q, k, v, o, lse, do, causal, scale):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
            scale, int(causal), torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return dq, dk, dv


@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row(cuda_ok, causal):
    dev = torch.device("cuda", 0)
    B, Hq, Hkv, N, d = 1, 4, 2, 1000, 128
    scale = 0.088
    q, do = (random_bf16((B, Hq, N, d), 60 + s).to(dev) for s in range(2))
    k, v = (random_bf16((B, Hkv, N, d), 62 + s).to(dev) for s in range(2))
    o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
    ref = _bwd(fa.fa_bwd, q, k, v, o, lse, do, causal, scale)
    for _ in range(2):
        got = _bwd(fa.fa_bwd_noalloc, q, k, v, o, lse, do, causal, scale)
        torch.cuda.synchronize()
        assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
        # dK, dV are reduced without atomics: identical bits
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
        # dQ is summed by reductions in any order: equal up to fp32 rounding of the sum
        diff = (got[0].float() - ref[0].float()).abs().max().item()
        assert diff <= 1e-2 * ref[0].float().abs().max().item(), diff


def test_noalloc_matches_gradient_oracle(cuda_ok):
    # Grouped heads, causal with Nq < Nk (bottom-right alignment), a ragged tail; the bar of
    # the backward's parity tests: relative RMS error <= 1e-2 and max error <= 2e-2 of the
    # largest reference magnitude, per gradient.
    dev = torch.device("cuda", 0)
    B, Hq, Hkv, Nq, Nk, d = 1, 4, 2, 333, 500, 64
    scale = float(torch.tensor(0.125, dtype=torch.float32))
    q, do = random_bf16((B, Hq, Nq, d), 70), random_bf16((B, Hq, Nq, d), 71)
    k, v = random_bf16((B, Hkv, Nk, d), 72), random_bf16((B, Hkv, Nk, d), 73)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa.forward(qd, kd, vd, causal=True, scale=scale)
    got = _bwd(fa.fa_bwd_noalloc, qd, kd, vd, o, lse, dod, True, scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    ref = oracle.attention_bwd(q, k, v, do, scale, True)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        e = g.cpu().to(torch.float64).numpy() - r
        rr = float(np.linalg.norm(e) / np.linalg.norm(r))
        mr = float(np.abs(e).max() / np.abs(r).max())
        print(name, rr, mr)
        assert rr <= 1e-2 and mr <= 2e-2, (name, rr, mr)

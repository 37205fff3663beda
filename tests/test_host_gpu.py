"""GPU tests of ``fa_fwd_host``: the forward for tensors in host memory, pipelined by
chunks of heads.  Every chunk runs the same kernel on the same rows as one ``fa_fwd`` call,
so the results must equal ``fa_fwd`` on the same data bit for bit, whatever the chunking,
the host memory kind (pinned or pageable) or the stream; one case is also checked against
the oracle directly."""
import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
import oracle
from parity_util import compare_bf16
from workloads import random_bf16

pytestmark = pytest.mark.gpu


def device_reference(q, k, v, causal, scale, out_dtype):
    dev = torch.device("cuda", 0)
    o, lse = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale,
                        out_dtype=out_dtype)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def inputs(B, Hq, Hkv, Nq, Nk, d, seed, pin):
    q = random_bf16((B, Hq, Nq, d), seed)
    k = random_bf16((B, Hkv, Nk, d), seed + 1)
    v = random_bf16((B, Hkv, Nk, d), seed + 2)
    if pin:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    return q, k, v


@pytest.mark.parametrize("pin", [True, False])
@pytest.mark.parametrize("chunks", [0, 1, 3, 1000])
@pytest.mark.parametrize("shape,causal,out_dtype", [
    ((1, 8, 2, 700, 700, 128), True, torch.bfloat16),
    ((3, 4, 4, 385, 385, 64), False, torch.bfloat16),
    ((2, 6, 3, 200, 333, 256), False, torch.float32),
    ((2, 4, 1, 300, 129, 128), True, torch.bfloat16),
])
def test_host_forward_equals_device_forward(cuda_ok, shape, causal, out_dtype, chunks, pin):
    B, Hq, Hkv, Nq, Nk, d = shape
    q, k, v = inputs(B, Hq, Hkv, Nq, Nk, d, 700 + d, pin)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.forward_host(q, k, v, causal=causal, scale=scale, out_dtype=out_dtype,
                             chunks=chunks)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    ro, rl = device_reference(q, k, v, causal, scale, out_dtype)
    assert torch.equal(o, ro) and torch.equal(lse, rl)


def test_host_forward_reuses_device_buffers_on_a_side_stream(cuda_ok):
    """Two calls in a row on one set of device buffers, on a non-default stream: the
    second call's input copies must wait for the first call's kernels, and the host
    results of both must be complete once the stream is synchronised."""
    dev = torch.device("cuda", 0)
    B, Hq, Hkv, N, d = 2, 8, 4, 640, 128
    a = inputs(B, Hq, Hkv, N, N, d, 800, True)
    b = inputs(B, Hq, Hkv, N, N, d, 810, True)
    bufs = (torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev),
            torch.empty((B, Hkv, N, d), dtype=torch.bfloat16, device=dev),
            torch.empty((B, Hkv, N, d), dtype=torch.bfloat16, device=dev),
            torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev),
            torch.empty((B, Hq, N), dtype=torch.float32, device=dev))
    side = torch.cuda.Stream(dev)
    oa, la = fa.forward_host(*a, causal=True, device_buffers=bufs, chunks=5, stream=side)
    ob, lb = fa.forward_host(*b, causal=True, device_buffers=bufs, chunks=3, stream=side)
    side.synchronize()
    ra = device_reference(*a, True, 1.0 / np.sqrt(d), torch.bfloat16)
    rb = device_reference(*b, True, 1.0 / np.sqrt(d), torch.bfloat16)
    assert torch.equal(oa, ra[0]) and torch.equal(la, ra[1])
    assert torch.equal(ob, rb[0]) and torch.equal(lb, rb[1])


def test_host_forward_against_oracle(cuda_ok):
    B, Hq, Hkv, N, d = 1, 4, 2, 515, 128
    q, k, v = inputs(B, Hq, Hkv, N, N, d, 820, True)
    scale = float(torch.tensor(1.0 / np.sqrt(d), dtype=torch.float32))
    o, lse = fa.forward_host(q, k, v, causal=True, scale=scale, chunks=2)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(q, k, v, scale, True)
    print(compare_bf16(o.reshape(-1, d), lse.reshape(-1), ro.reshape(-1, d), rl.reshape(-1)))

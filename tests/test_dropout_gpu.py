"""GPU parity of the fused dropout (``fa_fwd_dropout``) against the fp64 dropout oracle.

Both sides draw the keep decisions from the same Philox4x64-10 blocks (counter (key/32,
query, batch*Hq + head, 0), key (seed, offset)), each from its own implementation, so the
comparison is element by element, with the bf16 tolerances of the plain forward scaled by
1/(1 - p) (kept weights are scaled by it).  The page "Flash Attention" lists dropout among
the operations fused with the softmax.
"""
import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
import oracle
from parity_util import BF16_MAX_ABS, BF16_MEAN_ABS, LSE_MAX_ABS
from workloads import random_bf16

pytestmark = pytest.mark.gpu


def run(q, k, v, p, seed, offset, causal, scale, out_dtype=torch.bfloat16):
    dev = torch.device("cuda", 0)
    o, lse = fa.forward_dropout(q.to(dev), k.to(dev), v.to(dev), p, seed, offset,
                                causal=causal, scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 2, 200, 128), (2, 4, 1, 333, 64), (1, 2, 2, 129, 256)])
def test_dropout_matches_oracle(cuda_ok, shape, causal, p):
    B, Hq, Hkv, N, d = shape
    scale = float(torch.tensor(1 / np.sqrt(d), dtype=torch.float32))
    q = random_bf16((B, Hq, N, d), 600)
    k, v = random_bf16((B, Hkv, N, d), 601), random_bf16((B, Hkv, N, d), 602)
    seed, offset = 0x1234ABCD5678, 17
    o, lse = run(q, k, v, p, seed, offset, causal, scale, torch.float32)
    thr = min(255, int(round(p * 256)))
    ro, rl = oracle.attention_dropout_rows(q, k, v, scale, causal, thr, seed, offset)
    og = o.double().numpy().reshape(ro.shape)
    err = np.abs(og - ro)
    grow = 1.0 / (1.0 - thr / 256.0)
    stats = (float(err.max()), float(err.mean()), float(np.abs(lse.double().numpy().reshape(-1) - rl).max()))
    print(shape, causal, p, stats)
    assert stats[0] <= BF16_MAX_ABS * grow and stats[1] <= BF16_MEAN_ABS * grow
    assert stats[2] <= LSE_MAX_ABS


def test_threshold_zero_equals_fa_fwd_and_offset_changes_the_mask(cuda_ok):
    dev = torch.device("cuda", 0)
    q, k, v = (random_bf16((1, 2, 300, 128), 610 + s) for s in range(3))
    o0, l0 = run(q, k, v, 0.0, 5, 0, True, 0.088)
    o1, l1 = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal=True, scale=0.088)
    assert torch.equal(o0, o1.cpu()) and torch.equal(l0, l1.cpu())
    a = run(q, k, v, 0.25, 5, 0, False, 0.088)[0]
    b = run(q, k, v, 0.25, 5, 0, False, 0.088)[0]
    c = run(q, k, v, 0.25, 5, 1, False, 0.088)[0]
    assert torch.equal(a, b) and not torch.equal(a, c)


def test_dropout_full_size_sampled(cuda_ok):
    """The dropout benchmark workload at full size (B1 H32 N16384 d128, p = 0.1, offset 0
    as in the bench's first timed step), rows sampled over four heads, against the oracle."""
    import workloads
    from parity_util import sample_rows
    w = workloads.WORKLOADS["long_dropout"]
    inp = workloads.make_inputs(w)
    o, lse = run(inp.q, inp.k, inp.v, w.dropout, w.seed, 0, w.causal, w.scale)
    rows = sample_rows(w.B, w.Hq, w.N, n_heads=4, n_random=96, seed=w.seed)
    thr = min(255, int(round(w.dropout * 256)))
    ro, rl = oracle.attention_dropout_rows(inp.q, inp.k, inp.v, w.scale, w.causal, thr, w.seed,
                                           0, rows=rows)
    og = o.reshape(-1, w.d)[rows].double().numpy()
    err = np.abs(og - ro)
    grow = 1.0 / (1.0 - thr / 256.0)
    stats = (float(err.max()), float(err.mean()),
             float(np.abs(lse.reshape(-1)[rows].double().numpy() - rl).max()))
    print(stats)
    assert stats[0] <= BF16_MAX_ABS * grow and stats[1] <= BF16_MEAN_ABS * grow
    assert stats[2] <= LSE_MAX_ABS

"""Lazy rescaling of the online softmax on the GPU (page "FlashAttention 4: Praxisleitfaden
...", section "Intelligenteres Online-Softmax-Rescaling in FA4").

Scores that drift along the keys keep raising the running row maximum, so the accumulator
is rescaled on many key blocks: the results must still match the oracle (head dims 64, 128,
256 and fp8).  The CTA-pair kernel (head dim 128 without the mask, 256) also counts its
rescales (fa_rescale_stats): the number of (row, key block) steps follows from the shapes,
the drift forces lazy rescales, the eager rule would have made more, and on i.i.d. normal
inputs the lazy rule never fires after a row's first key block."""
import math

import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
import workloads
from parity_util import (FP8_RRMSE, LSE_MAX_ABS, compare_bf16, oracle_rows, rrmse,
                         run_cuda)

pytestmark = pytest.mark.gpu

SCALE = 0.3


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_drifting_scores_parity(cuda_ok, d, causal):
    inp = workloads.drift_inputs(1, 2, 1024, d, seed=5)
    o, lse = run_cuda(inp, causal, SCALE, torch.float32)
    o_ref, lse_ref = oracle_rows(inp, causal, SCALE)
    print(d, causal, compare_bf16(o.reshape(-1, d), lse.reshape(-1), o_ref, lse_ref))


@pytest.mark.parametrize("causal", [False, True])
def test_drifting_scores_fp8(cuda_ok, causal):
    inp = workloads.quantise_inputs_e4m3(workloads.drift_inputs(1, 2, 1024, 128, seed=6))
    o, lse = run_cuda(inp, causal, SCALE)
    o_ref, lse_ref = oracle_rows(inp, causal, SCALE)
    e = rrmse(o.reshape(-1, 128), o_ref)
    de = float(np.abs(lse.reshape(-1).double().numpy() - lse_ref).max())
    print("fp8 drift", causal, e, de)
    assert e <= FP8_RRMSE and de <= LSE_MAX_ABS


def _stats_of(inp, causal, scale):
    fa.rescale_stats(reset=True)
    run_cuda(inp, causal, scale)
    return fa.rescale_stats(reset=True)


def test_rescale_counters_drift(cuda_ok):
    B, H, N, d = 1, 2, 2048, 128
    inp = workloads.drift_inputs(B, H, N, d, seed=7)
    steps, lazy, eager = _stats_of(inp, False, SCALE)
    # every row of every 256-row unit meets every 128-key block once
    assert steps == B * H * math.ceil(N / 256) * 256 * math.ceil(N / 128), steps
    print("drift: steps", steps, "lazy", lazy, "eager", eager)
    assert lazy > 0
    assert eager >= 1.5 * lazy


def test_rescale_counters_normal_inputs(cuda_ok):
    B, H, N, d = 1, 4, 4096, 128
    inp = workloads.Inputs(*(workloads.random_bf16((B, H, N, d), 80 + s) for s in range(3)))
    steps, lazy, eager = _stats_of(inp, False, 1 / math.sqrt(d))
    assert steps == B * H * (N // 256) * 256 * (N // 128)
    print("normal: steps", steps, "lazy", lazy, "eager", eager)
    # a block maximum 8 (log2 units) above the first block's never occurs here
    assert lazy == 0
    assert eager > 0

"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs.  Small shapes are compared element by element over every output; the
full-size workloads are compared on whole (batch, head) slices and on sampled rows of
further slices, plus properties that hold at any size; an opt-in test compares whole
tensors."""
import os

import numpy as np
import pytest
import torch

import workloads
from parity_util import (BF16_MAX_ABS, BF16_MEAN_ABS, FP8_RRMSE, LSE_MAX_ABS, compare_bf16,
                         compare_fp8, oracle_rows, rows_of_slices, rrmse, run_cuda,
                         slice_plan, slice_rows)

pytestmark = pytest.mark.gpu
W = workloads.WORKLOADS


def small_case(B, Hq, Hkv, Nq, Nk, d, seed):
    w = workloads.Workload("case", B, Hq, Hkv, Nq, d, False, "bf16", "bf16", seed)
    return workloads.make_inputs(w, B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=d)


def full_compare(inp, causal, scale, out_dtype=torch.bfloat16):
    o, lse = run_cuda(inp, causal, scale, out_dtype)
    o_ref, lse_ref = oracle_rows(inp, causal, scale)
    return compare_bf16(o.reshape(-1, o.shape[-1]), lse.reshape(-1), o_ref, lse_ref)


def test_tiny_workload_full_tensor(cuda_ok):
    w = W["tiny"]
    inp = workloads.make_inputs(w)
    full_compare(inp, w.causal, w.scale, torch.float32)


# Odd shapes: single rows/keys, tile and unit boundaries (128, 256), ragged tails,
# d = 64/128/256, MHA/GQA/MQA, causal on and off, bf16 and fp32 outputs.
SHAPES = [
    # B, Hq, Hkv, N, d
    (1, 1, 1, 1, 64), (1, 1, 1, 17, 128), (1, 2, 1, 127, 64), (1, 2, 2, 128, 128),
    (2, 2, 2, 129, 64), (1, 4, 2, 255, 128), (1, 2, 2, 256, 64), (1, 2, 1, 257, 128),
    (1, 3, 3, 383, 64), (2, 4, 1, 513, 128), (1, 8, 8, 1000, 64), (1, 4, 4, 1000, 128),
    # head dim 256: one 128-row Q tile per unit
    (1, 1, 1, 1, 256), (1, 2, 1, 127, 256), (1, 2, 2, 128, 256), (2, 2, 2, 129, 256),
    (1, 4, 2, 513, 256), (1, 2, 2, 1000, 256),
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "B%dH%d-%dN%dd%d" % s)
def test_odd_shapes_full_tensor(cuda_ok, shape, causal):
    B, Hq, Hkv, N, d = shape
    inp = small_case(B, Hq, Hkv, N, N, d, seed=7 + N + d)
    full_compare(inp, causal, 1.0 / np.sqrt(d))


@pytest.mark.parametrize("nq,nk,d", [(1, 300, 64), (200, 1, 128), (300, 1000, 128), (700, 129, 64),
                                     (300, 700, 256)])
def test_non_square_non_causal(cuda_ok, nq, nk, d):
    inp = small_case(1, 2, 2, nq, nk, d, seed=nq * 7 + nk)
    full_compare(inp, False, 1.0 / np.sqrt(d))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_fp32_and_bf16_outputs_agree(cuda_ok, out_dtype):
    inp = small_case(1, 2, 2, 300, 300, 64, seed=99)
    full_compare(inp, True, 0.125, out_dtype)


def test_large_scores_trigger_lazy_rescale(cuda_ok):
    # Scores growing along the key axis force the running maximum up again and again, so
    # the lazy rescale of the accumulator runs on many tiles.
    B, H, N, d = 1, 2, 1024, 64
    g = torch.Generator().manual_seed(5)
    q = torch.randn((B, H, N, d), generator=g)
    k = torch.randn((B, H, N, d), generator=g) * 0.2
    k += torch.linspace(0, 12, N)[None, None, :, None] * q.mean(dim=2, keepdim=True).sign()
    v = torch.randn((B, H, N, d), generator=g)
    inp = workloads.Inputs(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))
    full_compare(inp, False, 0.3)
    full_compare(inp, True, 0.3)


def test_deterministic(cuda_ok):
    inp = small_case(2, 4, 2, 777, 777, 128, seed=3)
    a = run_cuda(inp, True, 0.088)
    b = run_cuda(inp, True, 0.088)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# The benchmark workloads are compared on whole (batch, head) slices -- every row and
# every column of O, and every LSE -- for the first, the last and two random slices, and on
# sampled rows of eight more slices.  The head dimension 256 workloads compare their last
# slice whole (one slice of the long d = 256 shape is about 20 s of oracle on 16 cores).
WHOLE_SLICES = {"gpt2": 4, "gpt2_causal": 4, "long": 4, "long_causal": 4, "gqa_causal": 4,
                "long_d256": 1, "long_d256_causal": 1}


def check_properties(w, inp, o, lse):
    """Properties every row must have, at any size."""
    # a convex combination of value rows lies inside their per-column range
    of = o.float()
    vf = inp.v.float()
    g = w.Hq // w.Hkv
    vmin = vf.amin(dim=2).repeat_interleave(g, dim=1)[:, :, None, :]
    vmax = vf.amax(dim=2).repeat_interleave(g, dim=1)[:, :, None, :]
    tol = 1e-2 * torch.maximum(vmax.abs(), vmin.abs())
    assert torch.all(of >= vmin - tol) and torch.all(of <= vmax + tol)
    assert torch.isfinite(lse).all()
    # causal row 0 attends to key 0 only: O = v_0 (exact in bf16), LSE = scale q0.k0
    if w.causal:
        v0 = inp.v[:, :, 0].repeat_interleave(g, dim=1)
        assert torch.equal(o[:, :, 0], v0)
        k0 = inp.k[:, :, 0].double().repeat_interleave(g, dim=1)
        l0 = w.scale * (inp.q[:, :, 0].double() * k0).sum(-1)
        assert torch.max(torch.abs(lse[:, :, 0].double() - l0)) < 1e-3


@pytest.mark.parametrize("name", list(WHOLE_SLICES))
def test_full_size_workloads(cuda_ok, name):
    w = W[name]
    inp = workloads.make_inputs(w)
    o, lse = run_cuda(inp, w.causal, w.scale)
    of, lf = o.reshape(-1, w.d), lse.reshape(-1)
    whole, sampled = slice_plan(w.B * w.Hq, w.seed, n_whole=WHOLE_SLICES[name], n_sampled=8)
    # 1. whole slices against the oracle, element by element
    for bh in whole:
        rows = slice_rows(bh, w.N)
        o_ref, lse_ref = oracle_rows(inp, w.causal, w.scale, rows)
        print(name, "slice", bh, "whole", compare_bf16(of[rows], lf[rows], o_ref, lse_ref))
    # 2. sampled rows of further slices against the oracle
    rows = rows_of_slices(sampled, w.N, n_random=160, seed=w.seed)
    o_ref, lse_ref = oracle_rows(inp, w.causal, w.scale, rows)
    print(name, "slices", sampled, "sampled", compare_bf16(of[rows], lf[rows], o_ref, lse_ref))
    # 3. properties of every row
    check_properties(w, inp, o, lse)


def test_fp8_small_full_tensor(cuda_ok):
    w = W["fp8"]
    inp = workloads.make_inputs(w, B=1, Hq=4, Hkv=2, Nq=700, Nk=700)
    o, lse = run_cuda(inp, False, w.scale)
    o_ref, lse_ref = oracle_rows(inp, False, w.scale)
    e = rrmse(o.reshape(-1, w.d), o_ref)
    print("fp8 small rrmse", e)
    assert e <= FP8_RRMSE
    assert np.max(np.abs(lse.reshape(-1).double().numpy() - lse_ref)) < 2e-2


def test_fp8_causal_small(cuda_ok):
    w = W["fp8"]
    inp = workloads.make_inputs(w, B=1, Hq=2, Hkv=2, Nq=600, Nk=600)
    o, lse = run_cuda(inp, True, w.scale)
    o_ref, _ = oracle_rows(inp, True, w.scale)
    assert rrmse(o.reshape(-1, w.d), o_ref) <= FP8_RRMSE


def test_fp8_full_size(cuda_ok):
    w = W["fp8"]
    inp = workloads.make_inputs(w)
    o, lse = run_cuda(inp, False, w.scale)
    of, lf = o.reshape(-1, w.d), lse.reshape(-1)
    whole, sampled = slice_plan(w.B * w.Hq, w.seed, n_whole=4, n_sampled=8)
    for bh in whole:
        rows = slice_rows(bh, w.N)
        o_ref, lse_ref = oracle_rows(inp, False, w.scale, rows)
        print("fp8 slice", bh, "whole", compare_fp8(of[rows], lf[rows], o_ref, lse_ref))
    rows = rows_of_slices(sampled, w.N, n_random=192, seed=w.seed)
    o_ref, lse_ref = oracle_rows(inp, False, w.scale, rows)
    print("fp8 slices", sampled, "sampled", compare_fp8(of[rows], lf[rows], o_ref, lse_ref))
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


# Opt-in: every slice of a benchmark workload against the oracle, i.e. the whole tensor
# (FA_WHOLE_TENSOR=1; the long workload alone is about 5.5 minutes of oracle time on 16
# cores).  Prints one summary line per workload.
@pytest.mark.skipif(os.environ.get("FA_WHOLE_TENSOR") != "1",
                    reason="opt-in whole-tensor comparison (set FA_WHOLE_TENSOR=1)")
@pytest.mark.parametrize("name", ["gpt2", "gpt2_causal", "long", "long_causal", "gqa_causal",
                                  "fp8", "long_d256", "long_d256_causal"])
def test_whole_tensor(cuda_ok, name):
    w = W[name]
    inp = workloads.make_inputs(w)
    o, lse = run_cuda(inp, w.causal, w.scale)
    og = o.reshape(-1, w.d).to(torch.float64).numpy()
    lg = lse.reshape(-1).to(torch.float64).numpy()
    BH, per = w.B * w.Hq, max(1, 65536 // w.N)
    mx = lmx = sad = sq = sqref = 0.0
    n = 0
    for h0 in range(0, BH, per):
        rows = np.arange(h0 * w.N, min(BH, h0 + per) * w.N, dtype=np.int64)
        o_ref, lse_ref = oracle_rows(inp, w.causal, w.scale, rows)
        d = np.abs(og[rows] - o_ref)
        mx, sad, n = max(mx, float(d.max())), sad + float(d.sum()), n + d.size
        sq, sqref = sq + float((d * d).sum()), sqref + float((o_ref * o_ref).sum())
        lmx = max(lmx, float(np.abs(lg[rows] - lse_ref).max()))
    stats = dict(workload=name, elements=n, max_abs=mx, mean_abs=sad / n,
                 rrmse=float(np.sqrt(sq / sqref)), lse_max=lmx)
    print("WHOLE_TENSOR", stats)
    if name == "fp8":
        assert stats["rrmse"] <= FP8_RRMSE and lmx <= LSE_MAX_ABS, stats
    else:
        assert mx <= BF16_MAX_ABS and sad / n <= BF16_MEAN_ABS and lmx <= LSE_MAX_ABS, stats

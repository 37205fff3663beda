"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle on the same seeded inputs."""
import numpy as np
import torch

import exact_attention_101_b200 as fa
import oracle

# Tolerances of the acceptance bar (bf16 inputs, fp32 accumulation): max |dO| 2e-2,
# mean |dO| 2e-3, max |dLSE| 1e-3; fp8 e4m3 inputs: relative RMSE of O 3e-2.
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
FP8_RRMSE = 3e-2


def run_cuda(inp, causal, scale, out_dtype=torch.bfloat16):
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in (inp.q, inp.k, inp.v))
    if inp.descale_q is not None:
        o, lse = fa.forward_fp8(q, k, v, inp.descale_q.to(dev), inp.descale_k.to(dev),
                                inp.descale_v.to(dev), causal=causal, scale=scale)
    else:
        o, lse = fa.forward(q, k, v, causal=causal, scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    return o.cpu(), lse.cpu()


def oracle_rows(inp, causal, scale, rows=None):
    kw = {}
    if inp.descale_q is not None:
        kw = dict(descale_q=inp.descale_q.double(), descale_k=inp.descale_k.double(),
                  descale_v=inp.descale_v.double())
    return oracle.attention_rows(inp.q, inp.k, inp.v, scale, causal, rows=rows, **kw)


def rows_of_slices(heads, Nq, n_random=256, seed=0):
    """Rows at tile and unit boundaries, the ragged tail and random rows of the given
    (batch, head) slices, as flattened row indices."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 2, 63, 64, 127, 128, 129, 255, 256, 257, 511, 512, Nq // 2, Nq - 129,
             Nq - 128, Nq - 2, Nq - 1]
    rows = []
    for bh in heads:
        rr = set(i for i in fixed if 0 <= i < Nq)
        rr |= set(int(x) for x in rng.integers(0, Nq, size=n_random))
        rows += [bh * Nq + i for i in sorted(rr)]
    return np.array(rows, dtype=np.int64)


def sample_rows(B, Hq, Nq, n_heads=4, n_random=256, seed=0):
    """Sampled rows (see rows_of_slices) over a few (batch, head) slices: the first, the
    last and random ones."""
    rng = np.random.default_rng(seed)
    BH = B * Hq
    heads = sorted(set([0, BH - 1] + list(rng.integers(0, BH, size=max(0, n_heads - 2)))))
    return rows_of_slices(heads, Nq, n_random, seed)


def slice_plan(BH, seed, n_whole=4, n_sampled=8):
    """(batch, head) slices to compare whole -- the first, the last and random others (only
    the last when n_whole is 1) -- and further random slices to compare on sampled rows."""
    rng = np.random.default_rng(seed)
    inner = [int(x) for x in rng.permutation(np.arange(1, BH - 1))] if BH > 2 else []
    ends = [BH - 1] if n_whole == 1 else [0, BH - 1]
    whole = sorted(set(ends + inner[:max(0, n_whole - 2)]))
    rest = [h for h in ([0] + inner) if h not in whole]
    return whole, sorted(rest[:n_sampled])


def slice_rows(bh, Nq):
    """Every row of (batch, head) slice bh, as flattened row indices."""
    return np.arange(bh * Nq, (bh + 1) * Nq, dtype=np.int64)


def compare_fp8(o_gpu, lse_gpu, o_ref, lse_ref, lse_bar=None):
    """fp8 bar: relative RMSE of O over the compared rows; the LSE (computed from the same
    e4m3 codes on both sides, unaffected by the rounding of P) within LSE_MAX_ABS."""
    lg = lse_gpu.to(torch.float64).numpy().reshape(lse_ref.shape)
    stats = dict(rrmse=rrmse(o_gpu, o_ref), lse_max=float(np.abs(lg - lse_ref).max()))
    assert stats["rrmse"] <= FP8_RRMSE, stats
    assert stats["lse_max"] <= (LSE_MAX_ABS if lse_bar is None else lse_bar), stats
    return stats


def compare_bf16(o_gpu, lse_gpu, o_ref, lse_ref):
    """o_gpu: [rows, d] (any float dtype), o_ref: [rows, d] float64."""
    og = o_gpu.to(torch.float64).numpy().reshape(o_ref.shape)
    lg = lse_gpu.to(torch.float64).numpy().reshape(lse_ref.shape)
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg))
    d = np.abs(og - o_ref)
    dl = np.abs(lg - lse_ref)
    stats = dict(max_abs=float(d.max()), mean_abs=float(d.mean()), lse_max=float(dl.max()))
    assert stats["max_abs"] <= BF16_MAX_ABS, stats
    assert stats["mean_abs"] <= BF16_MEAN_ABS, stats
    assert stats["lse_max"] <= LSE_MAX_ABS, stats
    return stats


def rrmse(o_gpu, o_ref):
    og = o_gpu.to(torch.float64).numpy().reshape(o_ref.shape)
    return float(np.linalg.norm(og - o_ref) / np.linalg.norm(o_ref))

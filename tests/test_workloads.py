"""The seeded input generator: determinism, shapes and the fp8 quantisation recipe."""
import torch

import workloads


def test_workload_table_shapes_and_flops():
    w = workloads.WORKLOADS
    assert (w["long"].B, w["long"].Hq, w["long"].N, w["long"].d) == (1, 32, 16384, 128)
    assert w["long"].flops == 4.0 * 32 * 16384 * 16384 * 128
    assert w["long_causal"].flops == w["long"].flops / 2
    assert (w["gqa_causal"].Hq, w["gqa_causal"].Hkv) == (32, 8)
    assert w["tiny"].out_dtype == "f32" and w["fp8"].in_dtype == "e4m3"
    assert w["gpt2"].scale == 0.125


def test_inputs_are_deterministic_and_seed_dependent():
    w = workloads.WORKLOADS["tiny"]
    a, b = workloads.make_inputs(w), workloads.make_inputs(w)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    c = workloads.make_inputs(w, seed=w.seed + 1)
    assert not torch.equal(a.q, c.q)
    assert a.q.dtype == torch.bfloat16 and a.q.shape == (1, 2, 256, 64)
    assert a.q.is_contiguous()


def test_fp8_per_head_amax_quantisation():
    w = workloads.WORKLOADS["fp8"]
    x = workloads.make_inputs(w, B=2, Hq=3, Hkv=3, Nq=512, Nk=512)
    for codes, ds in ((x.q, x.descale_q), (x.k, x.descale_k), (x.v, x.descale_v)):
        assert codes.dtype == torch.float8_e4m3fn and ds.shape == (6,)
        vals = codes.to(torch.float32).reshape(6, -1)
        # the largest magnitude of every (batch, head) slice maps onto the e4m3 maximum
        assert torch.all(vals.abs().amax(dim=1) == 448.0)
        # outliers (x50) push amax far above the N(0,1) bulk
        assert torch.all(ds * 448.0 > 10.0)

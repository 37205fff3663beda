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


def test_drift_inputs_move_the_scores_along_the_keys():
    """The drifting-score recipe: seeded, bf16, and each row's scores grow or shrink along
    the keys by far more than their spread within a block, so that on the rows that grow
    the online softmax's running maximum keeps moving."""
    a = workloads.drift_inputs(1, 2, 512, 64, seed=3)
    b = workloads.drift_inputs(1, 2, 512, 64, seed=3)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
    assert a.q.dtype == torch.bfloat16 and a.k.shape == (1, 2, 512, 64)
    s = torch.einsum("bhqd,bhkd->bhqk", a.q.float(), a.k.float())
    first, last = s[..., :64].mean(dim=-1), s[..., -64:].mean(dim=-1)
    spread = s[..., :64].std(dim=-1)
    # a trend well above the noise on nearly every row (a row nearly orthogonal to the
    # ramp's direction has little)
    assert ((last - first).abs() > 2 * spread).float().mean() > 0.9
    rising = (last > first).float().mean()
    assert 0.2 < rising < 0.8                             # both directions occur


def test_quantise_inputs_matches_the_fp8_recipe():
    """quantise_inputs_e4m3 applies the fp8 workload's own per-(batch, head) quantisation:
    the slice amax maps onto 448 and codes times descale give back the input within half a
    code step."""
    x = workloads.drift_inputs(1, 2, 256, 128, seed=4)
    y = workloads.quantise_inputs_e4m3(x)
    for src, codes, ds in ((x.q, y.q, y.descale_q), (x.k, y.k, y.descale_k), (x.v, y.v, y.descale_v)):
        vals = codes.to(torch.float32).reshape(2, -1)
        assert torch.all(vals.abs().amax(dim=1) == 448.0)
        back = vals * ds[:, None]
        err = (back - src.float().reshape(2, -1)).abs()
        # e4m3 has 3 mantissa bits: half a step is at most 1/16 of the magnitude (plus the
        # subnormal step near zero)
        bound = src.float().reshape(2, -1).abs() / 16 + ds[:, None] * 2.0 ** -9
        assert torch.all(err <= bound + 1e-6)

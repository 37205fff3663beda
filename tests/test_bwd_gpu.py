"""GPU parity of the backward pass (``fa_bwd``) against the fp64 gradient oracle.

The CUDA path runs the forward (fa_fwd: bf16 O and fp32 LSE) and then the backward on the
same seeded bf16 inputs; the oracle computes dQ, dK, dV from Q, K, V and dO alone.

Tolerance (per gradient tensor): the kernel rounds P and dS to bf16 for the tensor-core
products, takes D = rowsum(dO o O) from the bf16-rounded O, accumulates in fp32 and
rounds the results to bf16.  bf16's unit roundoff is u = 2^-8; a rounded value is off by
u/sqrt(3) (2.3e-3) in relative RMS, and the errors of the summed terms are independent,
so each gradient's relative RMS error should stay near 2.3e-3 (measured: 2.3e-3 to 2.7e-3).
The bar is rRMSE <= 1e-2 and max |error| <= 2e-2 * max |reference|.
"""
import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
import oracle
from workloads import random_bf16

pytestmark = pytest.mark.gpu

RRMSE_BAR = 1e-2
MAX_REL_BAR = 2e-2


def run_fwd_bwd(q, k, v, do, causal, scale):
    dev = torch.device("cuda", 0)
    q, k, v, do = (t.to(dev) for t in (q, k, v, do))
    o, lse = fa.forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    return dq.cpu(), dk.cpu(), dv.cpu()


def errors(got, ref, natural):
    """(relative RMS error, max error / max |ref|), each normalised by at least 1e-3 of
    the gradient's natural magnitude (a gradient can vanish exactly, e.g. dQ and dK with a
    single key, where only rounding noise is left to compare)."""
    g = got.to(torch.float64).numpy()
    d = g - ref
    floor = 1e-3 * natural
    return (float(np.linalg.norm(d) / max(np.linalg.norm(ref), floor * np.sqrt(ref.size))),
            float(np.abs(d).max() / max(np.abs(ref).max(), floor)))


def check(shape, causal, seed=0, scale=None, d=128):
    B, Hq, Hkv, Nq, Nk = shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    scale = float(torch.tensor(scale, dtype=torch.float32))
    q = random_bf16((B, Hq, Nq, d), seed + 1)
    k = random_bf16((B, Hkv, Nk, d), seed + 2)
    v = random_bf16((B, Hkv, Nk, d), seed + 3)
    do = random_bf16((B, Hq, Nq, d), seed + 4)
    got = run_fwd_bwd(q, k, v, do, causal, scale)
    ref = oracle.attention_bwd(q, k, v, do, scale, causal)
    mx = lambda t: float(t.float().abs().max())
    # |dS| <= |dP| + |D| <= 2 |dO| |V| d, so these bound each gradient up to a factor of d
    natural = {"dq": scale * mx(do) * mx(v) * mx(k), "dk": scale * mx(do) * mx(v) * mx(q),
               "dv": mx(do)}
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert torch.isfinite(g.float()).all(), name
        rr, mr = errors(g, r, natural[name])
        out[name] = (rr, mr)
        assert rr <= RRMSE_BAR and mr <= MAX_REL_BAR, (name, rr, mr)
    return out


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [
    (1, 1, 1, 1, 1), (1, 2, 2, 64, 64), (1, 2, 2, 128, 128), (1, 2, 1, 200, 200),
    (2, 4, 2, 333, 333), (1, 4, 1, 1000, 1000), (1, 2, 2, 513, 513),
])
def test_gradients_match_oracle(cuda_ok, shape, causal):
    print(shape, causal, check(shape, causal))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 2, 100, 300), (1, 2, 1, 300, 77), (1, 2, 2, 129, 513),
                                   (2, 4, 2, 513, 129), (1, 1, 1, 1, 700), (1, 2, 1, 700, 1)])
def test_gradients_non_square(cuda_ok, shape, causal):
    """Nq != Nk; under the causal mask aligned at the bottom right, so with Nq > Nk the
    first Nq - Nk query rows admit no key (zero dQ rows)."""
    print(shape, causal, check(shape, causal))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [
    (1, 1, 1, 1, 1), (1, 2, 2, 64, 64), (1, 2, 1, 200, 200), (2, 4, 2, 333, 333),
    (1, 4, 1, 1000, 1000),
])
def test_gradients_head_dim_64(cuda_ok, shape, causal):
    """d = 64: one 128-byte box per row; the dQ^T product runs on a zero-padded K^T."""
    print(shape, causal, check(shape, causal, seed=7, d=64))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 2, 100, 300), (1, 4, 2, 300, 77)])
def test_gradients_head_dim_64_non_square(cuda_ok, shape, causal):
    print(shape, causal, check(shape, causal, seed=9, d=64))


def test_gradients_larger_scores(cuda_ok):
    """A larger scale sharpens the softmax (fewer keys carry the weight)."""
    print(check((1, 2, 2, 256, 256), True, seed=5, scale=0.5))


def test_dk_dv_deterministic(cuda_ok):
    B, H, N, d = 1, 4, 700, 128
    t = [random_bf16((B, H, N, d), 40 + s) for s in range(4)]
    a = run_fwd_bwd(*t, True, 0.088)
    b = run_fwd_bwd(*t, True, 0.088)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dQ is summed with atomics: equal up to the order of fp32 additions
    assert (a[0].float() - b[0].float()).abs().max() <= 1e-2 * a[0].float().abs().max()


@pytest.mark.parametrize("shape", [(1, 8, 8, 16384, 128), (16, 12, 12, 2048, 64)],
                         ids=["long_h8", "gpt2"])
@pytest.mark.parametrize("causal", [False, True])
def test_full_size_gradient_identities(cuda_ok, causal, shape):
    """At the long-context size and the GPT-2 backward workload's size (d = 64), too large
    for the full oracle, check what holds for any input: sum_j dV_j = sum_i dO_i, and
    sum_j dK_j = 0 (rows of dS sum to zero).

    Error budget (u = 2^-8), per component (head, t): in the dV identity the bf16
    rounding of the summed rows gives about u/sqrt(3) * sqrt(sum_j dV_jt^2), and rounding
    P makes each row of P sum to 1 only within u, which adds at most about
    u * sqrt(sum_i dO_it^2); the bound takes 4u times the sum of the two.  (Under the
    causal mask a few early keys carry large dV, so the root of the sum of squares, not the
    mean magnitude, sets the scale.)  In the dK identity the rounding of O inside D_i shifts
    the whole dS row i by the same amount, so the errors do not average over keys: the sum
    is off by about scale * u * sqrt(N) * rms(O) rms(dO) sqrt(d) rms(q) per component;
    the bound takes 6 times that (the maximum over all components, and margin).  rms(O) is
    taken from 64 oracle rows per head."""
    B, Hq, Hkv, N, d = shape
    scale = float(torch.tensor(1.0 / np.sqrt(d), dtype=torch.float32))
    q, k, v, do = (random_bf16((B, Hq if s in (0, 3) else Hkv, N, d), 50 + s)
                   for s in range(4))
    dq, dk, dv = run_fwd_bwd(q, k, v, do, causal, scale)
    u = 2.0 ** -8
    dsum = do.double().sum(dim=2)                        # [B, H, d]
    err_v = (dv.double().sum(dim=2) - dsum).abs()
    bound_v = 4 * u * (dv.double().square().sum(dim=2).sqrt() + do.double().square().sum(dim=2).sqrt())
    assert bool((err_v <= bound_v).all()), (err_v.max().item(), bound_v.min().item())
    err_v, bound_v = err_v.max().item(), (err_v / bound_v).max().item()
    rows = (np.arange(B * Hq)[:, None] * N
            + np.random.default_rng(0).integers(0, N, size=(B * Hq, 64))).reshape(-1)
    o_rows, _ = oracle.attention_rows(q, k, v, scale, causal, rows=rows)
    rms = lambda t: float(np.sqrt(np.mean(np.square(t))))
    bound_k = 6 * scale * u * np.sqrt(N) * rms(o_rows) * rms(do.double().numpy()) * np.sqrt(d) \
        * rms(q.double().numpy())
    err_k = dk.double().sum(dim=2).abs().max().item()
    assert err_k <= bound_k, (err_k, bound_k)
    print("identities: dV %.3g (largest error / bound %.2f), dK %.3g (bound %.3g)"
          % (err_v, bound_v, err_k, bound_k))
    assert torch.isfinite(dq.float()).all()

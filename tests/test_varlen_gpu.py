"""GPU parity of variable-length (packed, cu_seqlens) attention and of causal attention with
Nq != Nk (bottom-right alignment) against the fp64 oracle, sequence by sequence.

Variable sequence lengths batch sequences of different length without padding (page
"FlashAttention 4: Praxisleitfaden ...", section "Kompatibilitaet und aktueller Stand").
Rows without any admissible key (causal with more queries than keys, or no keys at all)
must come out as O = 0 and LSE = -inf.
"""
import numpy as np
import pytest
import torch

import exact_attention_101_b200 as fa
import oracle
from parity_util import compare_bf16
from workloads import random_bf16

pytestmark = pytest.mark.gpu

D_SCALE = {64: 0.125, 128: float(torch.tensor(1 / np.sqrt(128), dtype=torch.float32)),
           256: 0.0625}


def packed(lengths, H, d, seed):
    total = int(sum(lengths))
    return random_bf16((max(total, 1), H, d), seed)[:total].contiguous()


def cu(lengths):
    return torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)


def check_rows(o_gpu, lse_gpu, o_ref, lse_ref):
    """Rows with keys: bf16 tolerances.  Rows without: O = 0, LSE = -inf exactly."""
    empty = np.isneginf(lse_ref)
    lg = lse_gpu.double().numpy()
    assert np.all(np.isneginf(lg[empty])), "rows without keys must have LSE = -inf"
    assert np.all(o_gpu.double().numpy()[empty] == 0.0), "rows without keys must have O = 0"
    if (~empty).any():
        return compare_bf16(o_gpu[torch.from_numpy(~empty)], lse_gpu[torch.from_numpy(~empty)],
                            o_ref[~empty], lse_ref[~empty])
    return {}


def run_varlen_case(lq, lk, Hq, Hkv, d, causal, seed, out_dtype=torch.bfloat16):
    dev = torch.device("cuda", 0)
    q, k, v = packed(lq, Hq, d, seed), packed(lk, Hkv, d, seed + 1), packed(lk, Hkv, d, seed + 2)
    cq, ck = cu(lq), cu(lk)
    scale = D_SCALE[d]
    o, lse = fa.forward_varlen(q.to(dev), k.to(dev), v.to(dev), cq.to(dev), ck.to(dev),
                               max(max(lq), 1), causal=causal, scale=scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    o, lse = o.cpu(), lse.cpu()
    stats = []
    for b in range(len(lq)):
        if lq[b] == 0:
            continue
        qs = q[cq[b]:cq[b + 1]].transpose(0, 1).unsqueeze(0).contiguous()
        if lk[b] == 0:   # no keys at all: every row is empty
            assert torch.all(o[cq[b]:cq[b + 1]] == 0) and torch.isneginf(lse[:, cq[b]:cq[b + 1]]).all()
            continue
        ks = k[ck[b]:ck[b + 1]].transpose(0, 1).unsqueeze(0).contiguous()
        vs = v[ck[b]:ck[b + 1]].transpose(0, 1).unsqueeze(0).contiguous()
        ro, rl = oracle.attention(qs, ks, vs, scale, causal)
        go = o[cq[b]:cq[b + 1]].transpose(0, 1)           # [Hq, len, d]
        gl = lse[:, cq[b]:cq[b + 1]]                     # [Hq, len]
        stats.append(check_rows(go.reshape(-1, d), gl.reshape(-1), ro[0].reshape(-1, d),
                                rl[0].reshape(-1)))
    return stats


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_varlen_self_attention(cuda_ok, d, causal):
    lengths = [1, 17, 128, 129, 256, 300, 511, 64, 1000]
    print(run_varlen_case(lengths, lengths, 4, 2, d, causal, seed=100 + d))


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_cross_lengths_and_empty_sequences(cuda_ok, causal):
    lq = [5, 0, 300, 70, 257, 3]
    lk = [9, 4, 100, 0, 600, 3]
    print(run_varlen_case(lq, lk, 2, 1, 128, causal, seed=200))


def test_varlen_fp32_output(cuda_ok):
    print(run_varlen_case([33, 190, 700], [33, 190, 700], 2, 2, 128, True, seed=300,
                          out_dtype=torch.float32))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_varlen_equal_lengths_equal_fixed_length(cuda_ok, causal, d):
    """Packed sequences of one length against the [B, H, N, d] path.  Where both run the
    same tiles of the one-CTA kernel (head dim 64, and 128 under the causal mask): equal
    bits.  Elsewhere the fixed-length path runs the CTA-pair kernel (another summation
    order): equal within the bf16 bar."""
    dev = torch.device("cuda", 0)
    B, H, N = 3, 4, 385
    q, k, v = (random_bf16((B, H, N, d), 400 + s) for s in range(3))
    o1, l1 = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=D_SCALE[d])
    pk = lambda t: t.permute(0, 2, 1, 3).reshape(B * N, H, d).contiguous().to(dev)
    c = cu([N] * B).to(dev)
    o2, l2 = fa.forward_varlen(pk(q), pk(k), pk(v), c, c, N, causal=causal, scale=D_SCALE[d])
    torch.cuda.synchronize()
    o1 = o1.permute(0, 2, 1, 3).reshape(B * N, H, d)
    l1 = l1.permute(1, 0, 2).reshape(H, B * N)
    if d == 64 or (d == 128 and causal):
        assert torch.equal(o1, o2)
        assert torch.equal(l1, l2)
    else:
        e = (o1.float() - o2.float()).abs()
        assert e.max().item() <= 2e-2 and e.mean().item() <= 2e-3
        assert (l1 - l2).abs().max().item() <= 1e-3


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("nq,nk", [(100, 300), (300, 100), (129, 513), (513, 129), (1, 700)])
def test_fixed_length_causal_bottom_right(cuda_ok, nq, nk, d):
    """Head dim 128 runs the one-CTA kernel under the mask, 256 the CTA-pair kernel."""
    dev = torch.device("cuda", 0)
    B, Hq, Hkv = 1, 4, 2
    q = random_bf16((B, Hq, nq, d), 500)
    k, v = random_bf16((B, Hkv, nk, d), 501), random_bf16((B, Hkv, nk, d), 502)
    o, lse = fa.forward(q.to(dev), k.to(dev), v.to(dev), causal=True, scale=D_SCALE[d])
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    ro, rl = oracle.attention(q, k, v, D_SCALE[d], True)
    print(check_rows(o.cpu().reshape(-1, d), lse.cpu().reshape(-1), ro.reshape(-1, d),
                     rl.reshape(-1)))


def test_varlen_full_size_sampled(cuda_ok):
    """The varlen benchmark workload at full size (16 sequences of 256 .. 8192 tokens,
    H = 32, d = 128, causal) in the bench's launch configuration; rows sampled from the
    shortest, the longest and a middle sequence (first, last and random rows of two heads
    each) against the oracle on that sequence alone."""
    import workloads
    w = workloads.WORKLOADS["varlen_causal"]
    inp = workloads.make_inputs(w)
    lens = workloads.varlen_lengths(w)
    dev = torch.device("cuda", 0)
    cu_d = inp.cu_seqlens.to(dev)
    o, lse = fa.forward_varlen(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), cu_d, cu_d,
                               max(lens), causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_check_device_error(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    o, lse = o.cpu(), lse.cpu()
    order = np.argsort(lens)
    rng = np.random.default_rng(w.seed)
    for b in (int(order[0]), int(order[len(order) // 2]), int(order[-1])):
        t0, n = int(inp.cu_seqlens[b]), lens[b]
        seq = lambda t: t[t0:t0 + n].transpose(0, 1).unsqueeze(0).contiguous()  # [1, H, n, d]
        heads = [0, w.Hq - 1]
        idx = sorted(set([0, 1, 127, 128, n // 2, n - 2, n - 1])
                     | set(int(x) for x in rng.integers(0, n, size=48)))
        rows = np.array([h * n + i for h in heads for i in idx])
        ro, rl = oracle.attention_rows(seq(inp.q), seq(inp.k), seq(inp.v), w.scale, w.causal,
                                       rows=rows)
        go = torch.stack([o[t0 + i, h] for h in heads for i in idx])
        gl = torch.stack([lse[h, t0 + i] for h in heads for i in idx])
        print(b, n, compare_bf16(go, gl, ro, rl))

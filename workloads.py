"""Seeded synthetic workloads for the attention forward pass.

This module only draws inputs.  It holds none of the attention arithmetic, so that both
the CUDA library (through the tests and ``bench.py``) and the CPU oracle can be fed the
same bytes.  Every tensor is drawn on the CPU from a ``torch.Generator`` seeded per
workload, in a fixed order (Q, then K, then V, then -- fp8 only -- the outlier masks),
and stored contiguous in [batch, heads, sequence, head_dim] order.

The shapes are the five workloads the attention pages motivate: a tiny case, a
GPT-2-small-shaped case (batch 16, 12 heads, 2048 tokens: the shape the "Flash
Attention" page uses for its memory comparison in "Performance-Benchmarks"), a 16K-token
long-context case (same page: 16K-token training), a grouped-query case (4 query heads
per K/V head) and an fp8-e4m3 case with sparse large-magnitude entries (the outliers
that the page "FlashAttention-3 (DE)" names as the risk of FP8 quantisation, section
"Niedrige Praezision (FP8) mit reduziertem Quantisierungsfehler").  None of the pages
benchmarks on a public dataset, so the values are i.i.d. standard normal.

Two workloads with head dimension 256 (FA2's largest, page "Flash Attention", section on
the versions) keep the long workload's FLOPs with 16 heads.  Two more workloads feed the
incoherent processing of that section (``rotate=True``):
bf16 Q/K/V with the fp8 case's outliers, or with a few outlier channels shared by Q and
K, that the library quantises itself after a random-sign Hadamard rotation of Q and K.
Their sign vector is drawn here, after the values, and passed to the library as input.
Backward workloads (``kind="bwd"``) use the forward shapes and draw the upstream gradient
dO after V, i.i.d. N(0, 1) in bf16.  The variable-length workload (``kind="varlen"``)
packs B sequences whose lengths are drawn uniformly (the pages give no length mix) into
token-major tensors with cu_seqlens offsets.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    in_dtype: str          # "bf16" or "e4m3"
    out_dtype: str         # "bf16" or "f32"
    seed: int
    outlier_rate: float = 0.0
    outlier_scale: float = 1.0
    outlier_kind: str = "entry"   # "entry": i.i.d. entries of Q, K, V; "channel": whole
    #                               channels of Q and K (outlier_channels of them)
    outlier_channels: int = 0
    rotate: bool = False          # bf16 source quantised on the GPU with Hadamard rotation
    kind: str = "fwd"             # "fwd": forward pass; "bwd": backward pass (dO drawn too);
    #                               "varlen": B packed sequences of lengths drawn in
    #                               [min_len, N] (token-major [tokens, H, d] tensors)
    min_len: int = 0
    dropout: float = 0.0          # dropout probability on the attention weights (fwd)

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d), rounded to fp32 (the value both sides receive)."""
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32))

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: forward 4*B*Hq*Nq*Nk*d (two products), backward 2.5 times
        that (five products); halved under the causal mask.  Variable lengths: the sum of
        4*Hq*len^2*d over the sequences."""
        if self.kind == "varlen":
            f = sum(4.0 * self.Hq * n * n * self.d for n in varlen_lengths(self))
            return f / 2 if self.causal else f
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        if self.kind == "bwd":
            f *= 2.5
        return f / 2 if self.causal else f

    def describe(self) -> Dict[str, object]:
        out = {"workload": self.name, "B": self.B, "Hq": self.Hq, "Hkv": self.Hkv,
               "Nq": self.N, "Nk": self.N, "d": self.d, "causal": self.causal,
               "in_dtype": self.in_dtype, "out_dtype": self.out_dtype,
               "seed": self.seed}
        if self.rotate:
            out["quantise"] = "e4m3 per head on the GPU, Q and K after random-sign Hadamard"
        if self.kind == "bwd":
            out["pass"] = "backward (dQ, dK, dV from Q, K, V, O, LSE, dO)"
        if self.dropout:
            out["dropout"] = self.dropout
        if self.kind == "varlen":
            lens = varlen_lengths(self)
            out.update({"Nq": None, "Nk": None, "sequences": self.B, "total_tokens": sum(lens),
                        "lengths": "uniform integers in [%d, %d], seeded" % (self.min_len, self.N),
                        "layout": "packed [tokens, H, d] with cu_seqlens"})
        return out


WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    Workload("tiny", 1, 2, 2, 256, 64, False, "bf16", "f32", 1001),
    Workload("gpt2", 16, 12, 12, 2048, 64, False, "bf16", "bf16", 1002),
    Workload("gpt2_causal", 16, 12, 12, 2048, 64, True, "bf16", "bf16", 1002),
    Workload("long_causal", 1, 32, 32, 16384, 128, True, "bf16", "bf16", 1003),
    Workload("long", 1, 32, 32, 16384, 128, False, "bf16", "bf16", 1003),
    Workload("gqa_causal", 4, 32, 8, 8192, 128, True, "bf16", "bf16", 1004),
    Workload("fp8", 8, 16, 16, 4096, 128, False, "e4m3", "bf16", 1005, 1e-3, 50.0),
    Workload("fp8_incoherent", 8, 16, 16, 4096, 128, False, "bf16", "bf16", 1006, 1e-3, 50.0,
             rotate=True),
    Workload("fp8_incoherent_channels", 8, 16, 16, 4096, 128, False, "bf16", "bf16", 1007,
             1.0, 10.0, outlier_kind="channel", outlier_channels=4, rotate=True),
    Workload("varlen_causal", 16, 32, 32, 8192, 128, True, "bf16", "bf16", 1008, kind="varlen",
             min_len=256),
    Workload("long_dropout", 1, 32, 32, 16384, 128, False, "bf16", "bf16", 1003, dropout=0.1),
    Workload("long_d256", 1, 16, 16, 16384, 256, False, "bf16", "bf16", 1009),
    Workload("long_d256_causal", 1, 16, 16, 16384, 256, True, "bf16", "bf16", 1009),
    Workload("long_bwd", 1, 32, 32, 16384, 128, False, "bf16", "bf16", 1003, kind="bwd"),
    Workload("long_causal_bwd", 1, 32, 32, 16384, 128, True, "bf16", "bf16", 1003, kind="bwd"),
    Workload("gqa_causal_bwd", 4, 32, 8, 8192, 128, True, "bf16", "bf16", 1004, kind="bwd"),
    Workload("gpt2_bwd", 16, 12, 12, 2048, 64, False, "bf16", "bf16", 1002, kind="bwd"),
    Workload("gpt2_causal_bwd", 16, 12, 12, 2048, 64, True, "bf16", "bf16", 1002, kind="bwd"),
]}


@dataclasses.dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    descale_q: Optional[torch.Tensor] = None   # fp32 [B*Hq]   (e4m3 only)
    descale_k: Optional[torch.Tensor] = None   # fp32 [B*Hkv]
    descale_v: Optional[torch.Tensor] = None   # fp32 [B*Hkv]
    signs: Optional[torch.Tensor] = None       # int8 [d] of +-1 (rotate workloads only)
    cu_seqlens: Optional[torch.Tensor] = None  # int32 [B+1] (varlen workloads only)
    dout: Optional[torch.Tensor] = None        # bf16 [B, Hq, Nq, d] (backward workloads only)


def _quantise_e4m3_per_head(x: torch.Tensor):
    """Per-(batch, head) amax scaling into OCP e4m3: s = amax/448, code = e4m3(x/s).

    Returns (codes as torch.float8_e4m3fn, descale s as fp32 [B*H]).  The cast is
    torch's round-to-nearest-even; the clamp keeps x/s inside the finite range.
    """
    B, H = x.shape[:2]
    amax = x.abs().amax(dim=(2, 3)).to(torch.float32)
    s = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / s[:, :, None, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).contiguous(), s.reshape(B * H).contiguous()


def varlen_lengths(w: Workload):
    """Sequence lengths of a varlen workload: B uniform integers in [min_len, N], from their
    own generator seeded with the workload seed."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    return [int(n) for n in torch.randint(w.min_len, w.N + 1, (w.B,), generator=g)]


def make_inputs(w: Workload, seed: Optional[int] = None, *, B: Optional[int] = None,
                Hq: Optional[int] = None, Hkv: Optional[int] = None,
                Nq: Optional[int] = None, Nk: Optional[int] = None,
                d: Optional[int] = None) -> Inputs:
    """Draw the inputs of workload ``w`` (shape overrides give smaller variants with the
    same value distribution)."""
    B = w.B if B is None else B
    Hq = w.Hq if Hq is None else Hq
    Hkv = w.Hkv if Hkv is None else Hkv
    Nq = w.N if Nq is None else Nq
    Nk = w.N if Nk is None else Nk
    d = w.d if d is None else d
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    if w.kind == "varlen":
        lens = varlen_lengths(w)
        total = sum(lens)
        q = torch.randn((total, Hq, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
        k = torch.randn((total, Hkv, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
        v = torch.randn((total, Hkv, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
        cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0)), dtype=torch.int32)
        return Inputs(q, k, v, cu_seqlens=cu)
    q32 = torch.randn((B, Hq, Nq, d), generator=g, dtype=torch.float32)
    k32 = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    v32 = torch.randn((B, Hkv, Nk, d), generator=g, dtype=torch.float32)
    if w.outlier_kind == "channel":
        channels = torch.randperm(d, generator=g)[:w.outlier_channels]
        q32[..., channels] *= w.outlier_scale
        k32[..., channels] *= w.outlier_scale
    elif w.outlier_rate > 0:
        for t in (q32, k32, v32):
            mask = torch.rand(t.shape, generator=g) < w.outlier_rate
            t[mask] *= w.outlier_scale
    if w.in_dtype == "bf16":
        inp = Inputs(q32.to(torch.bfloat16), k32.to(torch.bfloat16), v32.to(torch.bfloat16))
        if w.rotate:
            inp.signs = torch.where(torch.rand(d, generator=g) < 0.5, -1, 1).to(torch.int8)
        if w.kind == "bwd":
            inp.dout = torch.randn((B, Hq, Nq, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
        return inp
    if w.in_dtype != "e4m3":
        raise ValueError(w.in_dtype)
    q8, dq = _quantise_e4m3_per_head(q32)
    k8, dk = _quantise_e4m3_per_head(k32)
    v8, dv = _quantise_e4m3_per_head(v32)
    return Inputs(q8, k8, v8, dq, dk, dv)


def random_bf16(shape, seed: int) -> torch.Tensor:
    """Standard-normal bf16 tensor from a seeded generator (for ad-hoc test shapes)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def drift_inputs(B: int, H: int, N: int, d: int, seed: int, drift: float = 12.0) -> Inputs:
    """Scores that drift along the keys, so that the running row maximum keeps rising and
    the online softmax has to rescale again and again: Q i.i.d. N(0, 1); K = 0.2 N(0, 1)
    plus a ramp from 0 to `drift` along the keys times the sign of Q's mean over the rows
    (per head and dimension), so each row's scores grow or shrink linearly; V i.i.d.
    N(0, 1).  Drawn in the order Q, K noise, V; returned in bf16."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, H, N, d), generator=g)
    k = torch.randn((B, H, N, d), generator=g) * 0.2
    k += torch.linspace(0, drift, N)[None, None, :, None] * q.mean(dim=2, keepdim=True).sign()
    v = torch.randn((B, H, N, d), generator=g)
    return Inputs(q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def quantise_inputs_e4m3(inp: Inputs) -> Inputs:
    """The fp8 path's per-(batch, head) amax quantisation of bf16 inputs (codes and
    descales), the recipe of the fp8 workload."""
    out = {}
    for name in ("q", "k", "v"):
        codes, ds = _quantise_e4m3_per_head(getattr(inp, name).float())
        out[name], out["descale_" + name] = codes, ds
    return Inputs(out["q"], out["k"], out["v"], out["descale_q"], out["descale_k"],
                  out["descale_v"])

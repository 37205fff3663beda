"""Throughput benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one ``fa_fwd`` call over the whole workload (scheduler, TMA loads, S = QK^T,
masked online softmax with lazy rescaling, O += PV, epilogue).  The default workload is
the long-context non-causal case (B=1, H=32, N=16384, d=128, bf16), whose Q/K/V (402 MB)
exceed the 126 MB L2, so no flush is needed between steps.  Rank 0 prints one JSON line.

With N > 1 (launched by torchrun) every rank runs its own copy of the workload on its own
GPU with its own seed -- the (batch, head) units are independent, so the work shards with
no exchange step and no collective on the data path (weak scaling); the only
collectives are the timing barrier and the max over ranks of the elapsed time.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same workload
(rank 0 only) and prints the same line with ``"impl": "reference"``.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "attention fwd TFLOP/s on 1 B200 and % of dense tensor peak (causal halved)"
UNIT = "TFLOP/s"
DATASHEET_BF16_TFLOPS = 2250.0
DATASHEET_FP8_TFLOPS = 4500.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ["exact_attention_101_b200/csrc/fa_fwd_kernel.cuh",
                  "exact_attention_101_b200/csrc/fa_fwd_pair.cuh",
                  "exact_attention_101_b200/csrc/sm100.cuh",
                  "exact_attention_101_b200/csrc/fa_api.cu"]


# ------------------------------------------------------------------ host-side helpers

def uses_pair_kernel(w, fp8):
    """Whether the library runs this forward workload on its CTA-pair kernel (bf16 without
    dropout at head dim 256, and at 128 without the causal mask), as fa_api.cu's pair_path
    decides."""
    return (w.kind == "fwd" and not fp8 and not w.dropout
            and (w.d == 256 or (w.d == 128 and not w.causal)))


def rank_env():
    """(rank, local_rank, world_size) from the torchrun environment (defaults 0, 0, 1)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def rank_seed(w, rank):
    """Each rank draws its own batch: weak scaling over independent problems."""
    return w.seed + 7919 * rank


def max_over_ranks(value_ms, world_size, device=None):
    """Max of a per-rank elapsed time over all ranks (the job is as slow as its slowest
    rank).  Uses the default process group when world_size > 1."""
    if world_size <= 1:
        return float(value_ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def load_fp8_peak():
    """Measured dense e4m3 GEMM peak (TFLOP/s) from profiles/fp8_peak.json, if present."""
    try:
        with open(os.path.join(ROOT, "profiles", "fp8_peak.json")) as f:
            return float(json.load(f)["e4m3_tflops"])
    except (OSError, ValueError, KeyError):
        return None


def measure_fp8_peak():
    """Dense e4m3 GEMM throughput of torch._scaled_mm (8192^3, bf16 out), measured the way
    MEASURED_PEAKS.json measures bf16: best of 10 (burst) and back to back for 4 s
    (sustained).  Prints one JSON line."""
    import torch
    dev = torch.device("cuda", 0)
    n = 8192
    g = torch.Generator(device=dev).manual_seed(0)
    a = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn)
    bt = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev, dtype=torch.float32)
    mm = lambda: torch._scaled_mm(a, bt.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    reps, t0 = 0, time.perf_counter()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    while time.perf_counter() - t0 < 4.0:
        for _ in range(20):
            mm()
        reps += 20
        torch.cuda.synchronize()
    e1.record()
    torch.cuda.synchronize()
    flop = 2.0 * n ** 3
    print(json.dumps({"e4m3_tflops": flop / best / 1e9,
                      "e4m3_tflops_sustained": flop * reps / e0.elapsed_time(e1) / 1e9,
                      "how": "torch._scaled_mm e4m3 x e4m3 -> bf16, 8192^3, unit scales: best "
                             "of 10 (burst) and back to back for 4 s (sustained), CUDA events",
                      "gpu": torch.cuda.get_device_name(0), "torch": torch.__version__}))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_sha():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(workload_name)
    if not e or e.get("kernel_source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock, power and throttle reasons of this rank's GPU while the timed region runs.

    Polls NVML (the library nvidia-smi reads) every ~2 ms on a thread; begin()/end() mark the
    timed window on the host clock and stop() summarises the samples inside it, so that even a
    timed region of a few tens of milliseconds is described by samples taken under load.
    Without NVML it falls back to nvidia-smi at its 100 ms interval (whole run)."""

    SMI_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, gpu_index, device=None):
        self.gpu = gpu_index
        self.device = device
        self.samples = []          # (host time, sm MHz, reason bits, power W)
        self.window = [None, None]
        self.stop_flag = False
        self.thread = None
        self.proc = None
        self.lines = []
        self.nvml = None
        self.handle = None
        self.max_mhz = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        handle = None
        try:  # NVML numbers all GPUs; match this rank's CUDA device by its PCI bus id
            import torch
            props = torch.cuda.get_device_properties(self.device if self.device is not None
                                                     else self.gpu)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id,
                                        props.pci_device_id)
            handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            handle = pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu))
        return pynvml, handle

    def start(self):
        try:
            self.nvml, self.handle = self._nvml_handle()
            self.max_mhz = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle,
                                                                    self.nvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.SMI_QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _poll(self):
        nv, h = self.nvml, self.handle
        while not self.stop_flag:
            try:
                self.samples.append((time.perf_counter(),
                                     float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                     int(nv.nvmlDeviceGetCurrentClocksEventReasons(h)),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1e3))
            except Exception:
                return
            time.sleep(0.002)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def begin(self):
        self.window[0] = time.perf_counter()

    def end(self):
        self.window[1] = time.perf_counter()

    def stop(self):
        if self.nvml is not None:
            time.sleep(0.005)
            self.stop_flag = True
            self.thread.join(timeout=2)
            lo, hi = self.window
            inside = [x for x in self.samples
                      if (lo is None or x[0] >= lo) and (hi is None or x[0] <= hi)]
            if not inside and self.samples and lo is not None:  # window shorter than a poll
                inside = [min(self.samples, key=lambda x: abs(x[0] - lo))]
            if not inside:
                return None
            reasons = sorted(n for n, bit in self.REASONS if any(x[2] & bit for x in inside))
            sm = [x[1] for x in inside]
            return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm),
                    "sm_max_mhz": self.max_mhz, "reasons": reasons,
                    "power_w": round(statistics.median(x[3] for x in inside), 1),
                    "samples": len(inside), "source": "nvml, 2 ms, timed window only"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = [n for n, _ in self.REASONS]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, flag in zip(names, f[5:9]):
                if flag.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvidia-smi, 100 ms, whole run"}


# ------------------------------------------------------------------ CPU oracle timing

def _oracle_kwargs(inp):
    if inp.descale_q is None:
        return {}
    return dict(descale_q=inp.descale_q.double(), descale_k=inp.descale_k.double(),
                descale_v=inp.descale_v.double())


def _row_flops(w, rows):
    i = rows % w.N
    keys = (i + 1) if w.causal else (i * 0 + w.N)
    return float(4.0 * w.d * keys.sum())


def oracle_calibrate(w, inp, target_s, seed=0):
    """Number of random query rows the fp64 oracle processes in about target_s seconds."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    total_rows = w.B * w.Hq * w.N
    n = 16
    while True:
        rows = rng.integers(0, total_rows, size=n)
        t0 = time.perf_counter()
        oracle.attention_rows(inp.q, inp.k, inp.v, w.scale, w.causal, rows=rows,
                              **_oracle_kwargs(inp))
        dt = time.perf_counter() - t0
        if dt >= 0.5 * target_s or n >= total_rows:
            return int(min(total_rows, max(16, n * target_s / max(dt, 1e-4))))
        n = int(min(total_rows, 4 * n))


def oracle_timed_sample(w, inp, n_rows, seed=0):
    """Time the fp64 oracle on n_rows random query rows of the workload.  Returns
    (TFLOP/s, description, threads, seconds)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    total_rows = w.B * w.Hq * w.N
    rows = rng.integers(0, total_rows, size=n_rows)
    t0 = time.perf_counter()
    if w.dropout:
        oracle.attention_dropout_rows(inp.q, inp.k, inp.v, w.scale, w.causal,
                                      min(255, round(256 * w.dropout)), w.seed, 0, rows=rows)
    else:
        oracle.attention_rows(inp.q, inp.k, inp.v, w.scale, w.causal, rows=rows,
                              **_oracle_kwargs(inp))
    dt = time.perf_counter() - t0
    desc = ("%d random query rows (of %d) of workload %s, each over its full admissible key "
            "range, fp64" % (n_rows, total_rows, w.name))
    if w.rotate:
        desc += (" (attention over the bf16 source values; the oracle's quantisation, about "
                 "%.1f%% of its work at this shape, is not timed)" % (100.0 * w.d / w.N / 2))
    return _row_flops(w, rows) / dt / 1e12, desc, oracle.max_threads(), dt


def oracle_bwd_sample(w, inp, target_s):
    """Time the fp64 gradient oracle on the first n queries and keys of the first K/V head
    and its query heads (n doubled until the run takes at least a quarter of target_s).
    Returns (TFLOP/s, description, threads, seconds)."""
    import oracle
    g = w.Hq // w.Hkv
    n, dt = 256, 0.0
    while True:
        sl = lambda t, h: t[:1, :h, :n].contiguous()
        t0 = time.perf_counter()
        oracle.attention_bwd(sl(inp.q, g), sl(inp.k, 1), sl(inp.v, 1), sl(inp.dout, g), w.scale,
                             w.causal)
        dt = time.perf_counter() - t0
        if dt >= 0.25 * target_s or 2 * n > w.N:
            break
        n *= 2
    flops = 2.5 * 4.0 * g * n * n * w.d / (2 if w.causal else 1)
    desc = ("gradients of the first %d queries and keys of batch 0, K/V head 0 and its %d "
            "query head(s) of workload %s, fp64" % (n, g, w.name))
    return flops / dt / 1e12, desc, oracle.max_threads(), dt


def oracle_varlen_sample(w, inp, target_s, seed=0):
    """Time the fp64 oracle on random (sequence, head, query) rows of a varlen workload,
    drawing rows until about target_s of oracle time.  Returns (TFLOP/s, description,
    threads, seconds)."""
    import numpy as np
    import torch
    import oracle
    rng = np.random.default_rng(seed)
    cu = inp.cu_seqlens.tolist()
    flops, dt, rows = 0.0, 0.0, 0
    while dt < target_s:
        b = int(rng.integers(0, w.B))
        n = cu[b + 1] - cu[b]
        # bf16 bits as numpy, prepared outside the timed call
        seq = lambda t: t[cu[b]:cu[b + 1]].transpose(0, 1).unsqueeze(0).contiguous().view(
            torch.int16).numpy()
        q, k, v = seq(inp.q), seq(inp.k), seq(inp.v)
        r = rng.integers(0, w.Hq * n, size=256)
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, w.scale, w.causal, rows=r)
        dt += time.perf_counter() - t0
        keys = (r % n + 1) if w.causal else np.full(r.shape, n)
        flops += 4.0 * w.d * float(keys.sum())
        rows += len(r)
    desc = ("%d random (sequence, head, query) rows of workload %s, each over its admissible "
            "keys, fp64" % (rows, w.name))
    return flops / dt / 1e12, desc, oracle.max_threads(), dt


def oracle_sample_rate(w, inp, target_s, seed=0):
    """Calibrate, then time one sample of about target_s seconds."""
    n = oracle_calibrate(w, inp, target_s, seed)
    rate, desc, cores, dt = oracle_timed_sample(w, inp, n, seed + 1)
    return rate, desc, cores, n, dt


# ------------------------------------------------------------------ GPU arm

def run_ours(args):
    import torch
    import exact_attention_101_b200 as fa

    rank, local_rank, world = rank_env()
    w = select_workload(args)
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    inp = workloads.make_inputs(w, seed=rank_seed(w, rank))
    host = [inp.q, inp.k, inp.v]
    q, k, v = (t.to(dev) for t in host)
    fp8 = inp.descale_q is not None or w.rotate
    if inp.descale_q is not None:
        dq, dk, dv = (t.to(dev) for t in (inp.descale_q, inp.descale_k, inp.descale_v))
    out_dtype = torch.float32 if w.out_dtype == "f32" else torch.bfloat16
    o = torch.empty((w.B, w.Hq, w.N, w.d), dtype=out_dtype, device=dev)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    # Incoherent-processing workloads quantise their bf16 Q, K (rotated) and V on the GPU
    # every step, then run the fp8 kernel: 3 quantisation kernels + 1 attention kernel.
    launches_per_step = 4 if w.rotate else (3 if w.kind == "bwd" else 1)
    split = None
    if w.kind == "varlen":
        host.append(inp.cu_seqlens)
        cu_d = inp.cu_seqlens.to(dev)
        total = int(inp.cu_seqlens[-1])
        max_len = max(workloads.varlen_lengths(w))
        o = torch.empty((total, w.Hq, w.d), dtype=out_dtype, device=dev)
        lse = torch.empty((w.Hq, total), dtype=torch.float32, device=dev)
    if w.kind == "bwd":
        # The forward's O and LSE, computed once before timing; each step is one backward.
        host += [inp.dout]
        dout = inp.dout.to(dev)
        fa.forward(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if w.rotate:
        host.append(inp.signs)
        signs = inp.signs.to(dev)
        q8, k8, v8 = (torch.empty(t.shape, dtype=torch.float8_e4m3fn, device=dev)
                      for t in (q, k, v))
        dq = torch.empty((w.B * w.Hq,), dtype=torch.float32, device=dev)
        dk = torch.empty((w.B * w.Hkv,), dtype=torch.float32, device=dev)
        dv = torch.empty((w.B * w.Hkv,), dtype=torch.float32, device=dev)
        split = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
                 for _ in range(args.steps)]

    def step(i=None):
        ev = split[i] if (split is not None and i is not None) else None
        if w.rotate:
            if ev:
                ev[0].record(stream)
            fa.quantize_e4m3(q, signs, out=q8, descale=dq)
            fa.quantize_e4m3(k, signs, out=k8, descale=dk)
            fa.quantize_e4m3(v, None, out=v8, descale=dv)
            if ev:
                ev[1].record(stream)
            fa.forward_fp8(q8, k8, v8, dq, dk, dv, causal=w.causal, scale=w.scale, out=o,
                           lse=lse)
            if ev:
                ev[2].record(stream)
        elif w.kind == "bwd":
            fa.backward(q, k, v, o, lse, dout, causal=w.causal, scale=w.scale, dq=dq, dk=dk,
                        dv=dv)
        elif w.kind == "varlen":
            fa.forward_varlen(q, k, v, cu_d, cu_d, max_len, causal=w.causal, scale=w.scale,
                              out_dtype=out_dtype, out=o, lse=lse)
        elif fp8:
            fa.forward_fp8(q, k, v, dq, dk, dv, causal=w.causal, scale=w.scale, out=o, lse=lse)
        elif w.dropout:
            # a new mask every step, as in training (the offset is the step number)
            fa.forward_dropout(q, k, v, w.dropout, seed=w.seed, offset=0 if i is None else i,
                               causal=w.causal, scale=w.scale, out_dtype=out_dtype, out=o,
                               lse=lse)
        else:
            fa.forward(q, k, v, causal=w.causal, scale=w.scale, out_dtype=out_dtype, out=o,
                       lse=lse)

    # First call on its own (module load, attribute setup, descriptor encoding), wall clock.
    torch.cuda.synchronize(dev)
    t_first = time.perf_counter()
    step()
    torch.cuda.synchronize(dev)
    first_call_ms = (time.perf_counter() - t_first) * 1e3
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    fa.check_device_error(stream)

    clocks = ClockSampler(local_rank, dev)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    # One event at every step boundary: the total is first-to-last, and the per-step
    # times give the median and the best step.
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    clocks.begin()
    evs[0].record(stream)
    for i in range(args.steps):
        step(i)
        evs[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    clocks.end()
    barrier()
    clk = clocks.stop()
    fa.check_device_error(stream)
    elapsed_ms = evs[0].elapsed_time(evs[-1])
    per_step = sorted(evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps))
    ms_max = max_over_ranks(elapsed_ms, world, dev)
    ms_per_step = ms_max / args.steps
    value = w.flops * world * args.steps / (ms_max / 1e3) / 1e12
    # Dominant kernel: the attention kernel, launched once per step on `stream`.  Alone in
    # the step, its average launch duration is this rank's elapsed time / steps; after the
    # quantisation kernels, events recorded around it inside the timed loop give it.
    quant = None
    if split is None:
        kernel_ms = elapsed_ms / args.steps
    else:
        kernel_ms = sum(e[1].elapsed_time(e[2]) for e in split) / args.steps
        quant_ms = sum(e[0].elapsed_time(e[1]) for e in split) / args.steps
        # Algorithmic bytes of quantising Q, K and V: read bf16 once, write e4m3 codes and
        # one fp32 descale per (batch, head).
        elems = sum(t.numel() for t in (q, k, v))
        qbytes = 3.0 * elems + 4.0 * (dq.numel() + dk.numel() + dv.numel())
        quant = {"kernel": "fa_quant_kernel x 3 (Q and K rotated, V plain)",
                 "bound": "hbm", "ms_per_step": quant_ms,
                 "achieved": qbytes / (quant_ms / 1e3) / 1e9, "unit": "GB/s",
                 "algorithmic_bytes": qbytes}
    achieved = w.flops / (kernel_ms / 1e3) / 1e12

    # End to end through the public API: pinned host inputs -> device, forward, O and LSE
    # back to pinned host memory, every step inside the timed region.
    e2e_steps = 0 if args.no_e2e else max(3, min(args.steps, 20))
    hq_, hk_, hv_ = (t.pin_memory() for t in host[:3])
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    hds = []
    if w.kind == "bwd":
        hdo_ = inp.dout.pin_memory()
        ho_in = o.cpu().pin_memory()
        hl_in = lse.cpu().pin_memory()
        hdq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hdk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hdv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
    if w.kind == "varlen":
        hcu_ = inp.cu_seqlens.pin_memory()
    if w.rotate:
        hs_ = inp.signs.pin_memory()
    elif fp8:
        hds = [t.pin_memory() for t in (inp.descale_q, inp.descale_k, inp.descale_v)]

    # Plain bf16 forward: the public host-memory entry point (fa_fwd_host), whose copies in
    # both directions overlap the kernels chunk by chunk.  Other workloads: pinned copies on
    # the stream around the device-memory call.
    host_api = w.kind == "fwd" and not fp8 and not w.dropout
    # kernels per end-to-end step: fa_fwd_host's default chunk count (as many K/V heads per
    # chunk as fit one wave of work units), else the device call's own launches
    if host_api:
        # the library's chunk plan: as many K/V heads per chunk as fit one wave of work
        # units (CTA pairs: one unit per two SMs; one-CTA kernel at d = 256: 128-row units)
        pair = uses_pair_kernel(w, fp8)
        unit_rows = 128 if (w.d > 128 and not pair) else 256
        group_units = (w.Hq // w.Hkv) * (-(-w.N // unit_rows))
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        per = max(1, (sms // 2 if pair else sms) // group_units)
        e2e_launches = e2e_steps * (-(-(w.B * w.Hkv) // per))
    else:
        e2e_launches = e2e_steps * launches_per_step

    def e2e_step():
        if host_api:
            fa.forward_host(hq_, hk_, hv_, causal=w.causal, scale=w.scale, out_dtype=out_dtype,
                            out=ho, lse=hl, device_buffers=(q, k, v, o, lse), stream=stream)
            return
        q.copy_(hq_, non_blocking=True)
        k.copy_(hk_, non_blocking=True)
        v.copy_(hv_, non_blocking=True)
        if w.kind == "bwd":
            for dst, src in ((dout, hdo_), (o, ho_in), (lse, hl_in)):
                dst.copy_(src, non_blocking=True)
            step()
            for dst, src in ((hdq, dq), (hdk, dk), (hdv, dv)):
                dst.copy_(src, non_blocking=True)
            return
        if w.kind == "varlen":
            cu_d.copy_(hcu_, non_blocking=True)
        if w.rotate:
            signs.copy_(hs_, non_blocking=True)
        elif fp8:
            for dst, src in zip((dq, dk, dv), hds):
                dst.copy_(src, non_blocking=True)
        step()
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e = None
    if e2e_steps:
        e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        h2d = sum(t.numel() * t.element_size() for t in host)
        h2d += sum(t.numel() * t.element_size() for t in hds)
        d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
        if w.kind == "bwd":
            h2d += o.numel() * o.element_size() + lse.numel() * lse.element_size()
            d2h = sum(t.numel() * t.element_size() for t in (dq, dk, dv))
        e2e = {"value": w.flops * world * e2e_steps / (e2e_ms / 1e3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "api": ("fa_fwd_host: pinned host buffers, copies pipelined by head chunks"
                       if host_api else "pinned copies on the stream around the device call")}

    # Lazy-rescale statistics of the forward instances on the CTA-pair kernel (it counts
    # them): one more launch on the workload's inputs and one on scores that drift along the
    # keys (same shape), each against the eager rule's count on the same rows.
    pair_kernel = uses_pair_kernel(w, fp8)
    rescale = None
    if pair_kernel and w.out_dtype == "bf16":
        def counts(qq, kk, vv):
            fa.rescale_stats(reset=True, stream=stream)
            fa.forward(qq, kk, vv, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)
            steps, lazy, eager = fa.rescale_stats(reset=True, stream=stream)
            return {"row_block_steps": steps, "lazy_rescales": lazy, "eager_rescales": eager,
                    "eager_over_lazy": (eager / lazy) if lazy else None}
        rescale = {"rule": "lazy: move the maximum only when a block exceeds it by more than 8 "
                           "(log2 units); eager: whenever a block raises it",
                   w.name: counts(q, k, v)}
        dr = workloads.drift_inputs(w.B, w.Hq, w.N, w.d, seed=w.seed + 17)
        dq_, dk_, dv_ = (t.to(dev) for t in (dr.q, dr.k, dr.v))
        if w.Hkv != w.Hq:
            dk_, dv_ = dk_[:, :w.Hkv].contiguous(), dv_[:, :w.Hkv].contiguous()
        rescale["drift (scores ramp along the keys, workloads.drift_inputs)"] = counts(dq_, dk_, dv_)
        del dq_, dk_, dv_

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    if quant is not None:
        quant["peak"] = peaks["hbm_gbs"]
        quant["frac"] = quant["achieved"] / quant["peak"]
    fp8_peak = load_fp8_peak()
    if fp8 and fp8_peak is not None:
        peak = fp8_peak
        peak_note = "measured e4m3 torch._scaled_mm burst, profiles/fp8_peak.json"
    elif fp8:
        peak = peaks["bf16_tflops"] * 2.0   # fp8 dense = 2x bf16 dense (nominal ratio)
        peak_note = "fp8 peak = measured bf16 burst x 2 (nominal fp8/bf16 ratio)"
    else:
        peak = peaks["bf16_tflops"]
        peak_note = "measured cuBLAS bf16 burst (kernel timed alone)"
    datasheet = DATASHEET_FP8_TFLOPS if fp8 else DATASHEET_BF16_TFLOPS

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        if w.kind == "bwd":
            rate, desc, cores, _ = oracle_bwd_sample(w, inp, args.cpu_seconds)
        elif w.kind == "varlen":
            rate, desc, cores, _ = oracle_varlen_sample(w, inp, args.cpu_seconds)
        else:
            rate, desc, cores, _, _ = oracle_sample_rate(w, inp, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
               "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    kernel_name = "fa_fwd_pair_kernel (CTA pairs)" if pair_kernel else "fa_fwd_kernel"
    if w.kind == "bwd":
        kernel_name = ("fa_bwd: prep kernel + fa_bwd_kernel + dQ kernel (and the dQ "
                       "accumulator memset), timed together as one call")

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "ms_median": per_step[len(per_step) // 2], "ms_best": per_step[0],
        "ms_worst": per_step[-1],
        "first_call_ms": first_call_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
        "config": bench_config(w),
        "frac_of_datasheet_peak": achieved / datasheet,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": profiled_traffic(w.name),
                     "peak_source": "%s (%s)" % (peak_src, peak_note),
                     "datasheet_peak": datasheet, "frac_of_datasheet": achieved / datasheet,
                     "kernel": kernel_name},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps + e2e_launches,
        "clocks": clk,
    }
    if quant is not None:
        line["quantise"] = quant
    if rescale is not None:
        line["rescale"] = rescale
    print(json.dumps(line))


# ------------------------------------------------------------------ reference arm

def bench_config(w):
    """The `config` object of the JSON line, identical in both arms.  The inputs of every
    timed workload exceed the 126 MB L2, so no flush runs between steps."""
    return dict(w.describe(), l2="inputs larger than L2 (no flush)",
                parallelism="independent replicas of the workload per GPU")


def select_workload(args):
    """The named workload, optionally with fewer heads (a smaller case of the same
    kernel for profiling); the query/KV head ratio is kept."""
    import dataclasses
    w = workloads.WORKLOADS[args.workload]
    if args.heads:
        g = w.Hq // w.Hkv
        if args.heads % g:
            raise SystemExit("--heads must be a multiple of %d for %s" % (g, w.name))
        w = dataclasses.replace(w, name="%s_h%d" % (w.name, args.heads), Hq=args.heads,
                                Hkv=args.heads // g)
    return w


def run_reference(args):
    rank, _, world = rank_env()
    if rank != 0:
        return
    w = select_workload(args)
    inp = workloads.make_inputs(w)
    per_step = max(0.05, args.reference_budget_s / max(1, args.steps + args.warmup))
    if w.kind == "bwd":
        return run_reference_bwd(args, w, inp, per_step, world)
    if w.kind == "varlen":
        return run_reference_sampled(args, w, inp, per_step, world, oracle_varlen_sample)
    n_rows = oracle_calibrate(w, inp, per_step)
    for i in range(args.warmup):
        oracle_timed_sample(w, inp, n_rows, seed=100 + i)
    rates, descs, total_s = [], [], 0.0
    cores = 1
    for i in range(args.steps):
        rate, desc, cores, dt = oracle_timed_sample(w, inp, n_rows, seed=i)
        rates.append(rate)
        descs.append(desc)
        total_s += dt
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "per step: " + descs[-1]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line))


def run_reference_bwd(args, w, inp, per_step, world):
    return run_reference_sampled(args, w, inp, per_step, world, oracle_bwd_sample)


def run_reference_sampled(args, w, inp, per_step, world, sampler):
    for _ in range(args.warmup):
        sampler(w, inp, per_step)
    rates, total_s, desc, cores = [], 0.0, "", 1
    for _ in range(args.steps):
        rate, desc, cores, dt = sampler(w, inp, per_step)
        rates.append(rate)
        total_s += dt
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="long", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU time spent timing the oracle for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the number of query heads (smaller profiling case)")
    ap.add_argument("--measure-fp8-peak", action="store_true",
                    help="print the measured dense e4m3 GEMM peak (torch._scaled_mm) and exit")
    ap.add_argument("--reference-budget-s", type=float, default=120.0,
                    help="total CPU time of the reference arm")
    args = ap.parse_args(argv)
    if args.measure_fp8_peak:
        return measure_fp8_peak()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    _, _, world = rank_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus %d needs torchrun with %d processes" % (args.gpus, args.gpus))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()

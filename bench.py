"""Benchmark of the frozen-NF4 LoRA linear layer on B200.

One step = the whole hot path on one batch of a LLaMA-65B-shaped block:
the one-shot NF4 quantization (with double-quantized constants) of the
block's seven frozen weights (q, k, v, o 8192 x 8192; gate, up 22016 x 8192;
down 8192 x 22016; 809.5 M parameters, 2.04 GB read and written), then the
forward of the seven LoRA linears (T = s X A and the fused dequant-GEMM
Y = X W'^T + T B) and their backward (U, dB, the fused dequant-GEMM
dX = dY W' + U A^T, dA), 4096 tokens, r = 64, scale 0.25, seeded synthetic
inputs, all through the C ABI of libqlora.so.  This is the headline `value`
(TFLOP/s of the algorithmic fwd+bwd work over the whole step time,
quantization included) with tokens/s beside it.

The same JSON line carries, as nested objects measured the same way:
  mlp_trio   LLaMA-7B MLP (gate, up 11008 x 4096; down 4096 x 11008),
             8192 tokens, SiLU-gated, fwd+bwd through the three linears
             (weights quantized once, outside the step);
  attn_proj  LLaMA-7B attention projection 4096^2 with 0.1 % outliers,
             4096 tokens, quantize + fwd + bwd;
  small_m    the small-M forward sweep (M in {1, 4, 16, 64}) as NF4 weight
             GB/s against the HBM peak.

With --gpus N every rank runs its own 4096 tokens through the block (weak
scaling) and the adapter gradients of the seven linears, written by the
backward into one flat bucket, are summed over ranks by one NCCL all-reduce
per step (the data-parallel exchange).  Run without torchrun, --gpus N > 1
re-launches itself under torch.distributed.run with N processes.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle (the
float64 restatement in oracle/) on a bounded sample of the block step.
"""

from __future__ import annotations

import argparse
import json
import os
import socket
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s & tokens/s; small-M NF4 weight GB/s vs HBM peak"
M_BLOCK, R, SCALE = 4096, 64, 0.25
BLOCK_WORKLOAD = dict(
    workload="llama65b_block_linears", M=M_BLOCK, r=R, scale=SCALE,
    linears="q,k,v,o 8192x8192; gate,up 22016x8192; down 8192x22016 (out x in)",
    step="quantize_nf4 x7 (one-shot, 809.5M params) + linear_fwd x7 + linear_bwd x7")
L2_NOTE = "flushed between timed steps (256 MB write)"


def flops_fwd(M, K, N, r):
    return 2 * M * N * K + 2 * M * r * (K + N)


def flops_bwd(M, K, N, r):
    return 2 * M * N * K + 4 * M * r * (K + N)


def nf4_bytes(numel):
    """Packed bytes of a weight: codes, 8-bit constants, float group maxima."""
    nb = -(-numel // 64)
    return (numel + 1) // 2 + nb + 4 * (-(-nb // 256))


def quantize_bytes(numel):
    """Algorithmic HBM bytes of one quantization: bf16 in, packed out."""
    return 2 * numel + nf4_bytes(numel)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.poller = None

    # Preferred: NVML read every ~1 ms by a child process (a thread of this
    # process would share the GIL with the launch loop and could go unsampled
    # for a whole short timed region).  Read-only queries; nothing is set.
    POLL = (
        "import json, select, sys\n"
        "import pynvml\n"
        "pynvml.nvmlInit()\n"
        "try:\n"
        "    h = pynvml.nvmlDeviceGetHandleByPciBusId(sys.argv[1])\n"
        "except Exception:\n"
        "    h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[2]))\n"
        "gr = getattr(pynvml, 'nvmlDeviceGetCurrentClocksEventReasons', None) or "
        "getattr(pynvml, 'nvmlDeviceGetCurrentClocksThrottleReasons')\n"
        "mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)\n"
        "rows = []\n"
        "def sample():\n"
        "    rows.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), gr(h)))\n"
        "sample()\n"
        "print('ready', flush=True)\n"
        "while not select.select([sys.stdin], [], [], 0.001)[0]:\n"
        "    sample()\n"
        "print(json.dumps({'max': mx, 'rows': rows[1:] or rows}), flush=True)\n"
    )

    def _bus_id(self):
        import torch
        pr = torch.cuda.get_device_properties(self.gpu)
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"

    def start(self):
        try:
            self.poller = subprocess.Popen([sys.executable, "-c", self.POLL, self._bus_id(), str(self.gpu)],
                                           stdin=subprocess.PIPE, stdout=subprocess.PIPE,
                                           stderr=subprocess.DEVNULL, text=True)
            if self.poller.stdout.readline().strip() == "ready":
                return
            self.poller.kill()
        except Exception:
            pass
        self.poller = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.poller is not None:
            try:
                out, _ = self.poller.communicate(input="stop\n", timeout=30)
                d = json.loads(out.strip().splitlines()[-1])
            except Exception:
                self.poller.kill()
                return None
            rows = d["rows"]
            if not rows:
                return None
            # NVML reason bits: 0x4 sw power cap, 0x8 hw slowdown, 0x20 sw thermal, 0x40 hw thermal.
            bits = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}
            sm = sorted(r[0] for r in rows)
            reasons = sorted({name for r in rows for b, name in bits.items() if r[1] & b})
            return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": d["max"], "reasons": reasons,
                    "samples": len(rows), "source": "nvml"}
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi"}


# ---------------------------------------------------------------- CPU oracle
def cpu_oracle_block_sample(rows: int = 128, slab: int = 128):
    """Time the float64 oracle on a bounded sample of the block step and
    scale it to the whole step.

    Sample: for each of the seven linears, the quantization of a `slab`-row
    slab of its weight (slab x K of the N x K weight) and the forward +
    backward of `rows` tokens against that slab.  The whole step's time is
    estimated as (sampled quantize time) x (809.5 M / sampled parameters) +
    (sampled fwd+bwd time) x (step flops / sampled flops)."""
    import numpy as np
    from bit_quantized_lora_quantize_b200 import synthetic
    from oracle import dequantize_nf4, lora_linear_backward, lora_linear_forward, quantize_nf4

    rng = np.random.default_rng(5)
    t_q = t_g = 0.0
    p_s = fl_s = 0
    p_full = fl_full = 0
    for i, (name, N, K) in enumerate(synthetic.LLAMA65B_LINEARS):
        W = synthetic.weight_only(slab, K, seed=300 + i).float().numpy()
        X = rng.standard_normal((rows, K))
        dY = rng.standard_normal((rows, slab))
        A = rng.standard_normal((K, R)) * 0.01
        B = rng.standard_normal((R, slab)) * 0.01
        t0 = time.perf_counter()
        codes, aq, sc = quantize_nf4(W)
        t1 = time.perf_counter()
        Wdq = dequantize_nf4(codes, aq, sc, W.size).reshape(slab, K)
        lora_linear_forward(X, Wdq, A, B, SCALE)
        lora_linear_backward(dY, X, Wdq, A, B, SCALE)
        t2 = time.perf_counter()
        t_q += t1 - t0
        t_g += t2 - t1
        p_s += W.size
        fl_s += flops_fwd(rows, K, slab, R) + flops_bwd(rows, K, slab, R)
        p_full += N * K
        fl_full += flops_fwd(M_BLOCK, K, N, R) + flops_bwd(M_BLOCK, K, N, R)
    step_s = t_q * p_full / p_s + t_g * fl_full / fl_s
    try:
        from threadpoolctl import threadpool_info
        blas = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        blas = None
    return {"value": fl_full / step_s / 1e12, "unit": "TFLOP/s", "cores": host_cores(), "blas_threads": blas,
            "kind": "oracle",
            "sample": (f"per linear: quantize of a {slab}-row slab of the weight + fwd+bwd of {rows} tokens "
                       f"against it (float64 numpy); whole-step time scaled from the sample by parameter "
                       f"count (quantize) and by flops (fwd+bwd)"),
            "sample_seconds": t_q + t_g, "est_step_seconds": step_s, "tokens_per_s": M_BLOCK / step_s,
            "quantize_mparams_per_s": p_s / t_q / 1e6, "fwd_bwd_gflops": fl_s / t_g / 1e9}


def block_flops():
    from bit_quantized_lora_quantize_b200 import synthetic
    return sum(flops_fwd(M_BLOCK, K, N, R) + flops_bwd(M_BLOCK, K, N, R) for _, N, K in synthetic.LLAMA65B_LINEARS)


def run_reference(args, rank, world):
    if rank != 0:
        return
    for _ in range(args.warmup):
        cpu_oracle_block_sample(rows=16, slab=64)
    samples = [cpu_oracle_block_sample(rows=128, slab=128) for _ in range(args.steps)]
    vals = sorted(s["value"] for s in samples)
    v = vals[len(vals) // 2]
    cb = dict(samples[-1])
    cb["value"] = v
    ms_full = block_flops() / (v * 1e12) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_full, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(BLOCK_WORKLOAD, l2="n/a (host)"), "cpu_baseline": cb,
            "tokens_per_s": M_BLOCK / (ms_full * 1e-3),
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- timing helpers
def traffic_for(key: str):
    """DRAM bytes per launch from the committed ncu summary, if it still
    describes the current kernel source (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        ent = t[key]
        hsh = hashlib.sha256()
        for name in ent["sources"]:  # the kernel's .cu file and the headers it includes
            with open(os.path.join(ROOT, "bit_quantized_lora_quantize_b200", "csrc", name), "rb") as f:
                hsh.update(f.read())
        if hsh.hexdigest()[:16] != ent["sources_sha256_16"]:
            return None
        return ent["dram_bytes_per_launch"]
    except Exception:
        return None


class Calls:
    """Runs the library calls of a step.  Each call is exactly one kernel
    launch; in profiling mode a pair of CUDA events on the launching stream
    brackets every call, keyed by (kernel, linear)."""

    def __init__(self):
        self.recs = None

    def __call__(self, kernel, tag, work, fn):
        if self.recs is None:
            return fn()
        import torch
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        out = fn()
        b.record()
        self.recs.append((kernel, tag, work, a, b))
        return out

    def profile(self, step, n, flush):
        """Run `n` more steps with per-call events; return
        {(kernel, tag): dict(ms_total, launches, work)} and the launch count."""
        import torch
        self.recs = []
        for _ in range(n):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        agg = {}
        for kernel, tag, work, a, b in self.recs:
            e = agg.setdefault((kernel, tag), {"ms_total": 0.0, "launches": 0, "work": work})
            e["ms_total"] += a.elapsed_time(b)
            e["launches"] += 1
        self.recs = None
        return agg


def time_steps(step, steps, flush, world, local_rank, sample_clocks=True):
    """Device time of exactly `steps` steps (CUDA events around each step on
    the launching stream, L2 flushed before each), max over ranks."""
    import torch
    import torch.distributed as dist
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler(local_rank) if sample_clocks else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    total = sum(a.elapsed_time(b) for a, b in evs)
    t = torch.tensor([total], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item()) / steps, clocks


def time_e2e(e2e_step, steps, world, after=None):
    """Device time per step of the end-to-end step (host copies included).
    `after` makes the timing stream wait for work the step left on other
    streams, so that it ends inside the timed region."""
    import torch
    import torch.distributed as dist
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        e2e_step()
    if after is not None:
        after()
    e1.record(stream)
    torch.cuda.synchronize()
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item()) / steps


def kernel_table(agg):
    tot = sum(v["ms_total"] for v in agg.values()) or 1.0
    out = {}
    for (kernel, tag), v in sorted(agg.items()):
        out[f"{kernel}/{tag}"] = {"us_per_launch": v["ms_total"] * 1e3 / v["launches"], "launches": v["launches"],
                                  "share": v["ms_total"] / tot}
    return out


def gemm_roofline(agg, peaks, sustained=False):
    """Roofline of the dominant fused GEMM (largest total time over the
    profiled steps): algorithmic flops per launch / mean launch time, against
    the measured bf16 peak: the sustained figure for kernels timed inside a
    long step (power-capped clocks), the burst figure otherwise."""
    gem = {k: v for k, v in agg.items() if k[0].startswith("fused_nf4")}
    if not gem:
        return None
    key = max(gem, key=lambda k: gem[k]["ms_total"])
    v = gem[key]
    ms = v["ms_total"] / v["launches"]
    achieved = v["work"]["flops"] / (ms * 1e-3) / 1e12
    tkey = f"{key[0]}/{key[1]}"
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    kind = "sustained" if sustained else "burst"
    return {"bound": "tensor", "kernel": tkey, "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic_for(tkey),
            "peak_source": f"{peaks['source']} bf16 {kind} ({'of measured' if peaks['source'] == 'measured' else 'of fallback'})",
            "frac_of_burst": achieved / peaks["bf16_tflops"],
            "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"], "us_per_launch": ms * 1e3,
            "flops_per_launch": v["work"]["flops"],
            "flops_counted": "2MNK + 2Mr(N+K) (dense product, LoRA product and the rank-r intermediate)"}


def quantize_roofline(agg, peaks):
    qk = {k: v for k, v in agg.items() if k[0] == "quantize_nf4"}
    if not qk:
        return None
    by = sum(v["work"]["bytes"] * v["launches"] for v in qk.values())
    ms = sum(v["ms_total"] for v in qk.values())
    steps = max(v["launches"] for v in qk.values())
    achieved = by / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "quantize_nf4", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic_for("quantize_nf4/gate"),
            "traffic_note": "per launch, for the 22016 x 8192 weight (one of the seven)",
            "bytes_per_step": by / steps, "us_per_step": ms * 1e3 / steps,
            "bytes_counted": "2 B read + 0.5159 B written per weight",
            "peak_source": f"{peaks['source']} HBM copy bandwidth"}


# ---------------------------------------------------------------- the block step
class Linear:
    """Device-resident tensors of one LoRA linear (inputs, outputs, workspace)."""

    def __init__(self, q, case, tag, dev, grads=None):
        import torch
        self.tag = tag
        self.case = case
        self.M, self.K, self.N, self.r, self.s = case.M, case.K, case.N, case.r, case.scale
        self.W = case.W.to(dev)
        self.P = q.qlora_quantize_nf4(self.W)
        self.A, self.B, self.dY = case.A.to(dev), case.B.to(dev), case.dY.to(dev)
        self.ws = q.new_workspace(self.M, self.K, self.N, self.r, dev)
        self.Y = torch.empty(self.M, self.N, dtype=torch.bfloat16, device=dev)
        self.T = torch.empty(self.M, self.r, dtype=torch.float32, device=dev)
        self.dX = torch.empty(self.M, self.K, dtype=torch.bfloat16, device=dev)
        if grads is None:
            self.dA = torch.empty(self.K, self.r, dtype=torch.float32, device=dev)
            self.dB = torch.empty(self.r, self.N, dtype=torch.float32, device=dev)
        else:
            self.dA, self.dB = grads

    @property
    def numel(self):
        return self.N * self.K


def make_block(q, synthetic, dev, rank, grads_bucket_cls):
    import torch
    cases = synthetic.llama65b_block(M_BLOCK, R, SCALE)
    if rank != 0:
        # Other ranks take other tokens (and upstream gradients): weak scaling.
        g = torch.Generator().manual_seed(1000 + rank)
        X = (torch.randn(cases[0][1].X.shape, generator=g)).to(torch.bfloat16)
        Xd = (torch.randn(cases[-1][1].X.shape, generator=g)).to(torch.bfloat16)
        for _, c in cases:
            c.X = X if c.K == 8192 else Xd
            c.dY = torch.randn(c.dY.shape, generator=g).to(torch.bfloat16)
    bucket = grads_bucket_cls([(c.K, c.N, c.r) for _, c in cases], dev)
    X = cases[0][1].X.to(dev)
    Xd = cases[-1][1].X.to(dev)
    lins = []
    for i, (name, c) in enumerate(cases):
        lin = Linear(q, c, name, dev, grads=bucket[i])
        lin.X = X if c.K == 8192 else Xd
        lins.append(lin)
    return lins, bucket, X, Xd


def block_step_fn(q, lins, calls, bucket, world, streams=None):
    """The block step.  With `streams` (two CUDA streams, the first the
    current one) the seven linears' forward+backward chains alternate between
    them: the linears are independent, so one GEMM's last partial wave
    overlaps the next one's first tiles.  Each linear keeps its own
    workspace, and its forward and backward stay on one stream.  (Putting
    each weight's quantization at the head of its own chain instead of all
    seven first measured 0.8 % slower.)"""
    import torch

    def on(i):
        return streams[i % 2] if streams else torch.cuda.current_stream()

    def quantize(l):
        calls("quantize_nf4", l.tag, {"bytes": quantize_bytes(l.numel)},
              lambda l=l: q.qlora_quantize_nf4(l.W, out=l.P))

    def step():
        for l in lins:
            quantize(l)
        if streams:
            streams[1].wait_stream(streams[0])
        for i, l in enumerate(lins):
            with torch.cuda.stream(on(i)):
                calls("fused_nf4_fwd", l.tag, {"flops": 2 * l.M * l.N * l.K + 2 * l.M * l.r * (l.N + l.K)},
                      lambda l=l: q.qlora_linear_fwd(l.X, l.P, l.A, l.B, l.s, workspace=l.ws, Y=l.Y, T_save=l.T))
        for i in reversed(range(len(lins))):
            l = lins[i]
            with torch.cuda.stream(on(i)):
                calls("fused_nf4_dx", l.tag, {"flops": 2 * l.M * l.N * l.K + 2 * l.M * l.r * (l.N + l.K)},
                      lambda l=l: q.qlora_linear_bwd(l.dY, l.X, l.T, l.P, l.A, l.B, l.s, workspace=l.ws, dX=l.dX,
                                                     dA=l.dA, dB=l.dB))
        if streams:
            streams[0].wait_stream(streams[1])
        if world > 1:
            bucket.all_reduce()
    return step


def bench_block(args, q, synthetic, dp, dev, rank, world, local_rank, flush, peaks):
    import torch
    lins, bucket, X, Xd = make_block(q, synthetic, dev, rank, dp.GradBucket)
    calls = Calls()
    streams = None if args.one_stream else (torch.cuda.current_stream(), torch.cuda.Stream())
    step = block_step_fn(q, lins, calls, bucket, world, streams)
    # Per-launch durations (roofline, kernel table) come from the same step
    # with every launch on one stream: concurrent launches would share the
    # GPU inside each other's events.
    step_serial = block_step_fn(q, lins, calls, bucket, world, None)
    fl_step = sum(flops_fwd(l.M, l.K, l.N, l.r) + flops_bwd(l.M, l.K, l.N, l.r) for l in lins)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    for l in lins:
        if q.qlora_check_status(l.ws) != 0:
            raise RuntimeError("device pipeline timeout during warm-up")
    ms, clocks = time_steps(step, args.steps, flush, world, local_rank)
    agg = calls.profile(step_serial, args.steps, flush)

    # End to end through the public API: every step copies the seven bf16
    # weights, both inputs and the seven dY in from pinned host memory, and
    # the seven Y and dX and the gradient bucket back.
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    hW = [pin(l.case.W) for l in lins]
    hdY = [pin(l.case.dY) for l in lins]
    hX, hXd = pin(lins[0].case.X), pin(lins[-1].case.X)
    hY = [torch.empty(l.Y.shape, dtype=l.Y.dtype).pin_memory() for l in lins]
    hdX = [torch.empty(l.dX.shape, dtype=l.dX.dtype).pin_memory() for l in lins]
    hG = torch.empty(bucket.flat.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * 2 for t in hW + hdY) + hX.numel() * 2 + hXd.numel() * 2
    d2h = sum(t.numel() * 2 for t in hY + hdX) + hG.numel() * 4

    # Three streams: host->device copies, the library calls, device->host
    # copies; per-linear events order them, so the two copy directions and
    # the kernels overlap (within a step and across steps) and every buffer
    # is reused only after its previous use.
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    n = len(lins)
    w_ready, w_free = [ev() for _ in range(n)], [ev() for _ in range(n)]
    dy_ready, dy_free = [ev() for _ in range(n)], [ev() for _ in range(n)]
    y_done, y_free = [ev() for _ in range(n)], [ev() for _ in range(n)]
    dx_done, dx_free = [ev() for _ in range(n)], [ev() for _ in range(n)]
    x_ready, x_free, g_done, g_free = ev(), ev(), ev(), ev()
    state = {"first": True}

    def e2e_step():
        first = state["first"]
        state["first"] = False
        with torch.cuda.stream(s_in):
            if not first:
                s_in.wait_event(x_free)
            X.copy_(hX, non_blocking=True)
            Xd.copy_(hXd, non_blocking=True)
            x_ready.record(s_in)
            for i, (l, w) in enumerate(zip(lins, hW)):
                if not first:
                    s_in.wait_event(w_free[i])
                l.W.copy_(w, non_blocking=True)
                w_ready[i].record(s_in)
            for i in reversed(range(n)):
                if not first:
                    s_in.wait_event(dy_free[i])
                lins[i].dY.copy_(hdY[i], non_blocking=True)
                dy_ready[i].record(s_in)
        for i, l in enumerate(lins):
            comp.wait_event(w_ready[i])
            q.qlora_quantize_nf4(l.W, out=l.P)
            w_free[i].record(comp)
        comp.wait_event(x_ready)
        for i, l in enumerate(lins):
            if not first:
                comp.wait_event(y_free[i])
            q.qlora_linear_fwd(l.X, l.P, l.A, l.B, l.s, workspace=l.ws, Y=l.Y, T_save=l.T)
            y_done[i].record(comp)
        if not first:
            comp.wait_event(g_free)
        for i in reversed(range(n)):
            l = lins[i]
            comp.wait_event(dy_ready[i])
            if not first:
                comp.wait_event(dx_free[i])
            q.qlora_linear_bwd(l.dY, l.X, l.T, l.P, l.A, l.B, l.s, workspace=l.ws, dX=l.dX, dA=l.dA, dB=l.dB)
            dy_free[i].record(comp)
            dx_done[i].record(comp)
        x_free.record(comp)
        if world > 1:
            bucket.all_reduce()
        g_done.record(comp)
        with torch.cuda.stream(s_out):
            for i, (l, y) in enumerate(zip(lins, hY)):
                s_out.wait_event(y_done[i])
                y.copy_(l.Y, non_blocking=True)
                y_free[i].record(s_out)
            for i in reversed(range(n)):
                s_out.wait_event(dx_done[i])
                hdX[i].copy_(lins[i].dX, non_blocking=True)
                dx_free[i].record(s_out)
            s_out.wait_event(g_done)
            hG.copy_(bucket.flat, non_blocking=True)
            g_free.record(s_out)

    def e2e_flush():
        # The last step's copies out end before the timed region closes.
        comp.wait_stream(s_out)

    e2e_ms = time_e2e(e2e_step, args.steps, world, after=e2e_flush)
    for l in lins:
        if q.qlora_check_status(l.ws) != 0:
            raise RuntimeError("device pipeline timeout during timing")
    opt = bench_paged_adamw(args, lins, bucket, dev, flush, peaks) if rank == 0 else None
    launches_per_step = 3 * len(lins)
    res = {
        "ms_per_step": ms, "value": fl_step * world / (ms * 1e-3) / 1e12,
        "tokens_per_s": M_BLOCK * world / (ms * 1e-3),
        "tflops_dense_only": sum(4 * l.M * l.N * l.K for l in lins) * world / (ms * 1e-3) / 1e12,
        "flops_per_step": fl_step, "clocks": clocks, "kernels": kernel_table(agg),
        "roofline": gemm_roofline(agg, peaks, sustained=True), "roofline_quantize": quantize_roofline(agg, peaks),
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": fl_step * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "copies": "in: 7 bf16 weights, X, X_down, 7 dY; out: 7 Y, 7 dX, dA|dB bucket; "
                          "copy streams in each direction overlapped with the kernels"},
        "grad_bucket_bytes": bucket.nbytes, "paged_adamw": opt,
    }
    del lins, bucket, hW, hdY, hY, hdX
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- paged AdamW
def bench_paged_adamw(args, lins, bucket, dev, flush, peaks):
    """The optimizer step after the block's backward: AdamW over the seven
    adapters (one flat vector, states in unified memory), with the states
    resident on the GPU, and after an eviction to host memory brought back
    by a prefetch before the step (the paged pattern around a memory
    spike)."""
    import torch
    from bit_quantized_lora_quantize_b200 import paged
    opt = paged.PagedAdamW([(l.K, l.N, l.r) for l in lins], dev, lr=2e-4, weight_decay=0.01)
    opt.load([(l.A, l.B) for l in lins])
    bucket.flat.normal_()
    for _ in range(3):
        opt.step(bucket.flat)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def timed(pre):
        evs = []
        for _ in range(args.steps):
            flush.zero_()
            if pre:
                opt.evict()
                torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if pre:
                opt.prefetch()
            opt.step(bucket.flat)
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize()
        return sorted(x.elapsed_time(y) * 1e3 for x, y in evs)[len(evs) // 2]

    us = timed(False)
    us_paged = timed(True)
    by = opt.n * (16 + 12 + 2)  # p, g, m, v read; p, m, v written; bf16 copy written
    gbs = by / (us * 1e-6) / 1e9
    return {"params": opt.n, "state_bytes": opt.state_bytes, "us_per_step": us, "gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "bytes_per_step": by,
                         "bytes_counted": "30 B per parameter (16 read, 14 written)",
                         "traffic": traffic_for("adamw_step/block")},
            "us_per_step_after_eviction": us_paged,
            "note": "after eviction: prefetch of the 3 state vectors host->GPU plus the step, device time"}


# ---------------------------------------------------------------- MLP trio
def bench_trio(args, q, synthetic, dev, flush, peaks, local_rank):
    import torch
    t = synthetic.mlp_trio()
    M, D, Fd, r, s = t.X.shape[0], t.X.shape[1], t.Wg.shape[0], t.Ag.shape[1], t.scale
    d = lambda x: x.to(dev)  # noqa: E731
    Pg, Pu, Pd = (q.qlora_quantize_nf4(d(w)) for w in (t.Wg, t.Wu, t.Wd))
    X, dY = d(t.X), d(t.dY)
    Ag, Au, Ad, Bg, Bu, Bd = (d(x) for x in (t.Ag, t.Au, t.Ad, t.Bg, t.Bu, t.Bd))
    wsg, wsu = q.new_workspace(M, D, Fd, r, dev), q.new_workspace(M, D, Fd, r, dev)
    wsd = q.new_workspace(M, Fd, D, r, dev)
    bf = torch.bfloat16
    G, Up = torch.empty(M, Fd, dtype=bf, device=dev), torch.empty(M, Fd, dtype=bf, device=dev)
    Tg, Tu, Td = (torch.empty(M, r, dtype=torch.float32, device=dev) for _ in range(3))
    Y = torch.empty(M, D, dtype=bf, device=dev)
    dH = torch.empty(M, Fd, dtype=bf, device=dev)
    H, dG, dU = (torch.empty(M, Fd, dtype=bf, device=dev) for _ in range(3))
    dXg, dXu = torch.empty(M, D, dtype=bf, device=dev), torch.empty(M, D, dtype=bf, device=dev)
    dX = torch.empty(M, D, dtype=bf, device=dev)
    gA = [torch.empty(k, r, dtype=torch.float32, device=dev) for k in (D, D, Fd)]
    gB = [torch.empty(r, n, dtype=torch.float32, device=dev) for n in (Fd, Fd, D)]
    calls = Calls()
    fl = lambda K, N: 2 * M * N * K + 2 * M * r * (N + K)  # noqa: E731

    comp = torch.cuda.current_stream()
    aux = None if args.one_stream else torch.cuda.Stream()

    def pair(f_gate, f_up):
        # gate and up are independent: with a second stream they run side by
        # side (their partial last waves overlap), joined before the glue.
        if aux is None:
            f_gate()
            f_up()
            return
        aux.wait_stream(comp)
        f_gate()
        with torch.cuda.stream(aux):
            f_up()
        comp.wait_stream(aux)

    def step():
        pair(lambda: calls("fused_nf4_fwd", "gate", {"flops": fl(D, Fd)},
                           lambda: q.qlora_linear_fwd(X, Pg, Ag, Bg, s, workspace=wsg, Y=G, T_save=Tg)),
             lambda: calls("fused_nf4_fwd", "up", {"flops": fl(D, Fd)},
                           lambda: q.qlora_linear_fwd(X, Pu, Au, Bu, s, workspace=wsu, Y=Up, T_save=Tu)))
        calls("silu_gate_fwd", "trio", {"bytes": 3 * 2 * M * Fd}, lambda: q.qlora_silu_gate_fwd(G, Up, H))
        calls("fused_nf4_fwd", "down", {"flops": fl(Fd, D)},
              lambda: q.qlora_linear_fwd(H, Pd, Ad, Bd, s, workspace=wsd, Y=Y, T_save=Td))
        calls("fused_nf4_dx", "down", {"flops": fl(Fd, D)},
              lambda: q.qlora_linear_bwd(dY, H, Td, Pd, Ad, Bd, s, workspace=wsd, dX=dH, dA=gA[2], dB=gB[2]))
        calls("silu_gate_bwd", "trio", {"bytes": 5 * 2 * M * Fd}, lambda: q.qlora_silu_gate_bwd(G, Up, dH, dG, dU))
        pair(lambda: calls("fused_nf4_dx", "gate", {"flops": fl(D, Fd)},
                           lambda: q.qlora_linear_bwd(dG, X, Tg, Pg, Ag, Bg, s, workspace=wsg, dX=dXg, dA=gA[0],
                                                      dB=gB[0])),
             lambda: calls("fused_nf4_dx", "up", {"flops": fl(D, Fd)},
                           lambda: q.qlora_linear_bwd(dU, X, Tu, Pu, Au, Bu, s, workspace=wsu, dX=dXu, dA=gA[1],
                                                      dB=gB[1])))
        torch.add(dXg, dXu, out=dX)  # the input's two gradient paths (torch add, bf16)

    fl_step = 2 * (flops_fwd(M, D, Fd, r) + flops_bwd(M, D, Fd, r)) + flops_fwd(M, Fd, D, r) + flops_bwd(M, Fd, D, r)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    ms, clocks = time_steps(step, args.steps, flush, 1, local_rank)
    aux_saved, aux = aux, None  # per-launch events on one stream
    agg = calls.profile(step, args.steps, flush)
    aux = aux_saved
    hX, hdY = t.X.pin_memory(), t.dY.pin_memory()
    hY = torch.empty(Y.shape, dtype=bf).pin_memory()
    hdX = torch.empty(M, D, dtype=bf).pin_memory()

    def e2e_step():
        X.copy_(hX, non_blocking=True)
        dY.copy_(hdY, non_blocking=True)
        step()
        hY.copy_(Y, non_blocking=True)
        hdX.copy_(dX, non_blocking=True)

    e2e_ms = time_e2e(e2e_step, args.steps, 1)
    for w in (wsg, wsu, wsd):
        if q.qlora_check_status(w) != 0:
            raise RuntimeError("device pipeline timeout (trio)")
    res = {"workload": "llama7b_mlp_trio", "M": M, "D": D, "F": Fd, "r": r, "scale": s,
           "step": "linear_fwd gate, up; silu_gate_fwd; linear_fwd down; linear_bwd down; silu_gate_bwd; "
                   "linear_bwd gate, up; dX = dX_gate + dX_up (torch add) (weights quantized once, outside the step)",
           "value": fl_step / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
           "tokens_per_s": M / (ms * 1e-3), "clocks": clocks, "kernels": kernel_table(agg),
           "roofline": gemm_roofline(agg, peaks, sustained=True), "gpu_launches": 8 * args.steps,
           "e2e": {"value": fl_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                   "h2d_bytes_per_step": (hX.numel() + hdY.numel()) * 2,
                   "d2h_bytes_per_step": (hY.numel() + hdX.numel()) * 2, "ms_per_step": e2e_ms},
           "l2": L2_NOTE}
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- attention projection
def bench_attn(args, q, synthetic, dev, flush, peaks, local_rank):
    import torch
    case = synthetic.attn_proj_case()
    lin = Linear(q, case, "attn_proj", dev)
    lin.X = case.X.to(dev)
    calls = Calls()
    fl = 2 * lin.M * lin.N * lin.K + 2 * lin.M * lin.r * (lin.N + lin.K)

    def step():
        calls("quantize_nf4", "attn_proj", {"bytes": quantize_bytes(lin.numel)},
              lambda: q.qlora_quantize_nf4(lin.W, out=lin.P))
        calls("fused_nf4_fwd", "attn_proj", {"flops": fl},
              lambda: q.qlora_linear_fwd(lin.X, lin.P, lin.A, lin.B, lin.s, workspace=lin.ws, Y=lin.Y, T_save=lin.T))
        calls("fused_nf4_dx", "attn_proj", {"flops": fl},
              lambda: q.qlora_linear_bwd(lin.dY, lin.X, lin.T, lin.P, lin.A, lin.B, lin.s, workspace=lin.ws,
                                         dX=lin.dX, dA=lin.dA, dB=lin.dB))

    fl_step = flops_fwd(lin.M, lin.K, lin.N, lin.r) + flops_bwd(lin.M, lin.K, lin.N, lin.r)
    for _ in range(max(3, args.warmup)):
        step()
    ms, _ = time_steps(step, args.steps, flush, 1, local_rank, sample_clocks=False)
    agg = calls.profile(step, args.steps, flush)
    if q.qlora_check_status(lin.ws) != 0:
        raise RuntimeError("device pipeline timeout (attn_proj)")
    res = {"workload": "llama7b_attn_proj_qlora_linear", "M": lin.M, "K": lin.K, "N": lin.N, "r": lin.r,
           "outliers": "0.1% x10", "step": "quantize_nf4 + linear_fwd + linear_bwd",
           "value": fl_step / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
           "tokens_per_s": lin.M / (ms * 1e-3), "kernels": kernel_table(agg), "roofline": gemm_roofline(agg, peaks)}
    del lin
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------- single small layer
def bench_tiny(args, q, synthetic, dev, flush, iters=50):
    """The small parity case (W 256 x 256, 16 tokens, r = 8, scale 2):
    microseconds per quantize + forward + backward, each iteration after an
    L2 flush.  Launch-bound: three launches per step."""
    import torch
    case = synthetic.tiny_case()
    W = case.W.to(dev)
    X, A, B, dY = (t.to(dev) for t in (case.X, case.A, case.B, case.dY))
    ws = q.new_workspace(case.M, case.K, case.N, case.r, dev)
    Wp = q.qlora_quantize_nf4(W)
    Y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device=dev)
    T = torch.empty(case.M, case.r, dtype=torch.float32, device=dev)
    dX = torch.empty(case.M, case.K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(case.K, case.r, dtype=torch.float32, device=dev)
    dB = torch.empty(case.r, case.N, dtype=torch.float32, device=dev)

    def step():
        q.qlora_quantize_nf4(W, out=Wp)
        q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws, Y=Y, T_save=T)
        q.qlora_linear_bwd(dY, X, T, Wp, A, B, case.scale, workspace=ws, dX=dX, dA=dA, dB=dB)

    for _ in range(5):
        step()
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for i in range(iters):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if q.qlora_check_status(ws) != 0:
        raise RuntimeError("device pipeline timeout (tiny)")
    us = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)[iters // 2]
    fl = flops_fwd(case.M, case.K, case.N, case.r) + flops_bwd(case.M, case.K, case.N, case.r)
    return {"workload": "single_qlora_linear_256x256", "M": case.M, "K": case.K, "N": case.N, "r": case.r,
            "step": "quantize_nf4 + linear_fwd + linear_bwd", "us_per_step": us, "launches_per_step": 3,
            "gflops": fl / (us * 1e-6) / 1e9, "note": "launch-bound (median of 50 steps, L2 flushed)"}


# ---------------------------------------------------------------- small-M sweep
def weight_copies(Wp, nbytes, l2_bytes, at_least=4):
    """Wp and clones of it at distinct addresses, together at least three
    times the L2 size, so that a weight used once per rotation has left L2
    before its next use (L2 lines are physical: equal contents do not share)."""
    import dataclasses

    n = max(at_least, -(-3 * l2_bytes // nbytes))
    return [Wp] + [dataclasses.replace(Wp, codes=Wp.codes.clone(), absmax_q=Wp.absmax_q.clone(),
                                       absmax_scale=Wp.absmax_scale.clone()) for _ in range(n - 1)]


def small_m_sweep(q, synthetic, dev, flush, iters=10):
    """Small-M forward (W [N x 8192] NF4, M tokens, r = 64): NF4 weight bytes
    streamed per second, L2 flushed before every timed call (`us`).  Also
    `us_back_to_back`: calls on copies of the weight in turn, at least three
    times the L2 size in all (12 x 34.6 MB or 5 x 93 MB on B200), so that
    each call reads its weight from HBM, between one pair of events, per
    call -- what a decode loop over layers sees, without one event pair's
    launch latency per call."""
    import torch

    peaks = load_peaks()
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or (126 << 20)
    out = []
    for N in (8192, 22016):
        W = synthetic.weight_only(N, 8192, seed=4).to(dev)
        Wp = q.qlora_quantize_nf4(W)
        del W
        nb = nf4_bytes(N * 8192)
        Wps = weight_copies(Wp, nb, l2)
        for M in (1, 4, 16, 64):
            case = synthetic.small_m_case(M, N)
            X, A, B = (t.to(dev) for t in (case.X, case.A, case.B))
            ws = q.new_workspace(M, 8192, N, 64, dev)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            T = torch.empty(M, 64, dtype=torch.float32, device=dev)
            for _ in range(3):
                q.qlora_linear_fwd(X, Wp, A, B, 0.25, workspace=ws, Y=Y, T_save=T)
            stream = torch.cuda.current_stream()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
            for i in range(iters):
                flush.zero_()
                evs[i][0].record(stream)
                q.qlora_linear_fwd(X, Wp, A, B, 0.25, workspace=ws, Y=Y, T_save=T)
                evs[i][1].record(stream)
            torch.cuda.synchronize()
            us = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)[iters // 2]
            gbs = nb / (us * 1e-6) / 1e9
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush.zero_()
            e0.record(stream)
            for _ in range(iters):
                for w in Wps:
                    q.qlora_linear_fwd(X, w, A, B, 0.25, workspace=ws, Y=Y, T_save=T)
            e1.record(stream)
            torch.cuda.synchronize()
            us_b2b = e0.elapsed_time(e1) * 1e3 / (iters * len(Wps))
            out.append({"N": N, "K": 8192, "M": M, "us": us, "nf4_weight_gbs": gbs,
                        "frac_hbm": gbs / peaks["hbm_gbs"], "nf4_bytes": nb,
                        "us_back_to_back": us_b2b, "back_to_back_copies": len(Wps),
                        "frac_hbm_back_to_back": nb / (us_b2b * 1e-6) / 1e9 / peaks["hbm_gbs"],
                        "kernel": "small_m_nf4_fwd" if M <= 128 else "fused_nf4_fwd"})
            if q.qlora_check_status(ws) != 0:
                raise RuntimeError("device pipeline timeout (small M)")
    return out


# ---------------------------------------------------------------- driver
def run_ours(args, rank, world, local_rank):
    import torch

    import bit_quantized_lora_quantize_b200 as q
    from bit_quantized_lora_quantize_b200 import build as qbuild, dp, synthetic

    qbuild.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2 (126 MB)

    blk = bench_block(args, q, synthetic, dp, dev, rank, world, local_rank, flush, peaks)
    extra = rank == 0 and world == 1
    trio = bench_trio(args, q, synthetic, dev, flush, peaks, local_rank) if extra and not args.block_only else None
    attn = bench_attn(args, q, synthetic, dev, flush, peaks, local_rank) if extra and not args.block_only else None
    small_m = small_m_sweep(q, synthetic, dev, flush) if (extra and not args.no_small_m) else None
    tiny = bench_tiny(args, q, synthetic, dev, flush) if extra and not args.block_only else None
    if rank != 0:
        return
    cpu = cpu_oracle_block_sample(rows=256, slab=256) if (world == 1 and not args.no_cpu_baseline) else None
    line = {
        "metric": METRIC, "value": blk["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": blk["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(BLOCK_WORKLOAD, parallelism=f"dp{world}", global_batch_tokens=M_BLOCK * world, l2=L2_NOTE,
                       streams=1 if args.one_stream else 2),
        "tokens_per_s": blk["tokens_per_s"], "tflops_dense_only": blk["tflops_dense_only"],
        "flops_per_step": blk["flops_per_step"],
        "roofline": blk["roofline"], "roofline_quantize": blk["roofline_quantize"],
        "kernels": blk["kernels"], "gpu_launches": blk["gpu_launches"], "e2e": blk["e2e"],
        "clocks": blk["clocks"], "cpu_baseline": cpu,
        "grad_allreduce_bytes_per_step": blk["grad_bucket_bytes"] if world > 1 else 0,
        "paged_adamw": blk["paged_adamw"],
        "mlp_trio": trio, "attn_proj": attn, "small_m": small_m, "tiny": tiny,
    }
    print(json.dumps(line), flush=True)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def torchrun_argv(argv, gpus, port):
    """The command that re-runs this script with one process per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + list(argv)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-small-m", action="store_true")
    ap.add_argument("--block-only", action="store_true", help="only the headline block step")
    ap.add_argument("--one-stream", action="store_true", help="the block's linears one after another on one stream")
    args = ap.parse_args(argv)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # One process per GPU: re-launch under torch.distributed.run.
        env = dict(os.environ)
        env.setdefault("NCCL_DEBUG", "INFO")
        env.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
        return subprocess.call(torchrun_argv(argv, args.gpus, _free_port()), env=env)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one process per GPU")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

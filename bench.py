"""Benchmark of the frozen-NF4 LoRA linear layer on B200.

One step = the whole hot path on one batch: NF4 quantization of the frozen
weight (with double-quantized constants), the forward (T = s X A and the
fused dequant-GEMM Y = X W'^T + T B) and the backward (U, dB, the fused
dequant-GEMM dX = dY W' + U A^T, dA), through the C ABI of libqlora.so.

Workload (N = 1): the LLaMA-7B attention projection, W 4096 x 4096 bf16
~N(0, 0.02^2) with 0.1% of entries x10, 4096 tokens, r = 64, scale 0.25,
seeded synthetic data.  With --gpus N (torchrun, one process per GPU) every
rank runs its own batch of 4096 tokens (weak scaling) and the adapter
gradients dA, dB are summed over ranks with one NCCL all-reduce per step
(the data-parallel exchange).

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle (the
float64 restatement in oracle/) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s & tokens/s; small-M NF4 weight GB/s vs HBM peak"
WORKLOAD = dict(workload="llama7b_attn_proj_qlora_linear", M=4096, K=4096, N=4096, r=64, scale=0.25,
                outliers="0.1% x10", step="quantize_nf4 + linear_fwd + linear_bwd")


def flops_fwd(M, K, N, r):
    return 2 * M * N * K + 2 * M * r * (K + N)


def flops_bwd(M, K, N, r):
    return 2 * M * N * K + 4 * M * r * (K + N)


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


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


def cpu_oracle_sample(budget_rows: int = 1024):
    """Time the oracle on a bounded sample of the workload: quantize the whole
    4096 x 4096 weight, then forward + backward on `budget_rows` token rows."""
    import numpy as np
    from bit_quantized_lora_quantize_b200 import synthetic
    from oracle import dequantize_nf4, lora_linear_backward, lora_linear_forward, quantize_nf4

    case = synthetic.attn_proj_case()
    M, K, N, r = budget_rows, case.K, case.N, case.r
    W = case.W.float().numpy()
    X = case.X[:M].double().numpy()
    dY = case.dY[:M].double().numpy()
    A = case.A.double().numpy()
    B = case.B.double().numpy()
    t0 = time.perf_counter()
    codes, aq, sc = quantize_nf4(W)
    Wdq = dequantize_nf4(codes, aq, sc, W.size).reshape(N, K)
    lora_linear_forward(X, Wdq, A, B, case.scale)
    lora_linear_backward(dY, X, Wdq, A, B, case.scale)
    dt = time.perf_counter() - t0
    fl = flops_fwd(M, K, N, r) + flops_bwd(M, K, N, r)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    return {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": int(cores), "kind": "oracle",
            "sample": f"quantize of the full 4096x4096 weight + fwd+bwd on {M} of 4096 token rows (float64 numpy)",
            "seconds": dt, "tokens_per_s": M / dt}


def run_reference(args, rank, world):
    if rank != 0:
        return
    vals = []
    for _ in range(args.warmup):
        cpu_oracle_sample(256)
    samples = []
    for _ in range(args.steps):
        s = cpu_oracle_sample(512)
        samples.append(s)
        vals.append(s["value"])
    v = sorted(vals)[len(vals) // 2]
    cb = dict(samples[-1])
    cb["value"] = v
    # The whole step's flops at the sample's rate: the time one full step would take.
    M, K, N, r = WORKLOAD["M"], WORKLOAD["K"], WORKLOAD["N"], WORKLOAD["r"]
    ms_full = (flops_fwd(M, K, N, r) + flops_bwd(M, K, N, r)) / (v * 1e12) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_full, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(WORKLOAD), "cpu_baseline": cb, "tokens_per_s": M / (ms_full * 1e-3),
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def traffic_for(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it still
    describes the current kernel source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        ent = t[kernel]
        hsh = hashlib.sha256()
        for name in ent["sources"]:  # the kernel's .cu file and the headers it includes
            with open(os.path.join(ROOT, "bit_quantized_lora_quantize_b200", "csrc", name), "rb") as f:
                hsh.update(f.read())
        if hsh.hexdigest()[:16] != ent["sources_sha256_16"]:
            return None
        return ent["dram_bytes_per_launch"]
    except Exception:
        return None


def small_m_sweep(q, synthetic, dev, flush, iters=10):
    """Small-M forward (W [N x 8192] NF4, M tokens, r = 64): NF4 weight bytes
    streamed per second, L2 flushed before every timed call."""
    import torch

    peaks = load_peaks()
    out = []
    for N in (8192, 22016):
        W = synthetic.weight_only(N, 8192, seed=4).to(dev)
        Wp = q.qlora_quantize_nf4(W)
        del W
        nf4_bytes = Wp.codes.numel() + Wp.absmax_q.numel() + 4 * Wp.absmax_scale.numel()
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
            q.qlora_profile_start()
            for i in range(iters):
                flush.zero_()
                evs[i][0].record(stream)
                q.qlora_linear_fwd(X, Wp, A, B, 0.25, workspace=ws, Y=Y, T_save=T)
                evs[i][1].record(stream)
            torch.cuda.synchronize()
            prof = q.qlora_profile_stop()
            us = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)[iters // 2]
            gbs = nf4_bytes / (us * 1e-6) / 1e9
            ent = {"N": N, "K": 8192, "M": M, "us": us, "nf4_weight_gbs": gbs,
                   "frac_hbm": gbs / peaks["hbm_gbs"], "nf4_bytes": nf4_bytes}
            # The weight-streaming kernel alone (mean over the timed calls).
            for name, (ms, calls, _) in prof.items():
                if name in ("small_m_nf4_fwd", "fused_nf4_fwd"):
                    k_us = ms * 1e3 / max(calls, 1)
                    ent.update({"kernel": name, "kernel_us": k_us,
                                "kernel_frac_hbm": nf4_bytes / (k_us * 1e-6) / 1e9 / peaks["hbm_gbs"]})
            out.append(ent)
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_quantized_lora_quantize_b200 as q
    from bit_quantized_lora_quantize_b200 import build as qbuild, dp, synthetic

    qbuild.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    case = synthetic.attn_proj_case() if rank == 0 else synthetic.linear_case(
        4096, 4096, 4096, 64, 0.25, 1 + 1000 * rank, outlier_frac=0.001)
    M, K, N, r, s = case.M, case.K, case.N, case.r, case.scale
    W = case.W.to(dev)
    X, A, B, dY = (t.to(dev) for t in (case.X, case.A, case.B, case.dY))
    ws = q.new_workspace(M, K, N, r, dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    T = torch.empty(M, r, dtype=torch.float32, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(K, r, dtype=torch.float32, device=dev)
    dB = torch.empty(r, N, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2 (126 MB)
    reducer = dp.AdapterGradReducer(K, N, r, dev) if world > 1 else None

    def step():
        Wp = q.qlora_quantize_nf4(W)
        q.qlora_linear_fwd(X, Wp, A, B, s, workspace=ws, Y=Y, T_save=T)
        q.qlora_linear_bwd(dY, X, T, Wp, A, B, s, workspace=ws, dX=dX, dA=dA, dB=dB)
        if reducer is not None:
            reducer(dA, dB)
        return Wp

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if q.qlora_check_status(ws) != 0:
        raise RuntimeError("device pipeline timeout during warm-up")

    # ---------------- device-resident timing (kernels only), L2 flushed between steps
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    # Per-kernel durations (roofline, kernel table): the same K steps again
    # with CUDA events recorded around every launch on the launching stream.
    # Kept out of the timed steps above, because an event between two kernels
    # stops the next one from starting before the previous one ends.
    q.qlora_profile_start()
    for i in range(args.steps):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    prof = q.qlora_profile_stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = sum(step_ms)
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    fl_step = flops_fwd(M, K, N, r) + flops_bwd(M, K, N, r)
    value = fl_step * world / (ms_per_step * 1e-3) / 1e12
    tokens_per_s = M * world / (ms_per_step * 1e-3)
    # The same step time with only the dense products counted (4MNK: the
    # frozen-weight GEMMs of forward and input gradient).
    value_dense = 4 * M * N * K * world / (ms_per_step * 1e-3) / 1e12

    # ---------------- end to end through the public API with host buffers
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    hW, hX, hdY = pin(case.W), pin(case.X), pin(case.dY)
    hdA = torch.empty(K, r, dtype=torch.float32).pin_memory()
    hdB = torch.empty(r, N, dtype=torch.float32).pin_memory()
    h2d = hW.numel() * 2 + hX.numel() * 2 + hdY.numel() * 2
    d2h = hdA.numel() * 4 + hdB.numel() * 4

    def e2e_step():
        W.copy_(hW, non_blocking=True)
        X.copy_(hX, non_blocking=True)
        dY.copy_(hdY, non_blocking=True)
        step()
        hdA.copy_(dA, non_blocking=True)
        hdB.copy_(dB, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_ms = float(t.item()) / args.steps
    e2e_value = fl_step * world / (e2e_ms * 1e-3) / 1e12
    if q.qlora_check_status(ws) != 0:
        raise RuntimeError("device pipeline timeout during timing")

    small_m = small_m_sweep(q, synthetic, dev, flush) if (rank == 0 and not args.no_small_m) else None

    if rank != 0:
        return
    peaks = load_peaks()
    # Dominant kernel: the fused dequant-GEMM with the larger total time.
    fused = {k: v for k, v in prof.items() if k.startswith("fused_nf4")}
    dom = max(fused, key=lambda k: fused[k][0])
    dom_ms = fused[dom][0] / fused[dom][1]
    # Each fused launch also computes its rank-r intermediate (T = s X A in the
    # forward, U = s dY B^T in the input gradient) besides the LoRA product.
    dom_flops = 2 * M * N * K + 2 * M * r * (N + K)
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    launches = sum(v[2] for v in prof.values())
    kernels = {k: {"ms_per_call": v[0] / v[1], "calls": v[1], "share": v[0] / sum(x[0] for x in prof.values())}
               for k, v in prof.items()}
    cpu = cpu_oracle_sample(512) if (world == 1 and not args.no_cpu_baseline) else None
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(WORKLOAD, parallelism=f"dp{world}", global_batch_tokens=M * world,
                       l2="flushed between timed steps (256 MB write)"),
        "tokens_per_s": tokens_per_s,
        "tflops_dense_only": value_dense,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": traffic_for(dom),
                     "peak_source": f"{peaks['source']} bf16 burst", "ms_per_launch": dom_ms},
        "kernels": kernels,
        "gpu_launches": launches,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "clocks": clocks,
        "cpu_baseline": cpu,
        "small_m": small_m,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-small-m", action="store_true")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
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


if __name__ == "__main__":
    main()

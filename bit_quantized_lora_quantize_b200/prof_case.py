"""Run one library call on a seeded synthetic case, a few times, for profiling.

    python -m bit_quantized_lora_quantize_b200.prof_case quantize --n 22016 --k 8192
    python -m bit_quantized_lora_quantize_b200.prof_case fwd --m 16 --n 8192 --k 8192
    python -m bit_quantized_lora_quantize_b200.prof_case bwd --m 4096 --n 4096 --k 4096
    python -m bit_quantized_lora_quantize_b200.prof_case adamw --n 9994240
    python -m bit_quantized_lora_quantize_b200.prof_case silu --m 8192 --n 11008

Each case makes its inputs once, runs `--warmup` calls, then `--iters` calls
with a 256 MB buffer written between them (so the weight is read from HBM, not
from L2), and prints the mean device time per call measured with CUDA events.
A profiler attached to this process sees exactly the library's kernels plus
the flush writes.
"""

import argparse

import torch

from . import qlora as q
from . import synthetic


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("op", choices=["quantize", "dequantize", "fwd", "bwd", "adamw", "silu"])
    ap.add_argument("--m", type=int, default=4096, help="tokens")
    ap.add_argument("--n", type=int, default=4096, help="weight rows (out features)")
    ap.add_argument("--k", type=int, default=4096, help="weight columns (in features)")
    ap.add_argument("--r", type=int, default=64)
    ap.add_argument("--scale", type=float, default=0.25)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=7)
    a = ap.parse_args(argv)

    dev = "cuda:0"
    torch.cuda.set_device(0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    if a.op == "adamw":
        # a flat parameter vector of n (the block's adapters: 9994240)
        from . import paged
        opt = paged.PagedAdamW([(a.n, 0, 1)], dev, lr=2e-4, weight_decay=0.01)
        g = torch.randn(a.n, device=dev)
        call = lambda: opt.step(g)  # noqa: E731
    elif a.op == "silu":
        G = torch.randn(a.m, a.n, device=dev).to(torch.bfloat16)
        U = torch.randn(a.m, a.n, device=dev).to(torch.bfloat16)
        H = torch.empty_like(G)
        call = lambda: q.qlora_silu_gate_fwd(G, U, H)  # noqa: E731
    elif a.op in ("quantize", "dequantize"):
        W = synthetic.weight_only(a.n, a.k, seed=a.seed).to(dev)
        Wp = q.qlora_quantize_nf4(W)
        if a.op == "quantize":
            call = lambda: q.qlora_quantize_nf4(W, out=Wp)  # noqa: E731
        else:
            Wd = torch.empty_like(W)
            call = lambda: q.qlora_dequantize_nf4(Wp, out=Wd)  # noqa: E731
    else:
        case = synthetic.linear_case(a.m, a.k, a.n, a.r, a.scale, seed=a.seed)
        Wp = q.qlora_quantize_nf4(case.W.to(dev))
        X, A, B, dY = (t.to(dev) for t in (case.X, case.A, case.B, case.dY))
        ws = q.new_workspace(a.m, a.k, a.n, a.r, dev)
        Y, T = q.qlora_linear_fwd(X, Wp, A, B, a.scale, workspace=ws)
        if a.op == "fwd":
            call = lambda: q.qlora_linear_fwd(X, Wp, A, B, a.scale, workspace=ws, Y=Y, T_save=T)  # noqa: E731
        else:
            call = lambda: q.qlora_linear_bwd(dY, X, T, Wp, A, B, a.scale, workspace=ws)  # noqa: E731
    for _ in range(a.warmup):
        call()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(a.iters):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    print(f"{a.op} m={a.m} n={a.n} k={a.k} r={a.r}: {total / a.iters * 1e3:.1f} us per call")


if __name__ == "__main__":
    main()

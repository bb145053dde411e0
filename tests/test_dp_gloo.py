"""Data-parallel exchange on CPU: two gloo ranks each take their share of the
tokens, compute the adapter gradients of two linears with the oracle into
views of one gradient bucket (the structure the benchmark's backward writes
into), sum the bucket with its all-reduce, and must reproduce the full-batch
gradients."""

import datetime
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_quantized_lora_quantize_b200 import dp, synthetic


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from oracle import dequantize_nf4, lora_linear_backward, quantize_nf4

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # Two linears of different shapes share one bucket, as the block
        # step's seven linears do.
        cases = [synthetic.linear_case(37, 128, 96, 8, 0.5, seed=77),
                 synthetic.linear_case(37, 64, 200, 16, 0.25, seed=78)]
        bucket = dp.GradBucket([(c.K, c.N, c.r) for c in cases], "cpu")
        rows = dp.shard_rows(cases[0].M, rank, world)
        fulls = []
        for i, case in enumerate(cases):
            codes, aq, sc = quantize_nf4(case.W.float().numpy())
            Wdq = dequantize_nf4(codes, aq, sc, case.W.numel()).reshape(case.N, case.K)
            X = case.X[rows].double().numpy()
            dY = case.dY[rows].double().numpy()
            A, B = case.A.double().numpy(), case.B.double().numpy()
            _, dA, dB = lora_linear_backward(dY, X, Wdq, A, B, case.scale)
            vA, vB = bucket[i]
            vA.copy_(torch.from_numpy(dA.astype(np.float32)))
            vB.copy_(torch.from_numpy(dB.astype(np.float32)))
            if rank == 0:
                _, fA, fB = lora_linear_backward(case.dY.double().numpy(), case.X.double().numpy(), Wdq, A, B,
                                                 case.scale)
                fulls.append((fA, fB))
        bucket.all_reduce()
        if rank == 0:
            errs = []
            for i, (fA, fB) in enumerate(fulls):
                vA, vB = bucket[i]
                errs.append(float(np.max(np.abs(vA.numpy() - fA)) / np.sqrt(np.mean(fA ** 2))))
                errs.append(float(np.max(np.abs(vB.numpy() - fB)) / np.sqrt(np.mean(fB ** 2))))
            out["errs"] = errs
    finally:
        dist.destroy_process_group()


def test_shard_rows_cover_all_tokens():
    for M in (1, 7, 4096, 4097):
        for world in (1, 2, 3, 8):
            parts = [dp.shard_rows(M, r, world) for r in range(world)]
            assert parts[0].start == 0 and parts[-1].stop == M
            assert all(a.stop == b.start for a, b in zip(parts, parts[1:]))
            sizes = [p.stop - p.start for p in parts]
            assert max(sizes) - min(sizes) <= 1


def test_two_rank_gradient_sum_equals_full_batch():
    port = _free_port()
    # The result dict's server process is spawned like the ranks: forking a
    # process that already runs threads can deadlock the child.
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        assert len(out["errs"]) == 4 and max(out["errs"]) < 1e-5, out["errs"]

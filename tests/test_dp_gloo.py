"""Data-parallel exchange on CPU: two gloo ranks each take their share of the
tokens, compute the adapter gradients with the oracle, sum them with the
reducer the benchmark uses, and must reproduce the full-batch gradients."""

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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = synthetic.linear_case(37, 128, 96, 8, 0.5, seed=77)
        codes, aq, sc = quantize_nf4(case.W.float().numpy())
        Wdq = dequantize_nf4(codes, aq, sc, case.W.numel()).reshape(case.N, case.K)
        rows = dp.shard_rows(case.M, rank, world)
        X = case.X[rows].double().numpy()
        dY = case.dY[rows].double().numpy()
        _, dA, dB = lora_linear_backward(dY, X, Wdq, case.A.double().numpy(), case.B.double().numpy(), case.scale)
        tA = torch.from_numpy(dA.astype(np.float32))
        tB = torch.from_numpy(dB.astype(np.float32))
        dp.AdapterGradReducer(case.K, case.N, case.r, "cpu")(tA, tB)
        if rank == 0:
            _, fA, fB = lora_linear_backward(case.dY.double().numpy(), case.X.double().numpy(), Wdq,
                                             case.A.double().numpy(), case.B.double().numpy(), case.scale)
            out["errA"] = float(np.max(np.abs(tA.numpy() - fA)) / np.sqrt(np.mean(fA ** 2)))
            out["errB"] = float(np.max(np.abs(tB.numpy() - fB)) / np.sqrt(np.mean(fB ** 2)))
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
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        assert out["errA"] < 1e-5 and out["errB"] < 1e-5

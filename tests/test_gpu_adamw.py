"""The paged AdamW step of the LoRA parameters ("3. Paged Optimizers")
against the float64 oracle, with its states in unified memory resident on
the GPU, evicted to host memory, and prefetched back.

Tolerance: the kernel computes in float32 what the oracle computes in
float64; over a few steps each parameter may differ by a few float32
rounding errors of its update (lr-sized) and of itself, so |p - p_ref| <=
1e-5 * lr + 4 ulp_f32(p) elementwise (the update itself is lr-sized).  The
bf16 adapters must equal bf16_rne of the float32 master copy bit for bit.
"""

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import dp, paged, synthetic
from oracle import adamw_run, adamw_step, bf16_round, dequantize_nf4, lora_linear_backward, quantize_nf4
from tests.helpers import assert_close_rms, f32, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def assert_params_close(got, ref, lr):
    got = np.asarray(got, np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    bound = 1e-5 * lr + 4 * ulp
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{bad.sum()} params off: {got[bad][:4]} vs {ref[bad][:4]}"


def run_steps(opt, grads, evict):
    for g in grads:
        if evict:
            opt.evict()
        opt.step(g)
    torch.cuda.synchronize()


@pytest.mark.parametrize("n", [1 << 20 | 3, 1000])
def test_adamw_matches_oracle_resident_and_paged(n):
    rng = np.random.default_rng(n)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    gs = [rng.standard_normal(n).astype(np.float32) for _ in range(5)]
    lr, betas, eps, wd = 1e-3, (0.9, 0.95), 1e-8, 0.05
    results = []
    for evict in (False, True):
        opt = paged.PagedAdamW([(n, 0, 1)], DEV, lr=lr, betas=betas, eps=eps, weight_decay=wd)
        opt.master.copy_(torch.from_numpy(p0))
        run_steps(opt, [torch.from_numpy(g).to(DEV) for g in gs], evict)
        if evict:
            assert paged.location(opt.m) == -1  # last prefetch went to the host; the step paged it in
        results.append((opt.master.cpu().numpy().copy(), opt.m.cpu().numpy().copy(), opt.v.cpu().numpy().copy(),
                        opt.params.cpu()))
    # Where the states live does not change a bit of the result.
    for a, b in zip(results[0][:3], results[1][:3]):
        np.testing.assert_array_equal(a, b)
    p_ref, m_ref, v_ref = adamw_run(p0, gs, lr, betas[0], betas[1], eps, wd)
    p, m, v, pb = results[0]
    assert_params_close(p, p_ref, lr)
    np.testing.assert_allclose(m, m_ref, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(v, v_ref, rtol=1e-5, atol=1e-9)
    np.testing.assert_array_equal(f32(pb).view(np.uint32), bf16_round(p).view(np.uint32))


def test_unaligned_buffers_take_the_scalar_path():
    """Pointers one float past a 16-byte boundary: the element-wise path."""
    n = 777
    rng = np.random.default_rng(5)
    p0 = (rng.standard_normal(n + 1) * 0.02).astype(np.float32)
    g = rng.standard_normal(n + 1).astype(np.float32)
    p, gd = torch.from_numpy(p0).to(DEV), torch.from_numpy(g).to(DEV)
    m, v = torch.zeros(n + 1, device=DEV), torch.zeros(n + 1, device=DEV)
    pb = torch.zeros(n + 1, dtype=torch.bfloat16, device=DEV)
    st = q.lib().qlora_adamw_step(p.data_ptr() + 4, pb.data_ptr() + 2, gd.data_ptr() + 4, m.data_ptr() + 4,
                                  v.data_ptr() + 4, n, 1, 1e-3, 0.9, 0.999, 1e-8, 0.0,
                                  torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    p_ref, _, _ = adamw_step(p0[1:], g[1:], np.zeros(n), np.zeros(n), 1, 1e-3)
    got = p.cpu().numpy()
    assert got[0] == p0[0]
    assert_params_close(got[1:], p_ref, 1e-3)
    np.testing.assert_array_equal(f32(pb)[1:].view(np.uint32), bf16_round(got[1:]).view(np.uint32))


def test_prefetch_moves_the_states():
    opt = paged.PagedAdamW([(4096, 4096, 64)], DEV)
    opt.evict()
    torch.cuda.synchronize()
    assert paged.location(opt.master) == -1 and paged.location(opt.v) == -1
    opt.prefetch()
    torch.cuda.synchronize()
    assert paged.location(opt.master) == 0 and paged.location(opt.m) == 0


def test_training_step_of_two_linears():
    """Forward, backward into one gradient bucket, one paged AdamW step over
    both linears' adapters: the updated bf16 adapters the next forward reads
    equal the oracle's AdamW applied to the library's gradients, and those
    gradients match the float64 oracle."""
    cases = [synthetic.linear_case(300, 512, 384, 16, 0.5, seed=90),
             synthetic.linear_case(300, 384, 256, 8, 0.5, seed=91)]
    shapes = [(c.K, c.N, c.r) for c in cases]
    bucket = dp.GradBucket(shapes, DEV)
    opt = paged.PagedAdamW(shapes, DEV, lr=2e-4, weight_decay=0.01)
    opt.load([(c.A.to(DEV), c.B.to(DEV)) for c in cases])
    for i, c in enumerate(cases):
        Wp = q.qlora_quantize_nf4(c.W.to(DEV))
        A, B = opt.views[i]
        X, dY = c.X.to(DEV), c.dY.to(DEV)
        Y, T = q.qlora_linear_fwd(X, Wp, A, B, c.scale)
        dA, dB = bucket[i]
        q.qlora_linear_bwd(dY, X, T, Wp, A, B, c.scale, dA=dA, dB=dB)
        codes, aq, sc = quantize_nf4(f32(c.W))
        Wdq = dequantize_nf4(codes, aq, sc, c.W.numel()).reshape(c.N, c.K)
        _, rA, rB = lora_linear_backward(f64(c.dY), f64(c.X), Wdq, f64(c.A), f64(c.B), c.scale)
        assert_close_rms(f64(dA), rA, f"dA{i}")
        assert_close_rms(f64(dB), rB, f"dB{i}")
    opt.evict()  # a memory spike: the states go to the host before the step
    opt.step(bucket.flat)
    torch.cuda.synchronize()
    p0 = np.concatenate([np.concatenate([f32(c.A).ravel(), f32(c.B).ravel()]) for c in cases])
    p_ref, _, _ = adamw_step(p0, bucket.flat.cpu().numpy(), np.zeros_like(p0), np.zeros_like(p0), 1, 2e-4, wd=0.01)
    assert_params_close(opt.master.cpu().numpy(), p_ref, 2e-4)
    np.testing.assert_array_equal(f32(opt.params).view(np.uint32), bf16_round(opt.master.cpu().numpy()).view(np.uint32))
    # The adapters the layer reads are views of the updated buffer.
    A0, B0 = opt.views[0]
    assert A0.data_ptr() == opt.params.data_ptr() and B0.shape == (16, 384)

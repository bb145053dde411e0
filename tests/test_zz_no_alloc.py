"""The allocation-free forward entry point (qlora_linear_fwd_noalloc).

It serves callers that cannot allocate device memory: it takes its scratch
from a fixed array inside the library instead of a caller workspace.  This
file is named so that pytest collects it last; it must pass both alone in a
fresh process and after the other tests.  Two calls in a row are checked
against the regular qlora_linear_fwd and against the float64 oracle.  For
M > 128 both entry points run the same GEMM launch, so the outputs match bit
for bit; for M <= 128 this call still runs the pair GEMM (one partial
512-row block) while qlora_linear_fwd takes the weight-streaming kernel, so
the bar there is the parity tolerance.  A pipeline wait that runs out inside
this call is reported by qlora_check_status(NULL)."""

import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import dequantize_nf4, lora_linear_forward, quantize_nf4
from tests.helpers import REL_RMS_TOL, assert_close_rms, f32, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def call_noalloc(X, Wp, A, B, s, Y, T):
    L = q.lib()
    M, K = X.shape
    N = Wp.shape[0]
    r = A.shape[1]
    return L.qlora_linear_fwd_noalloc(X.data_ptr(), M, K, N, Wp.codes.data_ptr(), Wp.absmax_q.data_ptr(),
                                      Wp.absmax_scale.data_ptr(), A.data_ptr(), B.data_ptr(), r, ctypes.c_float(s),
                                      Y.data_ptr(), T.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,K,N,r,s", [(4096, 4096, 4096, 64, 0.25), (200, 320, 264, 16, 0.5),
                                       (1, 4096, 1000, 8, 0.5), (1, 4096, 1000, 64, 0.25),
                                       (16, 4096, 1000, 8, 0.5), (16, 4096, 1000, 64, 0.25),
                                       (64, 4096, 1000, 64, 0.25), (128, 4096, 1000, 8, 0.5),
                                       (128, 4096, 1000, 64, 0.25)])
def test_noalloc_forward_matches_regular_forward_twice(M, K, N, r, s):
    case = synthetic.linear_case(M, K, N, r, s, seed=31 + M + r, outlier_frac=0.001)
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B = (t.to(DEV) for t in (case.X, case.A, case.B))
    Y_ref, T_ref = q.qlora_linear_fwd(X, Wp, A, B, s)
    codes, aq, sc = quantize_nf4(f32(case.W))
    Wdq = dequantize_nf4(codes, aq, sc, case.W.numel()).reshape(N, K)
    rows = np.arange(M) if M <= 512 else np.sort(np.random.default_rng(7).choice(M, 256, replace=False))
    Yo, To = lora_linear_forward(f64(case.X)[rows], Wdq, f64(case.A), f64(case.B), s)
    for _ in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        T = torch.full((M, r), float("nan"), dtype=torch.float32, device=DEV)
        assert call_noalloc(X, Wp, A, B, s, Y, T) == 0
        torch.cuda.synchronize()
        assert_close_rms(f64(Y)[rows], Yo, "Y vs oracle")
        assert_close_rms(f64(T)[rows], To, "T vs oracle")
        # Both entry points are within the tolerance of the oracle, so they
        # are within twice of it of each other (two bf16 results may differ
        # by a whole ulp where each is within half an ulp of the exact sum).
        assert_close_rms(f64(Y), f64(Y_ref), "Y vs qlora_linear_fwd", tol=2 * REL_RMS_TOL)
        assert_close_rms(f64(T), f64(T_ref), "T vs qlora_linear_fwd", tol=2 * REL_RMS_TOL)
        if M > 128:  # the same GEMM launch as the regular forward
            assert torch.equal(Y, Y_ref) and torch.equal(T, T_ref)
    assert q.qlora_check_status(None) == 0


def test_noalloc_timeout_is_reported_and_clears():
    """With a 1 us wait limit the epilogue's wait for a 4096^3 accumulator
    (tens of microseconds of main loop) must give up: the call's status word
    inside the library is set, qlora_check_status(NULL) reports it once, and
    with the default limit the next calls give the regular forward's bits."""
    M = K = N = 4096
    r, s = 64, 0.25
    case = synthetic.linear_case(M, K, N, r, s, seed=77)
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B = (t.to(DEV) for t in (case.X, case.A, case.B))
    Y_ref, T_ref = q.qlora_linear_fwd(X, Wp, A, B, s)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    T = torch.empty(M, r, dtype=torch.float32, device=DEV)
    assert q.qlora_check_status(None) == 0
    q.qlora_set_wait_timeout(1000)
    try:
        assert call_noalloc(X, Wp, A, B, s, Y, T) == 0
        assert q.qlora_check_status(None) == 6
    finally:
        q.qlora_set_wait_timeout(0)
    assert q.qlora_check_status(None) == 0
    for _ in range(2):
        assert call_noalloc(X, Wp, A, B, s, Y, T) == 0
        assert q.qlora_check_status(None) == 0
        assert torch.equal(Y, Y_ref) and torch.equal(T, T_ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    M, K, N, r = 65536, 4096, 256, 128  # needs far more than the fixed scratch
    X = torch.zeros(16, dtype=torch.bfloat16, device=DEV)  # never read: the call must fail first
    ptr = X.data_ptr()
    L = q.lib()
    st = L.qlora_linear_fwd_noalloc(ptr, M, K, N, ptr, ptr, ptr, ptr, ptr, r, ctypes.c_float(1.0), ptr, ptr,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == 4  # QLORA_ERR_WORKSPACE

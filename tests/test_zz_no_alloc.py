"""The allocation-free forward entry point (qlora_linear_fwd_noalloc).

It serves callers that cannot allocate device memory: it takes its scratch
from a fixed array inside the library instead of a caller workspace.  This
file is named so that pytest collects it last; it must pass both alone in a
fresh process and after the other tests.  Two calls in a row are checked
against the regular qlora_linear_fwd (same kernels, so the outputs are
expected to match bit for bit; the bar is the parity tolerance)."""

import ctypes

import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from tests.helpers import assert_close_rms, f64

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


@pytest.mark.parametrize("M,K,N,r,s", [(4096, 4096, 4096, 64, 0.25), (200, 320, 264, 16, 0.5)])
def test_noalloc_forward_matches_regular_forward_twice(M, K, N, r, s):
    case = synthetic.linear_case(M, K, N, r, s, seed=31 + M, outlier_frac=0.001)
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B = (t.to(DEV) for t in (case.X, case.A, case.B))
    Y_ref, T_ref = q.qlora_linear_fwd(X, Wp, A, B, s)
    for _ in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        T = torch.full((M, r), float("nan"), dtype=torch.float32, device=DEV)
        assert call_noalloc(X, Wp, A, B, s, Y, T) == 0
        torch.cuda.synchronize()
        assert_close_rms(f64(Y), f64(Y_ref), "Y")
        assert_close_rms(f64(T), f64(T_ref), "T")
        if M > 128:  # the same GEMM launch as the regular forward
            assert torch.equal(Y, Y_ref) and torch.equal(T, T_ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    M, K, N, r = 65536, 4096, 256, 128  # needs far more than the fixed scratch
    X = torch.zeros(16, dtype=torch.bfloat16, device=DEV)  # never read: the call must fail first
    ptr = X.data_ptr()
    L = q.lib()
    st = L.qlora_linear_fwd_noalloc(ptr, M, K, N, ptr, ptr, ptr, ptr, ptr, r, ctypes.c_float(1.0), ptr, ptr,
                                    torch.cuda.current_stream().cuda_stream)
    assert st == 4  # QLORA_ERR_WORKSPACE

"""Failure handling on the GPU without a fault: a bounded pipeline wait is
made to run out on purpose, and the library must report it as
QLORA_ERR_TIMEOUT while the CUDA context stays usable.

The output tiles of the fused GEMMs wait for a per-512-row-block ready count
in the workspace that their rank units raise by 2.  Presetting that count to
a large negative value means it can never reach 2, so the tiles of that block
give up after the wait limit (set to 1 ms here).  The kernels then let their
own copies and MMAs end, free tensor memory and exit; the last CTA pair
returns the counters to zero.  Afterwards the workspace is zero-filled (as
include/qlora.h asks after a timeout) and the same call must pass parity.
"""

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import synthetic
from oracle import dequantize_nf4, lora_linear_backward, lora_linear_forward, quantize_nf4
from tests.helpers import assert_close_rms, f32, f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TIMEOUT = 6
STATUS_BYTES = 256  # the workspace starts with the 256-byte status word


def counters_offsets(M):
    """Byte offsets of the forward and input-gradient GEMM counters in the
    workspace: [status][fwd: ticket, done, ready per 512-row block][dX: same]."""
    ints = 2 + -(-M // 512)
    ctr_bytes = -(-ints * 4 // 256) * 256
    return STATUS_BYTES, STATUS_BYTES + ctr_bytes


@pytest.fixture
def short_waits():
    q.qlora_set_wait_timeout(1_000_000)  # 1 ms
    assert q.qlora_get_wait_timeout() == 1_000_000
    yield
    q.qlora_set_wait_timeout(0)
    assert q.qlora_get_wait_timeout() == 2_000_000_000


@pytest.mark.parametrize("which", ["fwd", "bwd"])
def test_ready_count_that_never_arrives_times_out(which, short_waits):
    case = synthetic.linear_case(1100, 512, 640, 64, 0.25, seed=41)
    Wp = q.qlora_quantize_nf4(case.W.to(DEV))
    X, A, B, dY = (t.to(DEV) for t in (case.X, case.A, case.B, case.dY))
    ws = q.new_workspace(case.M, case.K, case.N, case.r, DEV)
    Y, T = q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws)
    assert q.qlora_check_status(ws) == 0
    off_fwd, off_dx = counters_offsets(case.M)
    off = off_fwd if which == "fwd" else off_dx
    ready0 = ws[off + 8:off + 12].view(torch.int32)  # ready count of row block 0
    ready0.fill_(-(1 << 30))
    if which == "fwd":
        q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws, Y=Y, T_save=T)
    else:
        q.qlora_linear_bwd(dY, X, T, Wp, A, B, case.scale, workspace=ws)
    assert q.qlora_check_status(ws) == TIMEOUT
    # The word was cleared by the check, the context still works, and the
    # counters are back at zero.
    assert q.qlora_check_status(ws) == 0
    counters = ws[off:off + 20].view(torch.int32).cpu().numpy()
    assert np.all(counters == 0), counters

    # Recovery: zero-filled workspace, default limit, full parity.
    q.qlora_set_wait_timeout(0)
    ws.zero_()
    Y, T = q.qlora_linear_fwd(X, Wp, A, B, case.scale, workspace=ws)
    dX, dA, dB = q.qlora_linear_bwd(dY, X, T, Wp, A, B, case.scale, workspace=ws)
    assert q.qlora_check_status(ws) == 0
    codes, aq, sc = quantize_nf4(f32(case.W))
    Wdq = dequantize_nf4(codes, aq, sc, case.W.numel()).reshape(case.N, case.K)
    Yr, Tr = lora_linear_forward(f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    dXr, dAr, dBr = lora_linear_backward(f64(case.dY), f64(case.X), Wdq, f64(case.A), f64(case.B), case.scale)
    for name, got, ref in (("Y", Y, Yr), ("T", T, Tr), ("dX", dX, dXr), ("dA", dA, dAr), ("dB", dB, dBr)):
        assert_close_rms(f64(got), ref, name)


def test_wait_limit_is_validated():
    with pytest.raises(q.QloraError):
        q.qlora_set_wait_timeout(61 * 10**9)
    q.qlora_set_wait_timeout(0)
    assert q.qlora_get_wait_timeout() == 2_000_000_000


def test_codec_status_is_clear_after_normal_calls():
    W = synthetic.weight_only(512, 1024, seed=3).to(DEV)
    Wp = q.qlora_quantize_nf4(W)
    q.qlora_dequantize_nf4(Wp)
    assert q.qlora_check_status(None) == 0

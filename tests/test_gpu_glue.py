"""The SiLU-gate glue kernels of the gated MLP (not a method step) against a
float64 restatement of the same formulas: each output is one bf16 rounding of
a float32 computation, so it must lie within one bf16 ulp (plus float32
rounding noise) of the exact value.  Sizes cover the 8-wide vector path and a
ragged tail."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_quantize_b200 as q
from tests.helpers import f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (normal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check(got, ref, name):
    err = np.abs(got - ref)
    bound = bf16_ulp(ref) + 1e-6 * np.abs(ref) + 1e-30
    bad = err > bound
    assert not bad.any(), f"{name}: {bad.sum()} values off by more than one bf16 ulp, e.g. {got[bad][:3]} vs {ref[bad][:3]}"


@pytest.mark.parametrize("n", [8, 1000, 8 * 4099 + 5, 1 << 20])
def test_silu_gate_forward_and_backward(n):
    g = torch.Generator().manual_seed(n)
    G = (torch.randn(n, generator=g) * 3).to(torch.bfloat16)
    U = torch.randn(n, generator=g).to(torch.bfloat16)
    dH = torch.randn(n, generator=g).to(torch.bfloat16)
    Gd, Ud, dHd = G.to(DEV), U.to(DEV), dH.to(DEV)
    H = q.qlora_silu_gate_fwd(Gd, Ud)
    dG, dU = q.qlora_silu_gate_bwd(Gd, Ud, dHd)
    torch.cuda.synchronize()
    g64, u64, h64 = f64(G), f64(U), f64(dH)
    sg = 1.0 / (1.0 + np.exp(-g64))
    check(f64(H), g64 * sg * u64, "H")
    check(f64(dG), h64 * u64 * sg * (1 + g64 * (1 - sg)), "dG")
    check(f64(dU), h64 * g64 * sg, "dU")

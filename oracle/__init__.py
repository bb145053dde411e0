"""CPU oracle for the frozen-NF4 linear layer with a LoRA adapter.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this package: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg may.  It is a plain, slow, obviously-correct restatement of
what the method computes, in numpy float64 with every rounding step written
out, and it shares no code, table or constant generator with the CUDA library.

Sources (the pages describe the method in prose only):
  * "AI Glossary: QLoRA" (mangrove.ai), Definition and second paragraph:
    frozen weights stored as 4-bit numbers, dequantized to BFloat16 each time
    the layer is used, weight gradients only for the LoRA matrices, NF4 for
    normally distributed values, quantized quantization constants.
  * "QLoRA: Fine-Tuning 65-Billion Parameter Models on a Single Consumer GPU"
    (deepfa.ir), sections "LoRA: Prerequisite for Understanding QLoRA",
    "QLoRA's Technical Innovations" (1. 4-bit NormalFloat, 2. Double
    Quantization, 3. Paged Optimizers) and "QLoRA's Working Process".

Parity status per function (see each module's header):
  * nf4_codebook            pinned to the reading (invariants, two independent
                            normal-quantile routes, equal-probability spacing);
                            the numeric values themselves are not printed on
                            the pages.
  * fp4/int4_codebook       pinned to the reading (the printed rationals of
                            the 1-2-1 float and k/7, invariants) and to the
                            pages' claim that NF4 has the lower error on
                            normally distributed weights.
  * quantize / dequantize   pinned (brute force on tiny inputs in exact
                            rational arithmetic, closed forms, special cases).
  * forward / backward      pinned (finite differences, torch fp64 autograd,
                            special cases).
  * adamw_step / adamw_run  pinned (closed forms of the first step and of a
                            constant gradient, torch.optim.AdamW in float64).
"""

from .nf4_ref import (  # noqa: F401
    BLOCK,
    GROUP,
    nf4_codebook,
    fp4_codebook,
    int4_codebook,
    codebook,
    bf16_round,
    quantize_nf4,
    dequantize_nf4,
    dequantize_scales,
    dequantize_at,
)
from .linear_ref import lora_linear_forward, lora_linear_backward  # noqa: F401
from .adamw_ref import adamw_step, adamw_run  # noqa: F401

"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every function include/qlora.h declares, and rejects invalid calls on the
host before anything is launched (fake pointers are never dereferenced)."""

import ctypes
import os
import re

import numpy as np
import pytest

import bit_quantized_lora_quantize_b200 as q
from bit_quantized_lora_quantize_b200 import build as qbuild
from oracle import nf4_codebook

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    qbuild.build()
    return q.lib()


def declared_functions():
    with open(os.path.join(ROOT, "include", "qlora.h")) as f:
        src = f.read()
    return re.findall(r"QLORA_API\s+[\w\s\*]+?\b(qlora_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for must in ("qlora_quantize_nf4", "qlora_dequantize_nf4", "qlora_linear_fwd", "qlora_linear_bwd",
                 "qlora_workspace_bytes", "qlora_check_status", "qlora_nf4_codebook", "qlora_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_codebook_matches_oracle_in_float32(L):
    np.testing.assert_array_equal(np.array(q.qlora_nf4_codebook(), dtype=np.float32), nf4_codebook())


@pytest.mark.parametrize("code", ["nf4", "fp4", "int4"])
def test_every_codebook_matches_oracle_in_float32(L, code):
    from oracle import codebook
    np.testing.assert_array_equal(np.array(q.qlora_codebook(code), dtype=np.float32), codebook(code))


def test_unknown_code_is_rejected(L):
    buf = (ctypes.c_float * 16)()
    assert L.qlora_codebook(3, buf) == 1
    assert L.qlora_quantize_4bit(FAKE, 64, 7, FAKE, FAKE, FAKE, None) == 1
    assert L.qlora_dequantize_4bit(FAKE, FAKE, FAKE, 64, -1, FAKE, None) == 1


def test_adamw_validation(L):
    P = FAKE
    args = dict(n=10, step=1, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.0)

    def call(p=P, **kw):
        a = dict(args, **kw)
        return L.qlora_adamw_step(p, None, P, P, P, a["n"], a["step"], a["lr"], a["b1"], a["b2"], a["eps"], a["wd"],
                                  None)
    assert call(step=0) == 1            # steps count from 1
    assert call(n=0) == 1
    assert call(b1=1.0) == 1 and call(b2=-0.1) == 1
    assert call(lr=float("inf")) == 1
    assert call(p=P + 2) == 2           # float buffers must be 4-byte aligned
    assert L.qlora_paged_prefetch(None, 16, 1, None) == 1


def test_status_strings(L):
    for s in range(7):
        assert L.qlora_status_string(s)


FAKE = 1 << 20  # aligned, never dereferenced: every call below fails validation first


def fwd(L, **kw):
    a = dict(X=FAKE, M=16, K=256, N=256, codes=FAKE, aq=FAKE, sc=FAKE, A=FAKE, B=FAKE, r=8, s=2.0, Y=FAKE,
             T=FAKE, ws=FAKE, nws=1 << 30, st=None)
    a.update(kw)
    return L.qlora_linear_fwd(a["X"], a["M"], a["K"], a["N"], a["codes"], a["aq"], a["sc"], a["A"], a["B"], a["r"],
                              a["s"], a["Y"], a["T"], a["ws"], a["nws"], a["st"])


def test_linear_fwd_validation(L):
    assert fwd(L, X=None) == 1
    assert fwd(L, s=float("nan")) == 1
    assert fwd(L, M=0) == 1
    assert fwd(L, K=100) == 3          # K % 64 != 0
    assert fwd(L, N=260) == 3          # N % 8 != 0
    assert fwd(L, r=257) == 3          # r > 256
    assert fwd(L, r=0) == 1
    assert fwd(L, X=FAKE + 8) == 2     # misaligned
    assert fwd(L, ws=None) == 4
    assert fwd(L, nws=16) == 4


def test_linear_bwd_validation(L):
    P = FAKE
    base = [P, P, P, 16, 256, 256, P, P, P, P, P, 8, 2.0, P, P, P, P, 1 << 30, None]
    assert L.qlora_linear_bwd(*base[:13], None, *base[14:]) == 1
    bad = list(base)
    bad[4] = 96
    assert L.qlora_linear_bwd(*bad) == 3
    bad = list(base)
    bad[14] = P + 4
    assert L.qlora_linear_bwd(*bad) == 2
    bad = list(base)
    bad[17] = 64
    assert L.qlora_linear_bwd(*bad) == 4


def fwd_noalloc(L, **kw):
    a = dict(X=FAKE, M=16, K=256, N=256, codes=FAKE, aq=FAKE, sc=FAKE, A=FAKE, B=FAKE, r=8, s=2.0, Y=FAKE,
             T=FAKE, st=None)
    a.update(kw)
    return L.qlora_linear_fwd_noalloc(a["X"], a["M"], a["K"], a["N"], a["codes"], a["aq"], a["sc"], a["A"], a["B"],
                                      a["r"], a["s"], a["Y"], a["T"], a["st"])


def test_linear_fwd_noalloc_validation(L):
    """The allocation-free forward takes the same shape rules as the regular
    one, plus ranks that are multiples of 8 and shapes whose scratch fits its
    fixed device array (16 MiB)."""
    assert fwd_noalloc(L, T=None) == 1
    assert fwd_noalloc(L, s=float("nan")) == 1
    assert fwd_noalloc(L, s=float("inf")) == 1
    assert fwd_noalloc(L, s=float("-inf")) == 1
    assert fwd_noalloc(L, M=0) == 1
    assert fwd_noalloc(L, K=100) == 3
    assert fwd_noalloc(L, N=260) == 3
    assert fwd_noalloc(L, r=257) == 3
    assert fwd_noalloc(L, r=12) == 3   # not a multiple of 8: no room to pad here
    assert fwd_noalloc(L, Y=FAKE + 8) == 2
    assert fwd_noalloc(L, sc=FAKE + 2) == 2
    assert fwd_noalloc(L, M=65536, K=4096, r=128) == 4  # scratch beyond the fixed array


def test_four_bit_entry_points_validate_the_code(L):
    """The 4-bit calls take NF4, FP4 or Int4, optionally with the centred
    constants flag; any other code is rejected before the shape checks."""
    P = FAKE
    args = [P, 16, 256, 256, P, P, P, None, P, P, 8, 2.0, P, P, P, 1 << 30, None]
    for code in (3, -1, 0x200, 0x42, 3 | 0x100):  # no such code, stray bits, an unknown flag
        a = list(args)
        a[7] = code
        assert L.qlora_linear_fwd_4bit(*a) == 1, code
        b = [P, P, P, 16, 256, 256, P, P, P, code, P, P, 8, 2.0, P, P, P, P, 1 << 30, None]
        assert L.qlora_linear_bwd_4bit(*b) == 1, code
    for code in (q.qlora.CODES["nf4"], q.qlora.CODES["fp4"], q.qlora.CODES["int4"],
                 q.qlora.CODES["nf4"] | q.qlora.DQ["centred_fp8"], q.qlora.CODES["int4"] | q.qlora.DQ["centred_fp8"]):
        a = list(args)
        a[7] = code
        a[2] = 100  # valid code: the shape check now decides
        assert L.qlora_linear_fwd_4bit(*a) == 3, code
        b = [P, P, P, 16, 100, 256, P, P, P, code, P, P, 8, 2.0, P, P, P, P, 1 << 30, None]
        assert L.qlora_linear_bwd_4bit(*b) == 3, code


def test_paged_malloc_without_a_device_reports_why(L):
    """On a machine without a GPU the unified-memory allocation returns NULL
    and qlora_last_cuda_error names the CUDA error behind it."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the allocation would succeed")
    assert not L.qlora_paged_malloc(4096, -1, None)
    assert L.qlora_last_cuda_error()


def test_codec_validation(L):
    assert L.qlora_quantize_nf4(None, 64, FAKE, FAKE, FAKE, None) == 1
    assert L.qlora_quantize_nf4(FAKE, 0, FAKE, FAKE, FAKE, None) == 1
    assert L.qlora_quantize_nf4(FAKE + 2, 64, FAKE, FAKE, FAKE, None) == 2
    assert L.qlora_dequantize_nf4(FAKE, FAKE, FAKE, -5, FAKE, None) == 1
    assert L.qlora_dequantize_nf4(FAKE, FAKE, FAKE + 2, 64, FAKE, None) == 2


def test_any_rank_up_to_256_is_accepted(L):
    """Ranks that are not multiples of 8 run with the adapter padded inside
    the workspace, which is therefore larger; ranks above 128 take the pair
    GEMMs for every M; 257 and above are unsupported."""
    for r in (1, 4, 13, 64, 100, 136, 200, 256):
        assert q.qlora_workspace_bytes(16, 256, 256, r) > 0
        assert q.qlora_workspace_bytes(1000, 512, 384, r) > 0
    assert q.qlora_workspace_bytes(16, 256, 256, 257) == 0
    assert q.qlora_workspace_bytes(1000, 512, 384, 13) > q.qlora_workspace_bytes(1000, 512, 384, 16)


def test_workspace_bytes(L):
    assert q.qlora_workspace_bytes(16, 256, 256, 8) > 256
    assert q.qlora_workspace_bytes(16, 100, 256, 8) == 0
    a = q.qlora_workspace_bytes(4096, 4096, 4096, 64)
    b = q.qlora_workspace_bytes(8192, 4096, 4096, 64)
    assert b >= a > 4096 * 64 * 2


def test_product_path_has_no_cpu_fallback():
    import torch
    with pytest.raises(ValueError):
        q.qlora_quantize_nf4(torch.zeros(64, dtype=torch.bfloat16))

"""Thin Python binding of ``libqlora.so`` (C ABI declared in include/qlora.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  There is no
CPU fallback: if the library is missing or the device is not a CUDA device,
the calls raise.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlora.so")

QLORA_OK = 0
# 4-bit codes of the packed format (qlora_code in include/qlora.h) and the
# schemes of the 8-bit constants (QLORA_DQ_CENTRED_FP8 for "centred_fp8").
CODES = {"nf4": 0, "fp4": 1, "int4": 2}
DQ = {"linear8": 0, "centred_fp8": 0x100}
STATUS_NAMES = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_ALIGNMENT", 3: "QLORA_ERR_UNSUPPORTED",
                4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_CUDA", 6: "QLORA_ERR_TIMEOUT"}

# Exported symbols and their C signatures.
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "qlora_quantize_nf4": (ctypes.c_int, [_P, _I64, _P, _P, _P, _P]),
    "qlora_dequantize_nf4": (ctypes.c_int, [_P, _P, _P, _I64, _P, _P]),
    "qlora_quantize_4bit": (ctypes.c_int, [_P, _I64, ctypes.c_int32, _P, _P, _P, _P]),
    "qlora_dequantize_4bit": (ctypes.c_int, [_P, _P, _P, _I64, ctypes.c_int32, _P, _P]),
    "qlora_linear_fwd_4bit": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_int32, _P, _P,
                                             ctypes.c_int32, ctypes.c_float, _P, _P, _P, ctypes.c_size_t, _P]),
    "qlora_linear_bwd_4bit": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, ctypes.c_int32, _P, _P,
                                             ctypes.c_int32, ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t,
                                             _P]),
    "qlora_codebook": (ctypes.c_int, [ctypes.c_int32, ctypes.POINTER(ctypes.c_float)]),
    "qlora_linear_fwd": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_float,
                                        _P, _P, _P, ctypes.c_size_t, _P]),
    "qlora_linear_bwd": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, ctypes.c_int32,
                                        ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, ctypes.c_int32,
                                                ctypes.c_float, _P, _P, _P]),
    "qlora_silu_gate_fwd": (ctypes.c_int, [_P, _P, _P, _I64, _P]),
    "qlora_silu_gate_bwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _P]),
    "qlora_paged_malloc": (ctypes.c_void_p, [ctypes.c_size_t, ctypes.c_int, _P]),
    "qlora_paged_free": (None, [_P, ctypes.c_size_t, ctypes.c_int, _P]),
    "qlora_paged_prefetch": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.c_int32, _P]),
    "qlora_paged_location": (ctypes.c_int, [_P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32)]),
    "qlora_adamw_step": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, ctypes.c_int32, ctypes.c_float, ctypes.c_float,
                                        ctypes.c_float, ctypes.c_float, ctypes.c_float, _P]),
    "qlora_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, ctypes.c_int32]),
    "qlora_check_status": (ctypes.c_int, [_P, _P]),
    "qlora_set_wait_timeout": (ctypes.c_int, [ctypes.c_uint64]),
    "qlora_get_wait_timeout": (ctypes.c_uint64, []),
    "qlora_nf4_codebook": (None, [ctypes.POINTER(ctypes.c_float)]),
    "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_last_cuda_error": (ctypes.c_char_p, []),
    "qlora_profile_start": (None, []),
    "qlora_profile_stop": (ctypes.c_int, [ctypes.c_int, ctypes.c_char_p, ctypes.POINTER(ctypes.c_float),
                                          ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
}

_lib = None


class QloraError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{fn} -> {STATUS_NAMES.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """Load libqlora.so (built in-tree by ``build.py``); raise if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing (run bit_quantized_lora_quantize_b200/build.py)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def _check(fn: str, status: int) -> None:
    if status != QLORA_OK:
        detail = ""
        if status == 5:
            detail = lib().qlora_last_cuda_error().decode()
        raise QloraError(fn, status, detail)


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _require_cuda(*ts: torch.Tensor) -> None:
    for t in ts:
        if not t.is_cuda:
            raise ValueError("qlora kernels take CUDA tensors only (no CPU path)")
        if not t.is_contiguous():
            raise ValueError("qlora kernels take contiguous tensors")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


# ---------------------------------------------------------------- packed weight
@dataclass
class PackedNF4:
    """A frozen weight [N, K] in the packed format of include/qlora.h, with
    the NF4 levels (or the FP4 / Int4 ones, ``code``)."""

    codes: torch.Tensor         # uint8 [ceil(N*K/2)]
    absmax_q: torch.Tensor      # uint8 [NB]
    absmax_scale: torch.Tensor  # float32 [NB2]
    shape: tuple
    code: str = "nf4"
    dq: str = "linear8"

    @property
    def code_value(self) -> int:
        return CODES[self.code] | DQ[self.dq]

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= s
        return n


def packed_sizes(numel: int):
    nb = -(-numel // 64)
    return (numel + 1) // 2, nb, -(-nb // 256)


def qlora_nf4_codebook() -> list:
    buf = (ctypes.c_float * 16)()
    lib().qlora_nf4_codebook(buf)
    return list(buf)


def qlora_codebook(code: str = "nf4") -> list:
    buf = (ctypes.c_float * 16)()
    _check("qlora_codebook", lib().qlora_codebook(CODES[code], buf))
    return list(buf)


def qlora_quantize_nf4(W: torch.Tensor, out: PackedNF4 = None, code: str = "nf4", dq: str = "linear8") -> PackedNF4:
    """Quantize a bf16 CUDA tensor (any shape, flattened row-major) with the
    NF4 levels (or ``code`` = "fp4" / "int4") and the linear 8-bit constants
    (or ``dq`` = "centred_fp8").  `out`, if given, is a PackedNF4 of the same
    element count whose buffers are overwritten."""
    _require_cuda(W)
    if W.dtype != torch.bfloat16:
        raise ValueError("W must be bfloat16")
    n = W.numel()
    nc, nb, nb2 = packed_sizes(n)
    nsc = nb2 + (1 if dq == "centred_fp8" else 0)  # the centred scheme stores its mean last
    dev = W.device
    if out is None:
        codes = torch.empty(max(nc, 16), dtype=torch.uint8, device=dev)[:nc]
        aq = torch.empty(nb, dtype=torch.uint8, device=dev)
        sc = torch.empty(nsc, dtype=torch.float32, device=dev)
    else:
        codes, aq, sc = out.codes, out.absmax_q, out.absmax_scale
        if (codes.numel(), aq.numel(), sc.numel()) != (nc, nb, nsc):
            raise ValueError("out does not hold a weight of this size")
        _require_cuda(codes, aq, sc)
    if code == "nf4" and dq == "linear8":
        _check("qlora_quantize_nf4", lib().qlora_quantize_nf4(_ptr(W), n, _ptr(codes), _ptr(aq), _ptr(sc),
                                                              _stream()))
    else:
        _check("qlora_quantize_4bit", lib().qlora_quantize_4bit(_ptr(W), n, CODES[code] | DQ[dq], _ptr(codes),
                                                                _ptr(aq), _ptr(sc), _stream()))
    return PackedNF4(codes, aq, sc, tuple(W.shape), code, dq)


def qlora_dequantize_nf4(p: PackedNF4, out: torch.Tensor = None) -> torch.Tensor:
    _require_cuda(p.codes, p.absmax_q, p.absmax_scale)
    if out is None:
        out = torch.empty(p.shape, dtype=torch.bfloat16, device=p.codes.device)
    elif out.dtype != torch.bfloat16 or out.numel() != p.numel or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor of the weight's size")
    if p.code_value == 0:
        _check("qlora_dequantize_nf4", lib().qlora_dequantize_nf4(_ptr(p.codes), _ptr(p.absmax_q),
                                                                  _ptr(p.absmax_scale), p.numel, _ptr(out), _stream()))
    else:
        _check("qlora_dequantize_4bit", lib().qlora_dequantize_4bit(_ptr(p.codes), _ptr(p.absmax_q),
                                                                    _ptr(p.absmax_scale), p.numel, p.code_value,
                                                                    _ptr(out), _stream()))
    return out


def qlora_workspace_bytes(M: int, K: int, N: int, r: int) -> int:
    return int(lib().qlora_workspace_bytes(M, K, N, r))


def new_workspace(M: int, K: int, N: int, r: int, device) -> torch.Tensor:
    nbytes = qlora_workspace_bytes(M, K, N, r)
    if nbytes == 0:
        raise QloraError("qlora_workspace_bytes", 3, f"M={M} K={K} N={N} r={r}")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def qlora_linear_fwd(X: torch.Tensor, W: PackedNF4, A: torch.Tensor, B: torch.Tensor, scale: float,
                     workspace: torch.Tensor | None = None, Y: torch.Tensor | None = None,
                     T_save: torch.Tensor | None = None):
    """Return (Y, T_save) for Y = X W'^T + (s X A) B (see include/qlora.h)."""
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[1]
    _require_cuda(X, A, B, W.codes)
    dev = X.device
    if workspace is None:
        workspace = new_workspace(M, K, N, r, dev)
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    if T_save is None:
        T_save = torch.empty(M, r, dtype=torch.float32, device=dev)
    if W.code_value == 0:
        _check("qlora_linear_fwd", lib().qlora_linear_fwd(
            _ptr(X), M, K, N, _ptr(W.codes), _ptr(W.absmax_q), _ptr(W.absmax_scale), _ptr(A), _ptr(B), r,
            float(scale), _ptr(Y), _ptr(T_save), _ptr(workspace), workspace.numel(), _stream()))
    else:
        _check("qlora_linear_fwd_4bit", lib().qlora_linear_fwd_4bit(
            _ptr(X), M, K, N, _ptr(W.codes), _ptr(W.absmax_q), _ptr(W.absmax_scale), W.code_value, _ptr(A),
            _ptr(B), r, float(scale), _ptr(Y), _ptr(T_save), _ptr(workspace), workspace.numel(), _stream()))
    return Y, T_save


def qlora_linear_fwd_noalloc(X: torch.Tensor, W: PackedNF4, A: torch.Tensor, B: torch.Tensor, scale: float,
                             Y: torch.Tensor, T_save: torch.Tensor):
    """Forward into caller-provided Y and T_save with no workspace: the
    library takes its scratch from a fixed device array (see include/qlora.h)."""
    if W.code_value != 0:
        raise ValueError("the allocation-free forward takes NF4 weights with linear 8-bit constants only")
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[1]
    _require_cuda(X, A, B, W.codes, Y, T_save)
    _check("qlora_linear_fwd_noalloc", lib().qlora_linear_fwd_noalloc(
        _ptr(X), M, K, N, _ptr(W.codes), _ptr(W.absmax_q), _ptr(W.absmax_scale), _ptr(A), _ptr(B), r,
        float(scale), _ptr(Y), _ptr(T_save), _stream()))
    return Y, T_save


def qlora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, T_save: torch.Tensor, W: PackedNF4, A: torch.Tensor,
                     B: torch.Tensor, scale: float, workspace: torch.Tensor | None = None,
                     dX: torch.Tensor | None = None, dA: torch.Tensor | None = None, dB: torch.Tensor | None = None):
    """Return (dX, dA, dB) (see include/qlora.h)."""
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[1]
    _require_cuda(dY, X, T_save, A, B, W.codes)
    dev = X.device
    if workspace is None:
        workspace = new_workspace(M, K, N, r, dev)
    if dX is None:
        dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty(K, r, dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty(r, N, dtype=torch.float32, device=dev)
    if W.code_value == 0:
        _check("qlora_linear_bwd", lib().qlora_linear_bwd(
            _ptr(dY), _ptr(X), _ptr(T_save), M, K, N, _ptr(W.codes), _ptr(W.absmax_q), _ptr(W.absmax_scale),
            _ptr(A), _ptr(B), r, float(scale), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace), workspace.numel(),
            _stream()))
    else:
        _check("qlora_linear_bwd_4bit", lib().qlora_linear_bwd_4bit(
            _ptr(dY), _ptr(X), _ptr(T_save), M, K, N, _ptr(W.codes), _ptr(W.absmax_q), _ptr(W.absmax_scale),
            W.code_value, _ptr(A), _ptr(B), r, float(scale), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(workspace),
            workspace.numel(), _stream()))
    return dX, dA, dB


def _same_bf16(*ts: torch.Tensor) -> None:
    _require_cuda(*ts)
    for t in ts:
        if t.dtype != torch.bfloat16 or t.numel() != ts[0].numel():
            raise ValueError("bf16 tensors of one size expected")


def qlora_silu_gate_fwd(G: torch.Tensor, U: torch.Tensor, H: torch.Tensor | None = None) -> torch.Tensor:
    """H = silu(G) * U (glue between the linears of a gated MLP)."""
    if H is None:
        H = torch.empty_like(G)
    _same_bf16(G, U, H)
    _check("qlora_silu_gate_fwd", lib().qlora_silu_gate_fwd(_ptr(G), _ptr(U), _ptr(H), G.numel(), _stream()))
    return H


def qlora_silu_gate_bwd(G: torch.Tensor, U: torch.Tensor, dH: torch.Tensor, dG: torch.Tensor | None = None,
                        dU: torch.Tensor | None = None):
    """(dG, dU) of H = silu(G) * U for the upstream gradient dH."""
    dG = torch.empty_like(G) if dG is None else dG
    dU = torch.empty_like(U) if dU is None else dU
    _same_bf16(G, U, dH, dG, dU)
    _check("qlora_silu_gate_bwd", lib().qlora_silu_gate_bwd(_ptr(G), _ptr(U), _ptr(dH), _ptr(dG), _ptr(dU),
                                                            G.numel(), _stream()))
    return dG, dU


def qlora_check_status(workspace: torch.Tensor | None = None) -> int:
    """Synchronise and return the device status code (0 = OK, 6 = a pipeline
    wait timed out): the workspace's word (if given) and the library's own
    words for the calls without a workspace."""
    return int(lib().qlora_check_status(_ptr(workspace) if workspace is not None else None, _stream()))


def qlora_set_wait_timeout(timeout_ns: int) -> None:
    """Limit of every bounded wait in the kernels (0 = the default, 2 s)."""
    _check("qlora_set_wait_timeout", lib().qlora_set_wait_timeout(int(timeout_ns)))


def qlora_get_wait_timeout() -> int:
    return int(lib().qlora_get_wait_timeout())


def qlora_profile_start() -> None:
    lib().qlora_profile_start()


def qlora_profile_stop(max_entries: int = 32) -> dict:
    """Per-kernel {name: (total_ms, records, launches)} since qlora_profile_start."""
    names = ctypes.create_string_buffer(48 * max_entries)
    ms = (ctypes.c_float * max_entries)()
    calls = (ctypes.c_int * max_entries)()
    launches = (ctypes.c_int * max_entries)()
    n = lib().qlora_profile_stop(max_entries, names, ms, calls, launches)
    out = {}
    for i in range(n):
        name = names.raw[48 * i:48 * (i + 1)].split(b"\0", 1)[0].decode()
        out[name] = (float(ms[i]), int(calls[i]), int(launches[i]))
    return out


__all__ = ["CODES", "qlora_codebook", "qlora_profile_start", "qlora_profile_stop", "LIB_PATH", "lib", "QloraError", "PackedNF4", "packed_sizes", "qlora_nf4_codebook", "qlora_quantize_nf4",
           "qlora_dequantize_nf4", "qlora_workspace_bytes", "new_workspace", "qlora_linear_fwd", "qlora_linear_bwd",
           "qlora_linear_fwd_noalloc",
           "qlora_check_status", "qlora_set_wait_timeout", "qlora_get_wait_timeout", "qlora_silu_gate_fwd",
           "qlora_silu_gate_bwd"]

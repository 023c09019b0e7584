"""QLoRA linear layer on NVIDIA B200: Python binding of libqlora.

Thin marshalling over the C ABI declared in include/qlora.h: each function
here has the name of the C entry point it calls, takes torch tensors, and
passes their device pointers and the current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; torch only allocates device
memory (outputs and workspaces) and provides the stream.  There is no CPU
fallback: without the built library or a CUDA device the calls raise.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _ffi
from ._ffi import (COMPUTE_BF16, COMPUTE_FP32, FMT_AFFINE, FMT_NF4_DQ, FMT_NF4_FP32SCALE, OP_BWD,
                   OP_FWD, qlora_weight)

__all__ = [
    "QLoraError", "QuantizedWeight", "qlora_status_string", "qlora_nf4_codebook",
    "qlora_nf4_payload_bytes", "qlora_quantize_nf4", "qlora_quantize_nf4_noalloc", "qlora_quantize_affine",
    "qlora_nf4_fp32scale_payload_bytes", "qlora_quantize_nf4_fp32scale",
    "qlora_dequantize", "qlora_merge", "qlora_adam_step",
    "qlora_linear_workspace_bytes", "qlora_linear_fwd", "qlora_linear_bwd",
    "qlora_workspace_status", "qlora_selftest_wait_timeout", "qlora_kernel_launch_count",
    "qlora_kernel_timing_enable", "qlora_kernel_timing_collect",
    "COMPUTE_FP32", "COMPUTE_BF16", "FMT_NF4_DQ", "FMT_NF4_FP32SCALE", "FMT_AFFINE", "workspace",
]


class QLoraError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        msg = _ffi.load().qlora_status_string(self.status).decode()
        super().__init__(f"{where}: {msg} (status {self.status})" if where else msg)


def _check(status: int, where: str):
    if status != _ffi.OK:
        raise QLoraError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(where: str, name: str, t: Optional[torch.Tensor], dev, shape=None, dtype=None):
    """Reject (before any launch) a tensor the kernels would misread: not on
    the weight's CUDA device, not dense, or of the wrong shape or dtype."""
    if t is None:
        return
    if not t.is_cuda or t.device != dev:
        raise ValueError(f"{where}: {name} must be a CUDA tensor on {dev}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{where}: {name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{where}: {name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{where}: {name} must be contiguous")


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device workspace of at least nbytes (torch allocates)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


@dataclass
class QuantizedWeight:
    """Device buffers of a frozen quantized weight (immutable by convention)."""
    fmt: int
    O: int
    I: int
    block: int
    group: int
    bits: int
    codes: torch.Tensor
    scale_codes: Optional[torch.Tensor] = None
    group_absmax: Optional[torch.Tensor] = None
    mean: Optional[torch.Tensor] = None
    scale: Optional[torch.Tensor] = None
    bias: Optional[torch.Tensor] = None

    def c_struct(self) -> qlora_weight:
        return qlora_weight(self.fmt, self.O, self.I, self.block, self.group, self.bits,
                            *(t.data_ptr() if t is not None and t.numel() > 0 else None
                              for t in (self.codes, self.scale_codes, self.group_absmax, self.mean,
                                        self.scale, self.bias)))

    _BUFFERS = ("codes", "scale_codes", "group_absmax", "mean", "scale", "bias")

    def expected_sizes(self) -> dict:
        """Element count and dtype of every buffer the format defines."""
        N = self.O * self.I
        if self.fmt == FMT_NF4_DQ:
            M = -(-N // self.block)
            S = -(-M // self.group)
            return {"codes": ((N + 1) // 2, torch.uint8), "scale_codes": (M, torch.uint8),
                    "group_absmax": (S, torch.float32), "mean": (1, torch.float32)}
        if self.fmt == FMT_NF4_FP32SCALE:
            return {"codes": ((N + 1) // 2, torch.uint8), "scale": (-(-N // self.block), torch.float32)}
        ng = -(-N // self.block)
        return {"codes": (N if self.bits == 8 else (N + 1) // 2, torch.uint8),
                "scale": (ng, torch.float32), "bias": (ng, torch.float32)}

    def state_dict(self) -> dict:
        """Host copy of the format fields and the packed buffers, byte for
        byte (the canonical serialization for checkpoints)."""
        d = {"fmt": self.fmt, "O": self.O, "I": self.I, "block": self.block, "group": self.group,
             "bits": self.bits}
        for k in self._BUFFERS:
            t = getattr(self, k)
            if t is not None:
                d[k] = t.detach().cpu().contiguous().numpy().copy()
        return d

    @classmethod
    def from_state_dict(cls, d: dict, device="cuda") -> "QuantizedWeight":
        """Inverse of state_dict(); every buffer is checked against the size
        and dtype its format fields imply before it reaches the device."""
        import numpy as np
        w = cls(int(d["fmt"]), int(d["O"]), int(d["I"]), int(d["block"]), int(d["group"]), int(d["bits"]),
                codes=torch.empty(0, dtype=torch.uint8))
        if w.fmt not in (FMT_NF4_DQ, FMT_NF4_FP32SCALE, FMT_AFFINE) or w.O < 0 or w.I < 0 or w.block < 1 \
                or (w.fmt == FMT_NF4_DQ and (w.group < 1 or w.bits != 4)) \
                or (w.fmt == FMT_NF4_FP32SCALE and w.bits != 4) or (w.fmt == FMT_AFFINE and w.bits not in (4, 8)):
            raise ValueError("inconsistent format fields")
        for k, (n, dt) in w.expected_sizes().items():
            if k not in d or d[k] is None:
                raise ValueError(f"missing buffer {k}")
            a = np.ascontiguousarray(d[k])
            t = torch.from_numpy(a)
            if t.dtype != dt or t.numel() != n:
                raise ValueError(f"buffer {k}: expected {n} x {dt}, got {t.numel()} x {t.dtype}")
            setattr(w, k, t.reshape(-1).to(device))
        return w

    def payload_bytes(self) -> int:
        ts = [self.codes, self.scale_codes, self.group_absmax, self.mean, self.scale, self.bias]
        return sum(t.numel() * t.element_size() for t in ts if t is not None)


def qlora_status_string(status: int) -> str:
    return _ffi.load().qlora_status_string(int(status)).decode()


def qlora_nf4_codebook():
    out = (ctypes.c_float * 16)()
    _check(_ffi.load().qlora_nf4_codebook(out), "qlora_nf4_codebook")
    return [float(v) for v in out]


def qlora_nf4_payload_bytes(N: int, B: int = 64, C: int = 256) -> int:
    return int(_ffi.load().qlora_nf4_payload_bytes(N, B, C))


def qlora_quantize_nf4(W: torch.Tensor, B: int = 64, C: int = 256, stream=None) -> QuantizedWeight:
    """NF4 + double-quantized scales of a CUDA fp32 [O x I] matrix (synchronizes the stream)."""
    lib = _ffi.load()
    if W.dim() != 2 or W.dtype != torch.float32 or not W.is_cuda:
        raise ValueError("W must be a CUDA float32 matrix")
    W = W.contiguous()
    O, I = W.shape
    N = O * I
    M = -(-N // B)
    S = -(-M // C)
    dev = W.device
    codes = torch.empty((N + 1) // 2, dtype=torch.uint8, device=dev)
    q = torch.empty(M, dtype=torch.uint8, device=dev)
    t = torch.empty(S, dtype=torch.float32, device=dev)
    mu = torch.empty(1, dtype=torch.float32, device=dev)
    ws = workspace(lib.qlora_quantize_nf4_workspace_bytes(N, B, C), dev)
    st = lib.qlora_quantize_nf4(_ptr(W), O, I, B, C, _ptr(codes), _ptr(q), _ptr(t), _ptr(mu), _ptr(ws),
                                ws.numel(), _stream(stream))
    _check(st, "qlora_quantize_nf4")
    return QuantizedWeight(FMT_NF4_DQ, O, I, B, C, 4, codes, q, t, mu)


def qlora_quantize_nf4_noalloc(W: torch.Tensor, B: int = 64, C: int = 256, stream=None) -> QuantizedWeight:
    """As qlora_quantize_nf4, for callers that cannot supply a workspace: the
    library's fixed device scratch is used (see include/qlora.h).  The output
    buffers are still the caller's; calls sharing the scratch must not overlap."""
    lib = _ffi.load()
    if W.dim() != 2 or W.dtype != torch.float32 or not W.is_cuda:
        raise ValueError("W must be a CUDA float32 matrix")
    W = W.contiguous()
    O, I = W.shape
    N = O * I
    M = -(-N // B)
    S = -(-M // C)
    dev = W.device
    codes = torch.empty((N + 1) // 2, dtype=torch.uint8, device=dev)
    q = torch.empty(M, dtype=torch.uint8, device=dev)
    t = torch.empty(S, dtype=torch.float32, device=dev)
    mu = torch.empty(1, dtype=torch.float32, device=dev)
    st = lib.qlora_quantize_nf4_noalloc(_ptr(W), O, I, B, C, _ptr(codes), _ptr(q), _ptr(t), _ptr(mu),
                                        _stream(stream))
    _check(st, "qlora_quantize_nf4_noalloc")
    return QuantizedWeight(FMT_NF4_DQ, O, I, B, C, 4, codes, q, t, mu)


def qlora_nf4_fp32scale_payload_bytes(N: int, B: int = 64) -> int:
    return int(_ffi.load().qlora_nf4_fp32scale_payload_bytes(N, B))


def qlora_quantize_nf4_fp32scale(W: torch.Tensor, B: int = 64, stream=None) -> QuantizedWeight:
    """NF4 codes with the legacy scale storage (one fp32 absmax per block) of
    a CUDA fp32 [O x I] matrix (synchronizes the stream)."""
    lib = _ffi.load()
    if W.dim() != 2 or W.dtype != torch.float32 or not W.is_cuda:
        raise ValueError("W must be a CUDA float32 matrix")
    W = W.contiguous()
    O, I = W.shape
    N = O * I
    M = -(-N // B)
    dev = W.device
    codes = torch.empty((N + 1) // 2, dtype=torch.uint8, device=dev)
    scale = torch.empty(M, dtype=torch.float32, device=dev)
    ws = workspace(lib.qlora_quantize_nf4_fp32scale_workspace_bytes(N, B), dev)
    st = lib.qlora_quantize_nf4_fp32scale(_ptr(W), O, I, B, _ptr(codes), _ptr(scale), _ptr(ws), ws.numel(),
                                          _stream(stream))
    _check(st, "qlora_quantize_nf4_fp32scale")
    return QuantizedWeight(FMT_NF4_FP32SCALE, O, I, B, 0, 4, codes, scale=scale)


def qlora_quantize_affine(W: torch.Tensor, bits: int = 4, G: int = 64, stream=None) -> QuantizedWeight:
    """Affine group-wise 4/8-bit codes with fp32 scale and bias (synchronizes the stream)."""
    lib = _ffi.load()
    if W.dim() != 2 or W.dtype != torch.float32 or not W.is_cuda:
        raise ValueError("W must be a CUDA float32 matrix")
    W = W.contiguous()
    O, I = W.shape
    N = O * I
    ng = -(-N // G)
    dev = W.device
    codes = torch.empty(N if bits == 8 else (N + 1) // 2, dtype=torch.uint8, device=dev)
    scale = torch.empty(ng, dtype=torch.float32, device=dev)
    bias = torch.empty(ng, dtype=torch.float32, device=dev)
    ws = workspace(lib.qlora_quantize_affine_workspace_bytes(N, bits, G), dev)
    st = lib.qlora_quantize_affine(_ptr(W), O, I, bits, G, _ptr(codes), _ptr(scale), _ptr(bias), _ptr(ws),
                                   ws.numel(), _stream(stream))
    _check(st, "qlora_quantize_affine")
    return QuantizedWeight(FMT_AFFINE, O, I, G, 0, bits, codes, scale=scale, bias=bias)


def qlora_dequantize(w: QuantizedWeight, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Diagnostic fp32 reconstruction of the whole weight (never used by fwd/bwd)."""
    lib = _ffi.load()
    if out is None:
        out = torch.empty((w.O, w.I), dtype=torch.float32, device=w.codes.device)
    _need("qlora_dequantize", "out", out, w.codes.device, (w.O, w.I), torch.float32)
    cw = w.c_struct()
    _check(lib.qlora_dequantize(ctypes.byref(cw), _ptr(out), _stream(stream)), "qlora_dequantize")
    return out


def qlora_merge(w: QuantizedWeight, A: torch.Tensor, B: torch.Tensor, alpha: float,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Export: W_hat + (alpha/r) B A as an fp32 [O x I] matrix (A [r x I], B [O x r] fp32)."""
    lib = _ffi.load()
    r = A.shape[0]
    if A.dtype != torch.float32 or B.dtype != torch.float32 or tuple(A.shape) != (r, w.I) \
            or tuple(B.shape) != (w.O, r) or not A.is_contiguous() or not B.is_contiguous():
        raise ValueError("A must be contiguous fp32 [r x I] and B contiguous fp32 [O x r]")
    if out is None:
        out = torch.empty((w.O, w.I), dtype=torch.float32, device=w.codes.device)
    dev = w.codes.device
    _need("qlora_merge", "A", A, dev)
    _need("qlora_merge", "B", B, dev)
    _need("qlora_merge", "out", out, dev, (w.O, w.I), torch.float32)
    cw = w.c_struct()
    _check(lib.qlora_merge(ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha), _ptr(out), _stream(stream)),
           "qlora_merge")
    return out


def qlora_adam_step(params: torch.Tensor, grads: torch.Tensor, m: torch.Tensor, v: torch.Tensor, t: int,
                    lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                    page_elems: int = 0, stream=None) -> None:
    """One in-place Adam step over flat contiguous fp32 tensors (step count t >= 1)."""
    n = params.numel()
    for x in (params, grads, m, v):
        if x.dtype != torch.float32 or not x.is_contiguous() or x.numel() != n:
            raise ValueError("params, grads, m and v must be contiguous fp32 tensors of one size")
        _need("qlora_adam_step", "params/grads/m/v", x, params.device)
    st = _ffi.load().qlora_adam_step(_ptr(params), _ptr(grads), _ptr(m), _ptr(v), n, int(t), float(lr),
                                     float(beta1), float(beta2), float(eps), int(page_elems), _stream(stream))
    _check(st, "qlora_adam_step")


def qlora_linear_workspace_bytes(w: QuantizedWeight, R: int, r: int, op: int, compute: int) -> int:
    cw = w.c_struct()
    return int(_ffi.load().qlora_linear_workspace_bytes(ctypes.byref(cw), R, r, op, compute))


def _compute_of(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return COMPUTE_BF16
    if t.dtype == torch.float32:
        return COMPUTE_FP32
    raise ValueError("activations must be bfloat16 or float32")


def qlora_linear_fwd(w: QuantizedWeight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     Y: Optional[torch.Tensor] = None, U_out: Optional[torch.Tensor] = None,
                     ws: Optional[torch.Tensor] = None, stream=None,
                     want_u: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Y = X W_hat^T + (alpha/r)(X A^T) B^T; returns (Y, U = X A^T)."""
    lib = _ffi.load()
    R = X.shape[0]
    r = A.shape[0]
    compute = _compute_of(X)
    if Y is None:
        Y = torch.empty((R, w.O), dtype=X.dtype, device=X.device)
    if U_out is None and want_u:
        U_out = torch.empty((R, r), dtype=torch.float32, device=X.device)
    if ws is None:
        ws = workspace(qlora_linear_workspace_bytes(w, R, r, OP_FWD, compute), X.device)
    dev, f = w.codes.device, "qlora_linear_fwd"
    _need(f, "X", X, dev, (R, w.I))
    _need(f, "A", A, dev, (r, w.I), torch.float32)
    _need(f, "B", B, dev, (w.O, r), torch.float32)
    _need(f, "Y", Y, dev, (R, w.O), X.dtype)
    _need(f, "U_out", U_out, dev, (R, r), torch.float32)
    _need(f, "ws", ws, dev)
    cw = w.c_struct()
    st = lib.qlora_linear_fwd(ctypes.byref(cw), _ptr(X), R, _ptr(A), _ptr(B), r, float(alpha), compute,
                              _ptr(Y), _ptr(U_out), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "qlora_linear_fwd")
    return Y, U_out


def qlora_linear_bwd(w: QuantizedWeight, X: Optional[torch.Tensor], dY: torch.Tensor, A: torch.Tensor,
                     B: torch.Tensor, alpha: float, U: Optional[torch.Tensor] = None,
                     want_dx: bool = True, want_da: bool = True, want_db: bool = True,
                     dX: Optional[torch.Tensor] = None, dA: Optional[torch.Tensor] = None,
                     dB: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """(dX, dA, dB) of the QLoRA linear layer (no weight gradient)."""
    lib = _ffi.load()
    R = dY.shape[0]
    r = A.shape[0]
    compute = _compute_of(dY)
    dev = dY.device
    if want_dx and dX is None:
        dX = torch.empty((R, w.I), dtype=dY.dtype, device=dev)
    if want_da and dA is None:
        dA = torch.empty((r, w.I), dtype=torch.float32, device=dev)
    if want_db and dB is None:
        dB = torch.empty((w.O, r), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(qlora_linear_workspace_bytes(w, R, r, OP_BWD, compute), dev)
    wd, f = w.codes.device, "qlora_linear_bwd"
    _need(f, "dY", dY, wd, (R, w.O))
    _need(f, "X", X, wd, (R, w.I), dY.dtype)
    _need(f, "A", A, wd, (r, w.I), torch.float32)
    _need(f, "B", B, wd, (w.O, r), torch.float32)
    _need(f, "U", U, wd, (R, r), torch.float32)
    _need(f, "dX", dX if want_dx else None, wd, (R, w.I), dY.dtype)
    _need(f, "dA", dA if want_da else None, wd, (r, w.I), torch.float32)
    _need(f, "dB", dB if want_db else None, wd, (w.O, r), torch.float32)
    _need(f, "ws", ws, wd)
    cw = w.c_struct()
    st = lib.qlora_linear_bwd(ctypes.byref(cw), _ptr(X), _ptr(dY), R, _ptr(A), _ptr(B), r, float(alpha),
                              _ptr(U), compute, _ptr(dX if want_dx else None), _ptr(dA if want_da else None),
                              _ptr(dB if want_db else None), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "qlora_linear_bwd")
    return (dX if want_dx else None), (dA if want_da else None), (dB if want_db else None)


def qlora_workspace_status(ws: torch.Tensor, stream=None) -> int:
    """Device error word of the last call that used ws (synchronizes)."""
    return int(_ffi.load().qlora_workspace_status(_ptr(ws), _stream(stream)))


def qlora_selftest_wait_timeout(limit_us: int = 1000, stream=None, device="cuda") -> int:
    ws = workspace(256, device)
    return int(_ffi.load().qlora_selftest_wait_timeout(_ptr(ws), ws.numel(), int(limit_us), _stream(stream)))


def qlora_kernel_launch_count() -> int:
    return int(_ffi.load().qlora_kernel_launch_count())


def qlora_kernel_timing_enable(max_records: int) -> None:
    _check(_ffi.load().qlora_kernel_timing_enable(int(max_records)), "qlora_kernel_timing_enable")


def qlora_kernel_timing_collect(max_records: int = 4096):
    """[(kind, ms, flops)] of the tensor-core GEMM launches recorded since enable."""
    ms = (ctypes.c_float * max_records)()
    kind = (ctypes.c_int32 * max_records)()
    fl = (ctypes.c_double * max_records)()
    n = _ffi.load().qlora_kernel_timing_collect(ms, kind, fl, max_records)
    if n < 0:
        raise QLoraError(_ffi.ERR_CUDA, "qlora_kernel_timing_collect")
    return [(int(kind[i]), float(ms[i]), float(fl[i])) for i in range(n)]

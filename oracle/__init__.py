"""CPU oracle for the QLoRA linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (``qlora_bit_frozen_b200``)
never imports it and shares no code with it.

numpy front end over ``qlora_oracle.c`` (plain C, fp64 accumulation,
per-element nibble decode).  See the header of that file for the passages
each function follows and the readings taken where the pages are silent.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against values the pages print, closed forms, special cases, library
routines (scipy's normal quantile, numpy matmul on the dequantized matrix)
and finite differences; the NF4 levels equal the published canonical table
bit for bit.  Bit-level agreement with MLX's affine rounding is parity
unpinned (MLX is not available).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

FMT_NF4_DQ = 0
FMT_NF4_FP32SCALE = 1
FMT_AFFINE = 2

OK = 0
ERR_NONFINITE = 1
ERR_ARG = 2

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_double
        lib.oracle_norm_ppf.argtypes = [f64]
        lib.oracle_norm_ppf.restype = f64
        lib.oracle_nf4_codebook.argtypes = [P, P]
        lib.oracle_nf4_codebook.restype = None
        lib.oracle_quantize_levels.argtypes = [P, i64, i64, P, ctypes.c_int, P, P, P]
        lib.oracle_quantize_levels.restype = ctypes.c_int
        lib.oracle_quantize_nf4.argtypes = [P, i64, i32, i32, P, P, P, P, P]
        lib.oracle_quantize_nf4.restype = ctypes.c_int
        lib.oracle_decode_scale.argtypes = [ctypes.c_uint8, f32, f32]
        lib.oracle_decode_scale.restype = f32
        lib.oracle_quantize_affine.argtypes = [P, i64, i32, i32, P, P, P]
        lib.oracle_quantize_affine.restype = ctypes.c_int
        lib.oracle_dequantize.argtypes = [P, P]
        lib.oracle_dequantize.restype = None
        lib.oracle_linear_fwd.argtypes = [P, P, i64, P, i64, P, P, i32, f32, P, P]
        lib.oracle_linear_fwd.restype = None
        lib.oracle_linear_bwd.argtypes = [P, P, P, i64, P, i64, P, P, i32, f32, P, P, P]
        lib.oracle_linear_bwd.restype = None
        lib.oracle_merge.argtypes = [P, P, P, i32, f32, P]
        lib.oracle_merge.restype = None
        lib.oracle_adam_step.argtypes = [P, P, P, P, i64, i64, f32, f32, f32, f32, P, P, P]
        lib.oracle_adam_step.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def norm_ppf(p: float) -> float:
    return float(_load().oracle_norm_ppf(float(p)))


def nf4_codebook():
    """(fp64 levels, fp32 levels) of the NF4 data type, ascending."""
    c64 = np.zeros(16, np.float64)
    c32 = np.zeros(16, np.float32)
    _load().oracle_nf4_codebook(_ptr(c64), _ptr(c32))
    return c64, c32


def quantize_levels(w, block: int, levels):
    """Absmax block quantizer with an arbitrary sorted codebook."""
    w = _c(w, np.float32).ravel()
    lv = _c(levels, np.float64)
    n = w.size
    codes = np.zeros(n, np.uint8)
    scales = np.zeros(max(1, -(-n // block)), np.float32)
    w_hat = np.zeros(n, np.float64)
    st = _load().oracle_quantize_levels(_ptr(w), n, block, _ptr(lv), lv.size, _ptr(codes), _ptr(scales), _ptr(w_hat))
    if st != OK:
        raise ValueError(f"oracle_quantize_levels status {st}")
    return codes, scales, w_hat


@dataclass
class QWeight:
    """Quantized weight in the oracle's own view (numpy buffers)."""
    fmt: int
    O: int
    I: int
    block: int
    group: int
    bits: int
    codes: np.ndarray
    qcodes: Optional[np.ndarray] = None
    t: Optional[np.ndarray] = None
    mu: float = 0.0
    scale: Optional[np.ndarray] = None
    bias: Optional[np.ndarray] = None


class _CWeight(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("O", ctypes.c_int64), ("I", ctypes.c_int64),
        ("block", ctypes.c_int32), ("group", ctypes.c_int32), ("bits", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("qcodes", ctypes.c_void_p), ("t", ctypes.c_void_p),
        ("mu", ctypes.c_float), ("scale", ctypes.c_void_p), ("bias", ctypes.c_void_p),
    ]


def _cweight(w: QWeight) -> _CWeight:
    def p(a):
        return a.ctypes.data if a is not None and a.size > 0 else None
    return _CWeight(w.fmt, w.O, w.I, w.block, w.group, w.bits, p(w.codes), p(w.qcodes), p(w.t),
                    float(w.mu), p(w.scale), p(w.bias))


def nf4_sizes(N: int, B: int, C: int):
    M = -(-N // B)
    S = -(-M // C)
    return M, S


def quantize_nf4(W, B: int = 64, C: int = 256, return_s: bool = False):
    """NF4 + double-quantized scales of a row-major [O x I] matrix."""
    W = _c(W, np.float32)
    O, I = (W.shape if W.ndim == 2 else (1, W.size))
    N = W.size
    M, S = nf4_sizes(N, B, C)
    codes = np.zeros((N + 1) // 2, np.uint8)
    qcodes = np.zeros(M, np.uint8)
    t = np.zeros(S, np.float32)
    mu = np.zeros(1, np.float32)
    s = np.zeros(max(M, 1), np.float32)
    st = _load().oracle_quantize_nf4(_ptr(W), N, B, C, _ptr(codes), _ptr(qcodes), _ptr(t), _ptr(mu), _ptr(s))
    if st == ERR_NONFINITE:
        raise FloatingPointError("non-finite weight")
    if st != OK:
        raise ValueError(f"oracle_quantize_nf4 status {st}")
    w = QWeight(FMT_NF4_DQ, O, I, B, C, 4, codes, qcodes, t, float(mu[0]))
    return (w, s[:M]) if return_s else w


def quantize_nf4_legacy(W, B: int = 64) -> QWeight:
    """NF4 codes with the legacy scales: one fp32 block absmax s_b per block
    (the same codes as the double-quantized format, which encodes with the
    exact s_b too)."""
    W = _c(W, np.float32)
    w, s = quantize_nf4(W, B, 256, return_s=True)
    return QWeight(FMT_NF4_FP32SCALE, w.O, w.I, B, 0, 4, w.codes, scale=np.ascontiguousarray(s))


def decode_scale(q: int, t: float, mu: float) -> np.float32:
    return np.float32(_load().oracle_decode_scale(int(q), float(np.float32(t)), float(np.float32(mu))))


def quantize_affine(W, bits: int = 4, G: int = 64):
    W = _c(W, np.float32)
    O, I = (W.shape if W.ndim == 2 else (1, W.size))
    N = W.size
    ng = -(-N // G)
    codes = np.zeros(N if bits == 8 else (N + 1) // 2, np.uint8)
    scale = np.zeros(ng, np.float32)
    bias = np.zeros(ng, np.float32)
    st = _load().oracle_quantize_affine(_ptr(W), N, bits, G, _ptr(codes), _ptr(scale), _ptr(bias))
    if st == ERR_NONFINITE:
        raise FloatingPointError("non-finite weight or range")
    if st != OK:
        raise ValueError(f"oracle_quantize_affine status {st}")
    return QWeight(FMT_AFFINE, O, I, G, 0, bits, codes, scale=scale, bias=bias)


def dequantize(w: QWeight) -> np.ndarray:
    out = np.zeros((w.O, w.I), np.float32)
    cw = _cweight(w)
    _load().oracle_dequantize(ctypes.byref(cw), _ptr(out))
    return out


def _rows_arg(rows, R):
    if rows is None:
        return None, R
    rows = _c(rows, np.int64)
    assert rows.size == 0 or (rows.min() >= 0 and rows.max() < R)
    return rows, rows.size


def linear_fwd(w: QWeight, X, A, Bm, r: int, alpha: float, rows=None):
    """(Y [n x O], U [n x r]) in fp64 for the selected rows of X."""
    X = _c(X, np.float32)
    A = _c(A, np.float32)
    Bm = _c(Bm, np.float32)
    R = X.shape[0]
    rows, n = _rows_arg(rows, R)
    Y = np.zeros((n, w.O), np.float64)
    U = np.zeros((n, r), np.float64)
    cw = _cweight(w)
    _load().oracle_linear_fwd(ctypes.byref(cw), _ptr(X), R, _ptr(rows), n, _ptr(A), _ptr(Bm), r,
                              float(alpha), _ptr(Y), _ptr(U))
    return Y, U


def linear_bwd(w: QWeight, X, dY, A, Bm, r: int, alpha: float, rows=None,
               want_dx=True, want_da=True, want_db=True):
    """(dX [n x I] | None, dA [r x I] | None, dB [O x r] | None) in fp64."""
    X = _c(X, np.float32)
    dY = _c(dY, np.float32)
    A = _c(A, np.float32)
    Bm = _c(Bm, np.float32)
    R = X.shape[0]
    rows, n = _rows_arg(rows, R)
    dX = np.zeros((n, w.I), np.float64) if want_dx else None
    dA = np.zeros((r, w.I), np.float64) if want_da else None
    dB = np.zeros((w.O, r), np.float64) if want_db else None
    cw = _cweight(w)
    _load().oracle_linear_bwd(ctypes.byref(cw), _ptr(X), _ptr(dY), R, _ptr(rows), n, _ptr(A), _ptr(Bm),
                              r, float(alpha), _ptr(dX), _ptr(dA), _ptr(dB))
    return dX, dA, dB


def merge(w: QWeight, A, Bm, r: int, alpha: float) -> np.ndarray:
    """W_hat + (alpha/r) Bm A as an fp64 [O x I] matrix (export)."""
    A = _c(A, np.float32)
    Bm = _c(Bm, np.float32)
    out = np.zeros((w.O, w.I), np.float64)
    cw = _cweight(w)
    _load().oracle_merge(ctypes.byref(cw), _ptr(A), _ptr(Bm), r, float(alpha), _ptr(out))
    return out


def adam_step(p, g, m, v, t: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
              eps: float = 1e-8):
    """One Adam step with bias correction: (p', m', v') in fp64 from fp32 state."""
    p = _c(p, np.float32).ravel()
    g = _c(g, np.float32).ravel()
    m = _c(m, np.float32).ravel()
    v = _c(v, np.float32).ravel()
    n = p.size
    assert g.size == n and m.size == n and v.size == n and t >= 1
    po = np.zeros(n, np.float64)
    mo = np.zeros(n, np.float64)
    vo = np.zeros(n, np.float64)
    _load().oracle_adam_step(_ptr(p), _ptr(g), _ptr(m), _ptr(v), n, int(t), float(lr), float(beta1),
                             float(beta2), float(eps), _ptr(po), _ptr(mo), _ptr(vo))
    return po, mo, vo


def nf4_payload_bytes(N: int, B: int, C: int) -> int:
    """ceil(N/2) + M + 4S + 4: codes, scale codes, t_g, mu."""
    M, S = nf4_sizes(N, B, C)
    return (N + 1) // 2 + M + 4 * S + 4


def legacy_payload_bytes(N: int, B: int) -> int:
    """ceil(N/2) + 4 ceil(N/B): codes and one fp32 scale per block."""
    return (N + 1) // 2 + 4 * (-(-N // B))

"""Seeded synthetic inputs for the QLoRA linear workloads.

This module only draws numbers and describes shapes; it holds none of the
method's arithmetic (no quantization, no GEMM).  Tests, the benchmark and
the smoke check use it so that the CUDA path and the CPU oracle see the same
inputs.

Generator: splitmix64 as a counter-based stream (state_i = key + i * gamma,
output = the splitmix64 finalizer of state_i), 53-bit uniforms in (0, 1),
Box-Muller for normals.  Each tensor has its own seed
(seed = 1000 * workload_id + tensor_id).

bf16 inputs: values are drawn in fp32 and rounded to bf16 (round to nearest
even) on the host; the device receives the bf16 bits and the oracle the same
values widened back to fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int) -> np.uint64:
    with np.errstate(over="ignore"):
        return _mix(np.array([np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + _GAMMA], np.uint64))[0]


def uniform(seed: int, n: int, start: int = 0) -> np.ndarray:
    """n uniforms in (0, 1), float64, elements start .. start+n-1 of stream `seed`."""
    out = np.empty(n, np.float64)
    key = _key(seed)
    with np.errstate(over="ignore"):
        for c0 in range(0, n, _CHUNK):
            c1 = min(n, c0 + _CHUNK)
            idx = np.arange(start + c0 + 1, start + c1 + 1, dtype=np.uint64)
            z = _mix(key + idx * _GAMMA)
            out[c0:c1] = ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)
    return out


def normal(seed: int, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """float32 array of N(mean, std^2) draws (Box-Muller on stream `seed`)."""
    shape = tuple(int(s) for s in (shape if isinstance(shape, (tuple, list)) else (shape,)))
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, np.float32)
    npairs = (n + 1) // 2
    step = _CHUNK // 2
    for p0 in range(0, npairs, step):
        p1 = min(npairs, p0 + step)
        u = uniform(seed, 2 * (p1 - p0), start=2 * p0)
        u1, u2 = u[0::2], u[1::2]
        rad = np.sqrt(-2.0 * np.log(u1))
        z = np.empty(2 * (p1 - p0), np.float64)
        z[0::2] = rad * np.cos(2.0 * np.pi * u2)
        z[1::2] = rad * np.sin(2.0 * np.pi * u2)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = (z[: hi - lo] * std + mean).astype(np.float32)
    return out.reshape(shape)


def bf16_round(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Round fp32 values to bf16 (nearest even).  Returns (fp32 widened, uint16 bits)."""
    x = np.ascontiguousarray(x, np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))
    r = ((b + bias) >> np.uint64(16)).astype(np.uint16)
    wide = (r.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return wide.reshape(x.shape), r.reshape(x.shape)


# --------------------------------------------------------------------------
# Workloads (shapes and value distributions of the pages' models)
# --------------------------------------------------------------------------

@dataclass
class Linear:
    name: str
    O: int
    I: int


@dataclass
class Workload:
    wid: int
    name: str
    R: int
    linears: List[Linear]
    r: int
    alpha: float
    compute: str            # "fp32" or "bf16"
    w_std: float = 0.02
    ab_std: float = 0.02
    block: int = 64
    group: int = 256
    zero_block: Optional[int] = None      # flat block index forced to all-zero
    outlier_frac: float = 0.0             # fraction of weights scaled by outlier_mult
    outlier_mult: float = 20.0
    notes: str = ""
    extra: dict = field(default_factory=dict)

    def seed(self, lin_idx: int, tensor: str) -> int:
        tid = {"W": 1, "A": 2, "B": 3, "X": 4, "dY": 5, "outlier": 6}[tensor]
        return 1000 * self.wid + 10 * lin_idx + tid


def workload(name: str, R: Optional[int] = None) -> Workload:
    """The named workload; R overrides the token count (sweep / small cases)."""
    if name == "fp32_single_256":
        w = Workload(1, name, 64, [Linear("proj", 256, 256)], 8, 16.0, "fp32", zero_block=5,
                     notes="single QLoRA linear, fp32 compute")
    elif name == "qwen3_0.6b_attn_qv":
        w = Workload(2, name, 4096, [Linear("q_proj", 2048, 1024), Linear("v_proj", 1024, 1024)],
                     8, 16.0, "bf16", notes="Qwen3-0.6B-shaped q/v adapters, 4096 tokens")
    elif name == "8b_mlp":
        w = Workload(3, name, 8192, [Linear("gate_proj", 12288, 4096), Linear("up_proj", 12288, 4096),
                                     Linear("down_proj", 4096, 12288)],
                     32, 64.0, "bf16", notes="8B-class SwiGLU MLP linears, 8192 tokens")
    elif name == "14b_layer":
        w = Workload(4, name, 16384, [Linear("q_proj", 5120, 5120), Linear("k_proj", 1024, 5120),
                                      Linear("v_proj", 1024, 5120), Linear("o_proj", 5120, 5120),
                                      Linear("gate_proj", 17408, 5120), Linear("up_proj", 17408, 5120),
                                      Linear("down_proj", 5120, 17408)],
                     16, 32.0, "bf16", outlier_frac=0.001,
                     notes="14B-class decoder layer linears, 16384 tokens, 0.1% outliers x20")
    elif name == "bw_sweep_4096":
        w = Workload(5, name, 16, [Linear("w4096", 4096, 4096)], 8, 16.0, "bf16",
                     notes="small-R bandwidth sweep, W 4096x4096")
    elif name == "bw_sweep_12288":
        w = Workload(6, name, 16, [Linear("w12288", 12288, 4096)], 8, 16.0, "bf16",
                     notes="small-R bandwidth sweep, W 12288x4096")
    else:
        raise KeyError(name)
    if R is not None:
        w.R = int(R)
    return w


WORKLOADS = ["fp32_single_256", "qwen3_0.6b_attn_qv", "8b_mlp", "14b_layer", "bw_sweep_4096",
             "bw_sweep_12288"]


def weight(w: Workload, li: int) -> np.ndarray:
    """Frozen base weight [O x I] fp32 ~ N(0, w_std^2), with the workload's
    forced zero block and outliers."""
    lin = w.linears[li]
    W = normal(w.seed(li, "W"), (lin.O, lin.I), std=w.w_std)
    if w.outlier_frac > 0:
        u = uniform(w.seed(li, "outlier"), W.size).reshape(W.shape)
        W = np.where(u < w.outlier_frac, W * np.float32(w.outlier_mult), W).astype(np.float32)
    if w.zero_block is not None:
        flat = W.reshape(-1)
        b = w.zero_block
        flat[b * w.block:(b + 1) * w.block] = 0.0
    return W


def adapters(w: Workload, li: int):
    """LoRA factors A [r x I], B [O x r] (fp32, ~ N(0, ab_std^2))."""
    lin = w.linears[li]
    A = normal(w.seed(li, "A"), (w.r, lin.I), std=w.ab_std)
    B = normal(w.seed(li, "B"), (lin.O, w.r), std=w.ab_std)
    return A, B


def activations(w: Workload, li: int, R: Optional[int] = None):
    """X [R x I] and dY [R x O] ~ N(0, 1).  bf16 workloads return
    (x_fp32_widened, x_bf16_bits, dy_fp32_widened, dy_bf16_bits); fp32
    workloads return (x, None, dy, None)."""
    lin = w.linears[li]
    R = w.R if R is None else R
    X = normal(w.seed(li, "X"), (R, lin.I))
    dY = normal(w.seed(li, "dY"), (R, lin.O))
    if w.compute == "bf16":
        xw, xb = bf16_round(X)
        dw, db = bf16_round(dY)
        return xw, xb, dw, db
    return X, None, dY, None


def sample_rows(R: int, n: int, seed: int = 7) -> np.ndarray:
    """n distinct sorted row indices of R (always includes the first and last rows)."""
    if n >= R:
        return np.arange(R, dtype=np.int64)
    u = uniform(seed, R)
    order = np.argsort(u, kind="stable")
    rows = set(order[: max(0, n - 2)].tolist()) | {0, R - 1}
    return np.array(sorted(rows), dtype=np.int64)

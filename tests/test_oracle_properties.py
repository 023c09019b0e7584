"""Property checks of the oracle's quantizers on random shapes, block and
group sizes (hypothesis, CPU).  Each property follows from the definitions
on the pages alone: codes are the nearest level of w / s_b, the packed
layout puts weight 2j in the low nibble of byte j, the double-quantized
scale codes stay in 1..255 and decode to within half a code step, and the
affine codes stay on the grid within half a step of each weight."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle

_, C32 = oracle.nf4_codebook()
HALF_GAP = float(np.max(np.diff(C32.astype(np.float64)))) / 2


def _weights(seed, n, spread):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal(n) * np.float64(10.0) ** rng.uniform(-spread, spread, size=n)
    w[rng.random(n) < 0.05] = 0.0
    return w.astype(np.float32)


@settings(max_examples=60, deadline=None)
@given(seed=st.integers(0, 2 ** 31), n=st.integers(1, 700), B=st.sampled_from([1, 2, 7, 16, 64]),
       C=st.integers(1, 9), spread=st.floats(0, 3))
def test_nf4_properties(seed, n, B, C, spread):
    W = _weights(seed, n, spread).reshape(1, -1)
    w, s = oracle.quantize_nf4(W, B, C, return_s=True)
    M, S = oracle.nf4_sizes(n, B, C)
    assert w.codes.size == (n + 1) // 2 and w.qcodes.size == M and w.t.size == S
    codes = np.empty(2 * w.codes.size, np.uint8)
    codes[0::2] = w.codes & 15
    codes[1::2] = w.codes >> 4
    if n % 2:
        assert codes[-1] == 0
    codes = codes[:n]
    x = W.ravel().astype(np.float64)
    for b in range(M):
        blk = slice(b * B, min(n, (b + 1) * B))
        assert s[b] == np.max(np.abs(W.ravel()[blk]))
        if s[b] == 0:
            assert np.all(codes[blk] == 7)
            continue
        err = np.abs(C32[codes[blk]].astype(np.float64) * s[b] - x[blk])
        assert np.all(err <= HALF_GAP * s[b] * (1 + 1e-6))
    assert np.all((w.qcodes >= 1) & (w.qcodes <= 255))
    for g in range(S):
        blk = np.arange(g * C, min(M, (g + 1) * C))
        if w.t[g] == 0:
            assert np.all(w.qcodes[blk] == 128)
        sh = np.array([oracle.decode_scale(w.qcodes[b], w.t[g], w.mu) for b in blk], np.float64)
        assert np.all(np.abs(sh - np.maximum(s[blk], 0)) <= w.t[g] / 254.0 * (1 + 1e-5) + 4e-7 * np.abs(s[blk]) + 1e-30)


@settings(max_examples=60, deadline=None)
@given(seed=st.integers(0, 2 ** 31), n=st.integers(1, 700), bits=st.sampled_from([4, 8]),
       G=st.sampled_from([1, 3, 32, 64]), spread=st.floats(0, 2))
def test_affine_properties(seed, n, bits, G, spread):
    W = _weights(seed, n, spread).reshape(1, -1)
    w = oracle.quantize_affine(W, bits, G)
    Wh = oracle.dequantize(w).ravel().astype(np.float64)
    x = W.ravel().astype(np.float64)
    top = (1 << bits) - 1
    if bits == 8:
        q = w.codes[:n].astype(np.int64)
    else:
        q = np.empty(2 * w.codes.size, np.int64)
        q[0::2] = w.codes & 15
        q[1::2] = w.codes >> 4
        q = q[:n]
    assert np.all((q >= 0) & (q <= top))
    for g in range(-(-n // G)):
        blk = slice(g * G, min(n, (g + 1) * G))
        lo, hi = float(np.min(x[blk])), float(np.max(x[blk]))
        assert w.bias[g] == np.float32(lo)
        sc = float(w.scale[g])
        assert sc >= 0 and abs(sc * top - (hi - lo)) <= 1e-6 * max(abs(hi - lo), 1e-30)
        # each weight within half a grid step (plus fp32 rounding of the decode)
        tol = 0.5 * sc * (1 + 1e-5) + 4e-7 * (np.abs(x[blk]) + abs(lo) + sc * top)
        assert np.all(np.abs(Wh[blk] - x[blk]) <= tol)

"""CPU-side checks of the C-ABI library: it loads, exports every declared
entry point, and its host logic (argument checks, sizes, codebook) behaves.
No call here launches a kernel."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from qlora_bit_frozen_b200 import _ffi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlora.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _ffi.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_ffi.SIGNATURES), "binding and header disagree"


def test_codebook_matches_oracle_bitwise(lib):
    out = (ctypes.c_float * 16)()
    assert lib.qlora_nf4_codebook(out) == 0
    got = np.array(list(out), np.float32)
    _, ref = oracle.nf4_codebook()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("N,B,C", [(0, 64, 256), (1, 64, 256), (101, 64, 256), (65536, 64, 256),
                                   (89128960, 64, 256), (231, 16, 3)])
def test_payload_bytes_match_oracle(lib, N, B, C):
    assert lib.qlora_nf4_payload_bytes(N, B, C) == oracle.nf4_payload_bytes(N, B, C)


@pytest.mark.parametrize("N,B", [(0, 64), (1, 64), (101, 64), (65536, 64), (89128960, 64), (231, 16)])
def test_legacy_payload_bytes_match_oracle(lib, N, B):
    assert lib.qlora_nf4_fp32scale_payload_bytes(N, B) == oracle.legacy_payload_bytes(N, B)


def test_legacy_quantizer_arguments_rejected_before_launch(lib):
    ws = ctypes.create_string_buffer(1024)
    wsp = ctypes.c_void_p((ctypes.addressof(ws) + 255) // 256 * 256)
    d = ctypes.c_void_p(256)
    f = lib.qlora_quantize_nf4_fp32scale
    assert f(None, -1, 4, 64, None, None, wsp, 512, None) == _ffi.ERR_SHAPE
    assert f(None, 4, 4, 0, None, None, wsp, 512, None) == _ffi.ERR_SHAPE
    assert f(None, 4, 64, 64, None, None, wsp, 512, None) == _ffi.ERR_INVALID_ARG
    assert f(d, 4, 64, 64, d, d, ctypes.c_void_p(wsp.value + 8), 512, None) == _ffi.ERR_ALIGNMENT
    assert f(d, 4, 64, 64, d, d, wsp, 16, None) == _ffi.ERR_WORKSPACE
    assert f(d, 1 << 31, 1 << 31, 64, d, d, wsp, 512, None) == _ffi.ERR_SHAPE
    assert lib.qlora_quantize_nf4_fp32scale_workspace_bytes(1000, 64) >= 256


def test_overflowing_shapes_rejected_before_any_size_arithmetic(lib):
    """O * I beyond 2^40 weights is refused with a shape error before the
    library computes any size from it (2^31 x 2^31 would wrap a signed
    product, and a wrapped scratch size could pass the no-alloc size check).
    Pointers are never dereferenced: the check comes first."""
    d = ctypes.c_void_p(256)
    big = 1 << 31
    assert lib.qlora_quantize_nf4_noalloc(d, big, big, 1, 1, d, d, d, d, None) == _ffi.ERR_SHAPE
    assert lib.qlora_quantize_nf4(d, big, big, 1, 1, d, d, d, d, d, 1 << 20, None) == _ffi.ERR_SHAPE
    assert lib.qlora_quantize_affine(d, big, big, 4, 64, d, d, d, d, 1 << 20, None) == _ffi.ERR_SHAPE
    assert lib.qlora_quantize_nf4_workspace_bytes((1 << 40) + 1, 64, 256) == 0
    assert lib.qlora_quantize_nf4_noalloc(d, (1 << 40) + 1, 1, 64, 256, d, d, d, d, None) == _ffi.ERR_SHAPE


def test_bad_arguments_rejected_before_launch(lib):
    ws = ctypes.create_string_buffer(1024)
    wsp = ctypes.c_void_p((ctypes.addressof(ws) + 255) // 256 * 256)
    # negative shape, zero block, null outputs, misaligned workspace
    assert lib.qlora_quantize_nf4(None, -1, 4, 64, 256, None, None, None, None, wsp, 512, None) == _ffi.ERR_SHAPE
    assert lib.qlora_quantize_nf4(None, 4, 4, 0, 256, None, None, None, None, wsp, 512, None) == _ffi.ERR_SHAPE
    assert lib.qlora_quantize_nf4(None, 4, 64, 64, 256, None, None, None, None, wsp, 512, None) == _ffi.ERR_INVALID_ARG
    mis = ctypes.c_void_p(wsp.value + 8)
    dummy = ctypes.c_void_p(wsp.value)
    assert lib.qlora_quantize_nf4(dummy, 4, 64, 64, 256, dummy, dummy, dummy, dummy, mis, 512, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_quantize_nf4(dummy, 4, 64, 64, 256, dummy, dummy, dummy, dummy, wsp, 16, None) == _ffi.ERR_WORKSPACE
    assert lib.qlora_quantize_affine(dummy, 4, 64, 3, 64, dummy, dummy, dummy, wsp, 512, None) == _ffi.ERR_SHAPE

    w = _ffi.qlora_weight(_ffi.FMT_NF4_DQ, 64, 128, 64, 256, 4, wsp.value, wsp.value, wsp.value, wsp.value, None, None)
    P = ctypes.byref(w)
    # r out of range, bad compute enum, null adapters, I not a multiple of the block
    assert lib.qlora_linear_fwd(P, dummy, 4, dummy, dummy, 65, 1.0, 1, dummy, None, wsp, 1 << 20, None) == _ffi.ERR_UNSUPPORTED
    assert lib.qlora_linear_fwd(P, dummy, 4, dummy, dummy, 0, 1.0, 1, dummy, None, wsp, 1 << 20, None) == _ffi.ERR_SHAPE
    assert lib.qlora_linear_fwd(P, dummy, 4, dummy, dummy, 8, 1.0, 7, dummy, None, wsp, 1 << 20, None) == _ffi.ERR_INVALID_ARG
    assert lib.qlora_linear_fwd(P, dummy, 4, None, dummy, 8, 1.0, 1, dummy, None, wsp, 1 << 20, None) == _ffi.ERR_INVALID_ARG
    assert lib.qlora_linear_fwd(P, dummy, 4, dummy, dummy, 8, 1.0, 1, dummy, None, wsp, 16, None) == _ffi.ERR_WORKSPACE
    w.I = 100
    assert lib.qlora_linear_fwd(P, dummy, 4, dummy, dummy, 8, 1.0, 1, dummy, None, wsp, 1 << 20, None) == _ffi.ERR_SHAPE
    w.I = 128
    w.fmt = 9
    assert lib.qlora_dequantize(P, dummy, None) == _ffi.ERR_INVALID_ARG
    w.fmt = _ffi.FMT_AFFINE
    w.bits = 3
    assert lib.qlora_dequantize(P, dummy, None) == _ffi.ERR_SHAPE
    assert lib.qlora_dequantize(None, dummy, None) == _ffi.ERR_INVALID_ARG


def test_merge_and_adam_arguments_rejected_before_launch(lib):
    ws = ctypes.create_string_buffer(1024)
    d = ctypes.c_void_p((ctypes.addressof(ws) + 255) // 256 * 256)
    w = _ffi.qlora_weight(_ffi.FMT_NF4_DQ, 64, 128, 64, 256, 4, d.value, d.value, d.value, d.value, None, None)
    P = ctypes.byref(w)
    assert lib.qlora_merge(P, d, d, 0, 1.0, d, None) == _ffi.ERR_SHAPE
    assert lib.qlora_merge(P, None, d, 8, 1.0, d, None) == _ffi.ERR_INVALID_ARG
    assert lib.qlora_merge(P, d, d, 8, 1.0, None, None) == _ffi.ERR_INVALID_ARG
    assert lib.qlora_merge(None, d, d, 8, 1.0, d, None) == _ffi.ERR_INVALID_ARG
    w.bits = 8
    assert lib.qlora_merge(P, d, d, 8, 1.0, d, None) == _ffi.ERR_SHAPE
    adam = lib.qlora_adam_step
    assert adam(d, d, d, d, -1, 1, 1e-3, 0.9, 0.999, 1e-8, 0, None) == _ffi.ERR_SHAPE
    assert adam(d, d, d, d, 16, 0, 1e-3, 0.9, 0.999, 1e-8, 0, None) == _ffi.ERR_SHAPE
    assert adam(d, d, d, d, 16, 1, 1e-3, 0.9, 0.999, 1e-8, -4, None) == _ffi.ERR_SHAPE
    assert adam(d, d, d, d, 16, 1, 1e-3, 1.0, 0.999, 1e-8, 0, None) == _ffi.ERR_INVALID_ARG
    assert adam(d, d, d, d, 16, 1, 1e-3, 0.9, -0.5, 1e-8, 0, None) == _ffi.ERR_INVALID_ARG
    assert adam(d, d, d, d, 16, 1, 1e-3, 0.9, 0.999, 0.0, 0, None) == _ffi.ERR_INVALID_ARG
    assert adam(d, d, d, d, 16, 1, float("nan"), 0.9, 0.999, 1e-8, 0, None) == _ffi.ERR_INVALID_ARG
    assert adam(d, None, d, d, 16, 1, 1e-3, 0.9, 0.999, 1e-8, 0, None) == _ffi.ERR_INVALID_ARG
    # an empty arena is a valid no-op, even with null pointers
    assert adam(None, None, None, None, 0, 1, 1e-3, 0.9, 0.999, 1e-8, 0, None) == _ffi.OK


def test_misaligned_element_pointers_rejected_before_launch(lib):
    ws = ctypes.create_string_buffer(4096)
    d = ctypes.c_void_p((ctypes.addressof(ws) + 255) // 256 * 256)
    odd = ctypes.c_void_p(d.value + 2)     # 2-byte aligned: fine for bf16, not for fp32
    byte = ctypes.c_void_p(d.value + 1)
    assert lib.qlora_quantize_nf4(odd, 4, 64, 64, 256, d, d, d, d, d, 2048, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_quantize_nf4_noalloc(d, 4, 64, 64, 256, d, d, odd, d, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_quantize_affine(d, 4, 64, 4, 64, d, odd, d, d, 2048, None) == _ffi.ERR_ALIGNMENT
    w = _ffi.qlora_weight(_ffi.FMT_NF4_DQ, 64, 128, 64, 256, 4, d.value, d.value, odd.value, d.value, None, None)
    P = ctypes.byref(w)
    assert lib.qlora_dequantize(P, d, None) == _ffi.ERR_ALIGNMENT
    w.group_absmax = d.value
    assert lib.qlora_dequantize(P, odd, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_merge(P, d, odd, 8, 1.0, d, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_adam_step(d, d, odd, d, 16, 1, 1e-3, 0.9, 0.999, 1e-8, 0, None) == _ffi.ERR_ALIGNMENT
    big = 1 << 20
    # bf16 activations may sit on a 2-byte boundary, fp32 ones may not
    assert lib.qlora_linear_fwd(P, byte, 4, d, d, 8, 1.0, 1, d, None, d, big, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_linear_fwd(P, odd, 4, d, d, 8, 1.0, 0, d, None, d, big, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_linear_fwd(P, d, 4, odd, d, 8, 1.0, 1, d, None, d, big, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_linear_bwd(P, d, byte, 4, d, d, 8, 1.0, None, 1, d, d, d, d, big, None) == _ffi.ERR_ALIGNMENT
    assert lib.qlora_linear_bwd(P, d, d, 4, d, d, 8, 1.0, None, 1, d, odd, d, d, big, None) == _ffi.ERR_ALIGNMENT


def test_workspace_sizes_are_consistent(lib):
    w = _ffi.qlora_weight(_ffi.FMT_NF4_DQ, 2048, 1024, 64, 256, 4, None, None, None, None, None, None)
    P = ctypes.byref(w)
    for R in (0, 1, 16, 130, 4096):
        for op in (0, 1):
            for comp in (0, 1):
                n = lib.qlora_linear_workspace_bytes(P, R, 8, op, comp)
                assert n >= 256 and n % 256 == 0
    assert lib.qlora_linear_workspace_bytes(P, 16, 65, 0, 1) == 0
    assert lib.qlora_linear_workspace_bytes(P, 16, 8, 2, 1) == 0


def _a256(x):
    return -(-x // 256) * 256


def _planned_splits(Mw, KB, R, sms=148):
    """The tensor-core tile plan as the design states it: token tile = the
    smallest power of two >= R in 16..256, halved (not below 64) while the
    grid fills under 3/4 of a wave; below one wave of tiles, split K so the
    grid is one wave (two CTAs per SM below 256-token tiles), keeping at
    least 4 K steps per split and no empty split."""
    mt = Mw // 128
    bn = 16
    while bn < 256 and bn < R:
        bn *= 2
    while bn > 64 and 4 * mt * (-(-R // bn)) < 3 * sms:
        bn //= 2
    tiles = mt * (-(-R // bn))
    splits = 1
    if 0 < tiles < sms:
        splits = max(1, min((1 if bn >= 256 else 2) * sms // tiles, max(1, KB // 4)))
    per = -(-KB // splits)
    return bn, -(-KB // per)


def _smallr_splits(dx, O, I, R, sms=148):
    """The few-token plan as the design states it (1..16 tokens, O % 128 == 0,
    I % 64 == 0): 128-row tiles (forward) or 64-column blocks (input
    gradient) times K splits filling at most one wave at two CTAs per SM, at least
    one 64-column block per K warp (4) or one 16-row step per warp (8), no
    empty split.  0 when the path does not apply."""
    if not (1 <= R <= 16 and O % 128 == 0 and I % 64 == 0 and O <= 65536 and I <= 32768):
        return 0
    target = 2 * sms  # NF4: two CTAs per SM
    if not dx:
        tiles, n, per_min = O // 128, I // 64, 4
    else:
        tiles, n, per_min = I // 64, O // 16, 8
    sp = max(1, target // tiles)
    sp = min(sp, max(1, n // per_min))
    per = -(-n // sp)
    return -(-n // per)


@pytest.mark.parametrize("O,I,R", [(12288, 4096, 1), (12288, 4096, 16), (4096, 4096, 1), (4096, 4096, 16),
                                   (4096, 4096, 128), (2048, 1024, 4096), (1024, 1024, 4096),
                                   (12288, 4096, 8192), (5120, 17408, 16384), (128, 128, 3),
                                   (2048, 2048, 2047), (2048, 2048, 2048)])
def test_tensor_core_plan_through_workspace_sizes(lib, O, I, R):
    """The bf16 workspace exceeds the fp32 one by exactly the tensor-core
    region: the padded U/V copy (R x 64 bf16), the adapter weight operand
    (rows x 64 bf16), when K is split one fp32 partial per split, for the
    input gradient from 2048 tokens on 256-token tiles the bf16 copy of the
    decoded weight; at
    1..16 tokens also the few-token path's split partials.  This checks the
    host planners (split count, no empty split) without a GPU; the planners
    see 148 SMs here (no device)."""
    w = _ffi.qlora_weight(_ffi.FMT_NF4_DQ, O, I, 64, 256, 4, None, None, None, None, None, None)
    P = ctypes.byref(w)
    for op, Mw, KB in ((0, O, I // 64), (1, I, O // 64)):
        extra = lib.qlora_linear_workspace_bytes(P, R, 8, op, 1) - lib.qlora_linear_workspace_bytes(P, R, 8, op, 0)
        bn, splits = _planned_splits(Mw, KB, R)
        part = _a256(splits * R * Mw * 4) if splits > 1 else 0
        # input gradient from 2048 tokens on 256-token tiles without a K
        # split: the bf16 copy of the decoded weight
        wbuf = _a256(O * I * 2) if (op == 1 and bn == 256 and splits == 1 and R >= 2048) else 0
        srs = _smallr_splits(op == 1, O, I, R)
        sr = _a256(srs * R * (I if op == 1 else O) * 4) if srs > 1 else 0
        assert extra == _a256(R * 128) + _a256(Mw * 128) + part + wbuf + sr, (op, splits, srs)
        per = -(-KB // splits)
        assert 1 <= splits <= max(1, KB) and (splits - 1) * per < KB <= splits * per


def test_status_strings(lib):
    for s in range(9):
        assert lib.qlora_status_string(s)


def test_no_device_means_error_not_fallback(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    ws = ctypes.create_string_buffer(4096)
    wsp = ctypes.c_void_p((ctypes.addressof(ws) + 255) // 256 * 256)
    d = ctypes.c_void_p(wsp.value)
    st = lib.qlora_quantize_nf4(d, 1, 64, 64, 256, d, d, d, d, wsp, 2048, None)
    assert st == _ffi.ERR_CUDA


def test_binding_rejects_host_and_misshapen_tensors(lib):
    """The Python binding refuses, before any launch, tensors the kernels
    would misread: host tensors, wrong shapes or dtypes, non-dense views."""
    import torch
    import qlora_bit_frozen_b200 as q
    O, I, r, R = 64, 128, 8, 4
    w = q.QuantizedWeight(q.FMT_NF4_DQ, O, I, 64, 256, 4, torch.zeros(O * I // 2, dtype=torch.uint8),
                          torch.zeros(O * I // 64, dtype=torch.uint8), torch.zeros(1), torch.zeros(1))
    X = torch.zeros(R, I, dtype=torch.bfloat16)
    A = torch.zeros(r, I)
    B = torch.zeros(O, r)
    dY = torch.zeros(R, O, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        q.qlora_linear_fwd(w, X, A, B, 16.0)
    with pytest.raises(ValueError, match="CUDA"):
        q.qlora_linear_bwd(w, X, dY, A, B, 16.0)
    with pytest.raises(ValueError, match="CUDA"):
        q.qlora_dequantize(w)
    with pytest.raises(ValueError, match="CUDA"):
        q.qlora_merge(w, A, B, 16.0)
    p = torch.zeros(16)
    with pytest.raises(ValueError, match="CUDA"):
        q.qlora_adam_step(p, p.clone(), p.clone(), p.clone(), 1, 1e-3)
    with pytest.raises(ValueError):
        q.qlora_merge(w, A.t(), B, 16.0)                      # wrong shape
    with pytest.raises(ValueError):
        q.qlora_adam_step(p, p[::2].clone(), p.clone(), p.clone(), 1, 1e-3)   # sizes differ
    with pytest.raises(ValueError):
        q.qlora_linear_fwd(w, X.to(torch.float16), A, B, 16.0)  # unsupported activation dtype

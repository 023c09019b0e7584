"""The allocation-free NF4 quantizer (qlora_quantize_nf4_noalloc).

It exists for callers that cannot allocate device memory themselves -- e.g.
a plugin inside a framework whose caching allocator owns the GPU memory, or
a C caller with no allocator -- and therefore cannot hand the library a
workspace.  Checked here through the C ABI against qlora_quantize_nf4 (which
uses a caller workspace) and against the CPU oracle: two calls in a row must
both give bit-identical packed codes, scale codes, t_g and mu, since the
shared scratch keeps the previous call's contents.  This file is collected
last on purpose."""
import ctypes

import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(O, I, B, C, dev):
    N = O * I
    M = -(-N // B)
    S = -(-M // C)
    return (torch.empty((N + 1) // 2, dtype=torch.uint8, device=dev), torch.empty(M, dtype=torch.uint8, device=dev),
            torch.empty(S, dtype=torch.float32, device=dev), torch.empty(1, dtype=torch.float32, device=dev))


def test_noalloc_matches_workspace_entry_point_twice():
    from qlora_bit_frozen_b200 import _ffi, build
    build.build()
    lib = _ffi.load()
    assert torch.cuda.is_available()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [(synth.weight(synth.workload("qwen3_0.6b_attn_qv"), 0), 64, 256),
             (synth.weight(synth.workload("fp32_single_256"), 0), 64, 256),   # has an all-zero block
             (synth.normal(31, (7, 33), std=0.02), 16, 3)]                    # odd N, partial groups
    for W_host, B, C in cases:
        W = torch.from_numpy(W_host).cuda()
        O, I = W.shape
        ref = _outputs(O, I, B, C, W.device)
        ws = torch.empty(lib.qlora_quantize_nf4_workspace_bytes(O * I, B, C), dtype=torch.uint8, device=W.device)
        st = lib.qlora_quantize_nf4(_ptr(W), O, I, B, C, *map(_ptr, ref), _ptr(ws), ws.numel(), stream)
        assert st == _ffi.OK
        ow = oracle.quantize_nf4(W_host, B, C)
        want = (ow.codes, ow.qcodes, np.asarray(ow.t, np.float32), np.array([ow.mu], np.float32))
        for _ in range(2):  # the second call runs on scratch holding the first call's contents
            out = _outputs(O, I, B, C, W.device)
            st = lib.qlora_quantize_nf4_noalloc(_ptr(W), O, I, B, C, *map(_ptr, out), stream)
            assert st == _ffi.OK, lib.qlora_status_string(st)
            for a, b, o in zip(out, ref, want):
                got = a.cpu().numpy().view(np.uint8)
                assert np.array_equal(got, b.cpu().numpy().view(np.uint8))
                assert np.array_equal(got, np.ascontiguousarray(o).view(np.uint8))


def test_noalloc_rejects_inputs_beyond_its_scratch():
    from qlora_bit_frozen_b200 import _ffi
    lib = _ffi.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    d = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    st = lib.qlora_quantize_nf4_noalloc(d, 1 << 20, 1 << 10, 64, 256, d, d, d, d, stream)
    assert st == _ffi.ERR_WORKSPACE

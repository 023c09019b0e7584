"""Checkpointing a quantized weight: the packed buffers are the canonical
serialization.  state_dict() -> file -> from_state_dict() keeps every byte,
and a truncated, mistyped or missing buffer is refused before it can reach
the device.  CPU only (buffers held in host tensors)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import qlora_bit_frozen_b200 as q


def _host_weight(fmt):
    W = synth.normal(70, (96, 256), std=0.02)
    if fmt == "nf4":
        ow = oracle.quantize_nf4(W, 64, 3)
        return q.QuantizedWeight(q.FMT_NF4_DQ, 96, 256, 64, 3, 4, torch.from_numpy(ow.codes),
                                 torch.from_numpy(ow.qcodes), torch.from_numpy(ow.t),
                                 torch.tensor([ow.mu], dtype=torch.float32))
    ow = oracle.quantize_affine(W, 8, 32)
    return q.QuantizedWeight(q.FMT_AFFINE, 96, 256, 32, 0, 8, torch.from_numpy(ow.codes),
                             scale=torch.from_numpy(ow.scale), bias=torch.from_numpy(ow.bias))


@pytest.mark.parametrize("fmt", ["nf4", "affine"])
def test_state_dict_file_round_trip_is_byte_exact(tmp_path, fmt):
    w = _host_weight(fmt)
    path = tmp_path / "w.npz"
    np.savez(path, **w.state_dict())
    with np.load(path) as f:
        w2 = q.QuantizedWeight.from_state_dict({k: f[k] for k in f.files}, device="cpu")
    assert (w2.fmt, w2.O, w2.I, w2.block, w2.group, w2.bits) == (w.fmt, w.O, w.I, w.block, w.group, w.bits)
    for k in q.QuantizedWeight._BUFFERS:
        a, b = getattr(w, k), getattr(w2, k)
        assert (a is None) == (b is None), k
        if a is not None:
            assert a.dtype == b.dtype and np.array_equal(a.numpy().view(np.uint8), b.numpy().view(np.uint8)), k
    assert w2.payload_bytes() == w.payload_bytes()


def test_bad_checkpoints_are_refused():
    d = _host_weight("nf4").state_dict()
    bad = dict(d, codes=d["codes"][:-1])
    with pytest.raises(ValueError, match="codes"):
        q.QuantizedWeight.from_state_dict(bad, device="cpu")
    bad = dict(d, group_absmax=d["group_absmax"].astype(np.float64))
    with pytest.raises(ValueError, match="group_absmax"):
        q.QuantizedWeight.from_state_dict(bad, device="cpu")
    bad = {k: v for k, v in d.items() if k != "mean"}
    with pytest.raises(ValueError, match="mean"):
        q.QuantizedWeight.from_state_dict(bad, device="cpu")
    with pytest.raises(ValueError):
        q.QuantizedWeight.from_state_dict(dict(d, bits=8), device="cpu")

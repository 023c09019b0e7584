"""Shared test helpers: device transfer of synthetic inputs and error metrics."""
import numpy as np

import synth


def rel_fro(got, ref) -> float:
    """||got - ref||_F / ||ref||_F in fp64."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    return float(num / den) if den > 0 else float(num)


TOL = {"fp32": 1e-5, "bf16": 1e-2}


def to_dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def to_host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def bf16_bits_of(t):
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def layer_inputs(wl: "synth.Workload", li: int, R=None):
    """Host inputs of linear li: dict with W, A, B, x (fp32 values the oracle
    sees), xd (device activation), dy, dyd."""
    W = synth.weight(wl, li)
    A, B = synth.adapters(wl, li)
    xw, xb, dw, db = synth.activations(wl, li, R)
    if wl.compute == "bf16":
        xd, dyd = to_dev_bf16(xb), to_dev_bf16(db)
    else:
        xd, dyd = to_dev_f32(xw), to_dev_f32(dw)
    return dict(W=W, A=A, B=B, x=xw, xd=xd, dy=dw, dyd=dyd)

"""GPU parity of the training-lifecycle entry points around the layer: the
adapter Adam step and the merged fp32 export, through the C ABI, against
the CPU oracle.

Tolerances are per element and follow from the fp32 arithmetic of the
kernels (unit roundoff u = 2^-24):
  merge: the decoded weight is exact; the rank-r delta is r FMAs in k order
         (error <= r u sum_k |B_ok A_ki|), then one product and one sum:
         |err| <= u |W| + |s| (r + 1) u sum_k |B_ok A_ki|, taken with a
         factor of 2 of margin.
  Adam:  m and v are two products and a sum (v one product more), so
         |dm| <= 3u (|b1 m| + |(1-b1) g|), |dv| <= 4u (|b2 v| + |(1-b2) g^2|);
         the step lr m_hat / (sqrt(v_hat) + eps) adds a few roundings
         (<= 12u relative) and carries dm / bc1; p - step rounds once."""
import numpy as np
import pytest

import oracle
import synth
from helpers import rel_fro, to_dev_f32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import qlora_bit_frozen_b200 as q  # noqa: E402

U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _built():
    from qlora_bit_frozen_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _weights(fmt, W, B=64, C=256, bits=4, G=64):
    if fmt == "nf4":
        return q.qlora_quantize_nf4(to_dev_f32(W), B, C), oracle.quantize_nf4(W, B, C)
    return q.qlora_quantize_affine(to_dev_f32(W), bits, G), oracle.quantize_affine(W, bits, G)


def _merge_bound(ref, A, Bm, s, r):
    mag = np.abs(Bm.astype(np.float64)) @ np.abs(A.astype(np.float64))
    return 2.0 * (U * np.abs(ref) + abs(s) * (r + 1) * U * mag) + 1e-30


# ----------------------------------------------------------------- merge

MERGE_CASES = [
    # fmt, O, I, r, bits, G   (tiles of 64 x 64: ragged rows and columns)
    ("nf4", 200, 320, 8, 4, 64),
    ("nf4", 130, 256, 1, 4, 64),
    ("nf4", 96, 192, 33, 4, 64),       # two rank chunks, the second of one rank
    ("nf4", 1024, 4096, 64, 4, 64),
    ("affine", 136, 384, 16, 4, 64),
    ("affine", 72, 256, 8, 8, 32),
]


@pytest.mark.parametrize("fmt,O,I,r,bits,G", MERGE_CASES)
def test_merge_matches_oracle(fmt, O, I, r, bits, G):
    W = synth.normal(300 + O, (O, I), std=0.02)
    gw, ow = _weights(fmt, W, bits=bits, G=G)
    A = synth.normal(301, (r, I), std=0.02)
    Bm = synth.normal(302, (O, r), std=0.02)
    alpha = 2.0 * r
    s = float(np.float32(alpha) / np.float32(r))
    got = q.qlora_merge(gw, to_dev_f32(A), to_dev_f32(Bm), alpha).cpu().numpy().astype(np.float64)
    ref = oracle.merge(ow, A, Bm, r, alpha)
    assert np.all(np.abs(got - ref) <= _merge_bound(ref, A, Bm, s, r))
    assert rel_fro(got, ref) <= 1e-6


@pytest.mark.parametrize("fmt", ["nf4", "affine"])
def test_merge_zero_adapter_is_the_dequantized_weight(fmt):
    W = synth.normal(310, (192, 256), std=0.02)
    gw, _ = _weights(fmt, W)
    r = 8
    A = to_dev_f32(synth.normal(311, (r, 256), std=0.02))
    Z = torch.zeros((192, r), device="cuda")
    Wh = q.qlora_dequantize(gw)
    assert torch.equal(q.qlora_merge(gw, A, Z, 16.0), Wh)
    Bm = to_dev_f32(synth.normal(312, (192, r), std=0.02))
    assert torch.equal(q.qlora_merge(gw, A, Bm, 0.0), Wh)


def test_merge_unaligned_shapes_and_output():
    """Rows that are not a multiple of 4 wide (blocks straddle rows) and an
    output that does not start on a 16-byte boundary take the per-element
    path; both must agree with the oracle."""
    O, I, r = 70, 130, 5
    W = synth.normal(320, (O, I), std=0.02)
    gw, ow = _weights("nf4", W, B=64, C=3)
    A = synth.normal(321, (r, I), std=0.02)
    Bm = synth.normal(322, (O, r), std=0.02)
    s = float(np.float32(10.0) / np.float32(r))
    ref = oracle.merge(ow, A, Bm, r, 10.0)
    got = q.qlora_merge(gw, to_dev_f32(A), to_dev_f32(Bm), 10.0).cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= _merge_bound(ref, A, Bm, s, r))
    # same weight, I = 128: aligned rows but an output offset by one float
    W2 = synth.normal(323, (64, 128), std=0.02)
    gw2, ow2 = _weights("nf4", W2)
    A2 = synth.normal(324, (r, 128), std=0.02)
    B2 = synth.normal(325, (64, r), std=0.02)
    buf = torch.empty(64 * 128 + 1, device="cuda")
    out = buf[1:].view(64, 128)
    q.qlora_merge(gw2, to_dev_f32(A2), to_dev_f32(B2), 10.0, out=out)
    ref2 = oracle.merge(ow2, A2, B2, r, 10.0)
    got2 = out.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got2 - ref2) <= _merge_bound(ref2, A2, B2, s, r))


# ----------------------------------------------------------------- Adam

def _adam_bounds(p, g, m, v, t, lr, b1, b2, eps, po, mo, vo):
    g, m, v, p = (x.astype(np.float64) for x in (g, m, v, p))
    bm = 3 * U * (np.abs(b1 * m) + np.abs((1 - b1) * g)) + 1e-45
    bv = 4 * U * (np.abs(b2 * v) + np.abs((1 - b2) * g * g)) + 1e-45
    bc1 = 1 - b1 ** t
    bc2 = 1 - b2 ** t
    den = np.sqrt(vo / bc2) + eps
    step = np.abs(p - po)
    bp = U * np.abs(po) + 12 * U * step + lr * (bm / bc1) / den
    return 2 * bm, 2 * bv, 2 * bp + 1e-45


@pytest.mark.parametrize("n,page", [(100003, 0), (100003, 4096), (777, 0)])
def test_adam_steps_match_oracle(n, page):
    lr, b1, b2, eps = 1e-3, 0.9, 0.999, 1e-8
    b1f, b2f = float(np.float32(b1)), float(np.float32(b2))
    lrf, epsf = float(np.float32(lr)), float(np.float32(eps))
    p = synth.normal(400, n, std=0.02)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    dp, dm, dv = to_dev_f32(p), to_dev_f32(m), to_dev_f32(v)
    for t in range(1, 6):
        g = synth.normal(401 + t, n, std=1e-2)
        g[::97] = 0.0                     # some exact zeros
        g[5::101] *= 1e3                  # and some large entries
        dg = to_dev_f32(g)
        hp, hm, hv = (x.cpu().numpy() for x in (dp, dm, dv))
        q.qlora_adam_step(dp, dg, dm, dv, t, lr, b1, b2, eps, page_elems=page)
        po, mo, vo = oracle.adam_step(hp, g, hm, hv, t, lr, b1, b2, eps)
        bm, bv, bp = _adam_bounds(hp, g, hm, hv, t, lrf, b1f, b2f, epsf, po, mo, vo)
        gp, gm, gv = (x.cpu().numpy().astype(np.float64) for x in (dp, dm, dv))
        assert np.all(np.abs(gm - mo) <= bm), t
        assert np.all(np.abs(gv - vo) <= bv), t
        assert np.all(np.abs(gp - po) <= bp), t


def test_adam_paged_equals_single_launch_bitwise():
    n = 50001
    p = to_dev_f32(synth.normal(410, n, std=0.02))
    g = to_dev_f32(synth.normal(411, n, std=1e-2))
    m = to_dev_f32(synth.normal(412, n, std=1e-3))
    v = to_dev_f32(np.abs(synth.normal(413, n, std=1e-4)))
    ref = [x.clone() for x in (p, m, v)]
    q.qlora_adam_step(ref[0], g, ref[1], ref[2], 7, 1e-3)
    for page in (4096, 1000, n, 3 * n):
        got = [x.clone() for x in (p, m, v)]
        q.qlora_adam_step(got[0], g, got[1], got[2], 7, 1e-3, page_elems=page)
        for a, b in zip(got, ref):
            assert torch.equal(a, b), page


def test_training_loop_keeps_packed_weight_and_exports():
    """Quantize, then three steps of forward, backward and an Adam step on a
    flat arena holding A and B; the packed payload stays byte-identical, the
    arena follows the oracle's Adam on the GPU's own gradients, and the
    export matches the oracle's merge of the trained factors."""
    O, I, r, R, alpha = 256, 512, 8, 64, 16.0
    W = synth.normal(420, (O, I), std=0.02)
    gw, ow = _weights("nf4", W)
    before = [t.clone() for t in (gw.codes, gw.scale_codes, gw.group_absmax, gw.mean)]
    nA, nB = r * I, O * r
    arena = torch.zeros(nA + nB, device="cuda")
    arena[:nA] = to_dev_f32(synth.normal(421, nA, std=0.02))   # B starts at zero
    m = torch.zeros_like(arena)
    v = torch.zeros_like(arena)
    grads = torch.zeros_like(arena)
    A = arena[:nA].view(r, I)
    Bm = arena[nA:].view(O, r)
    lr = 1e-2
    for t in range(1, 4):
        X = to_dev_f32(synth.normal(430 + t, (R, I)))
        dY = to_dev_f32(synth.normal(440 + t, (R, O)))
        Y, Uf = q.qlora_linear_fwd(gw, X, A, Bm, alpha)
        _, dA, dB = q.qlora_linear_bwd(gw, X, dY, A, Bm, alpha, U=Uf, want_dx=False,
                                       dA=grads[:nA].view(r, I), dB=grads[nA:].view(O, r))
        hp, hg, hm, hv = (x.cpu().numpy() for x in (arena, grads, m, v))
        q.qlora_adam_step(arena, grads, m, v, t, lr)
        po, mo, vo = oracle.adam_step(hp, hg, hm, hv, t, lr)
        assert rel_fro(arena.cpu().numpy(), po) <= 1e-6
    for a, b in zip(before, (gw.codes, gw.scale_codes, gw.group_absmax, gw.mean)):
        assert torch.equal(a, b)
    hA, hB = A.cpu().numpy(), Bm.cpu().numpy()
    got = q.qlora_merge(gw, A.contiguous(), Bm.contiguous(), alpha).cpu().numpy().astype(np.float64)
    ref = oracle.merge(ow, hA, hB, r, alpha)
    s = float(np.float32(alpha) / np.float32(r))
    assert np.all(np.abs(got - ref) <= _merge_bound(ref, hA, hB, s, r))


def test_checkpoint_round_trip_keeps_outputs_bitwise(tmp_path):
    """A quantized weight written to a file with state_dict() and read back
    with from_state_dict() decodes and multiplies to the same bits."""
    W = synth.normal(450, (256, 512), std=0.02)
    gw, _ = _weights("nf4", W)
    path = tmp_path / "w.npz"
    np.savez(path, **gw.state_dict())
    with np.load(path) as f:
        gw2 = q.QuantizedWeight.from_state_dict({k: f[k] for k in f.files})
    assert torch.equal(q.qlora_dequantize(gw), q.qlora_dequantize(gw2))
    X = to_dev_f32(synth.normal(451, (64, 512))).to(torch.bfloat16)
    A = to_dev_f32(synth.normal(452, (8, 512), std=0.02))
    Bm = to_dev_f32(synth.normal(453, (256, 8), std=0.02))
    Y1, _ = q.qlora_linear_fwd(gw, X, A, Bm, 16.0)
    Y2, _ = q.qlora_linear_fwd(gw2, X, A, Bm, 16.0)
    assert torch.equal(Y1, Y2)

"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact for codes, scale codes, t_g, mu and dequantized values; relative
Frobenius error <= 1e-5 (fp32 compute) or <= 1e-2 (bf16 compute) for Y, dX,
dA and dB.  Full-size workloads compare sampled rows of Y / dX (the oracle
computes those rows one by one) and the full dA / dB."""
import numpy as np
import pytest

import oracle
import synth
from helpers import TOL, bf16_bits_of, layer_inputs, rel_fro, to_dev_f32, to_host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import qlora_bit_frozen_b200 as q  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _built():
    from qlora_bit_frozen_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _assert_same_nf4(gw, ow):
    assert np.array_equal(gw.codes.cpu().numpy(), ow.codes), "packed codes differ"
    assert np.array_equal(gw.scale_codes.cpu().numpy(), ow.qcodes), "scale codes differ"
    assert np.array_equal(gw.group_absmax.cpu().numpy().view(np.uint32), ow.t.view(np.uint32)), "t_g differ"
    assert np.float32(gw.mean.cpu().numpy()[0]).view(np.uint32) == np.float32(ow.mu).view(np.uint32), "mu differs"


# ----------------------------------------------------------------- quantizers

NF4_CASES = [
    ("fp32_single_256", 0, 64, 256),      # forced zero block
    ("qwen3_0.6b_attn_qv", 0, 64, 256),
    ("14b_layer", 4, 64, 256),            # 17408 x 5120 with 0.1% outliers x20
    ("raw_odd", (1, 101), 64, 256),       # odd N, partial block
    ("raw_odd", (7, 33), 16, 3),          # partial groups
    ("raw_odd", (3, 4096), 64, 5),        # groups straddle rows
]


def _case_weight(name, li):
    if name == "raw_odd":
        return synth.normal(99, li, std=0.02)
    return synth.weight(synth.workload(name), li)


@pytest.mark.parametrize("name,li,B,C", NF4_CASES)
def test_quantize_nf4_bit_exact(name, li, B, C):
    W = _case_weight(name, li)
    ow = oracle.quantize_nf4(W, B, C)
    gw = q.qlora_quantize_nf4(to_dev_f32(W), B, C)
    _assert_same_nf4(gw, ow)
    Wh = q.qlora_dequantize(gw).cpu().numpy()
    assert np.array_equal(Wh.view(np.uint32), oracle.dequantize(ow).view(np.uint32))


def test_quantize_nf4_deterministic_and_empty():
    W = to_dev_f32(synth.normal(5, (512, 1024), std=0.02))
    a = q.qlora_quantize_nf4(W)
    b = q.qlora_quantize_nf4(W)
    for x, y in ((a.codes, b.codes), (a.scale_codes, b.scale_codes), (a.group_absmax, b.group_absmax),
                 (a.mean, b.mean)):
        assert torch.equal(x, y)
    e = q.qlora_quantize_nf4(torch.zeros((0, 64), device="cuda"))
    assert e.codes.numel() == 0 and float(e.mean.item()) == 0.0


def test_quantize_nonfinite_rejected():
    W = torch.ones((4, 64), device="cuda")
    W[2, 5] = float("nan")
    with pytest.raises(q.QLoraError) as ei:
        q.qlora_quantize_nf4(W)
    assert ei.value.status == 4
    W[2, 5] = float("inf")
    with pytest.raises(q.QLoraError):
        q.qlora_quantize_affine(W, 4, 64)


@pytest.mark.parametrize("bits,G", [(4, 32), (4, 64), (4, 128), (8, 32), (8, 64), (8, 128)])
def test_quantize_affine_bit_exact(bits, G):
    W = synth.normal(321 + bits + G, (1024, 1024), std=0.02)
    ow = oracle.quantize_affine(W, bits, G)
    gw = q.qlora_quantize_affine(to_dev_f32(W), bits, G)
    assert np.array_equal(gw.codes.cpu().numpy(), ow.codes)
    assert np.array_equal(gw.scale.cpu().numpy().view(np.uint32), ow.scale.view(np.uint32))
    assert np.array_equal(gw.bias.cpu().numpy().view(np.uint32), ow.bias.view(np.uint32))
    Wh = q.qlora_dequantize(gw).cpu().numpy()
    assert np.array_equal(Wh.view(np.uint32), oracle.dequantize(ow).view(np.uint32))


@pytest.mark.parametrize("name,li,B", [("fp32_single_256", 0, 64), ("qwen3_0.6b_attn_qv", 0, 64),
                                       ("raw_odd", (1, 101), 64), ("raw_odd", (7, 33), 16)])
def test_quantize_nf4_fp32scale_bit_exact(name, li, B):
    """Legacy scale storage ("NF4 representation": one fp32 absmax per
    block): codes and s_b bit-exact against the oracle, and the dequantized
    weight c[code] * s_b too."""
    W = _case_weight(name, li)
    ow = oracle.quantize_nf4_legacy(W, B)
    gw = q.qlora_quantize_nf4_fp32scale(to_dev_f32(W), B)
    assert np.array_equal(gw.codes.cpu().numpy(), ow.codes)
    assert np.array_equal(gw.scale.cpu().numpy().view(np.uint32), ow.scale.view(np.uint32))
    assert gw.payload_bytes() == oracle.legacy_payload_bytes(W.size, B)
    Wh = q.qlora_dequantize(gw).cpu().numpy()
    assert np.array_equal(Wh.view(np.uint32), oracle.dequantize(ow).view(np.uint32))


# ------------------------------------------------------------ forward/backward

def _run_layer(wl, li, rows=None, want=("Y", "dX", "dA", "dB"), fmt="nf4", bits=4, G=64, R=None):
    d = layer_inputs(wl, li, R)
    Wd = to_dev_f32(d["W"])
    if fmt == "nf4":
        gw = q.qlora_quantize_nf4(Wd, wl.block, wl.group)
        ow = oracle.quantize_nf4(d["W"], wl.block, wl.group)
        _assert_same_nf4(gw, ow)
    elif fmt == "nf4_fp32scale":
        gw = q.qlora_quantize_nf4_fp32scale(Wd, wl.block)
        ow = oracle.quantize_nf4_legacy(d["W"], wl.block)
        assert np.array_equal(gw.codes.cpu().numpy(), ow.codes)
        assert np.array_equal(gw.scale.cpu().numpy().view(np.uint32), ow.scale.view(np.uint32))
    else:
        gw = q.qlora_quantize_affine(Wd, bits, G)
        ow = oracle.quantize_affine(d["W"], bits, G)
    A, B = to_dev_f32(d["A"]), to_dev_f32(d["B"])
    Y, U = q.qlora_linear_fwd(gw, d["xd"], A, B, wl.alpha)
    dX, dA, dB = q.qlora_linear_bwd(gw, d["xd"], d["dyd"], A, B, wl.alpha, U=U,
                                    want_da="dA" in want, want_db="dB" in want)
    torch.cuda.synchronize()
    Rr = d["x"].shape[0]
    sel = np.arange(Rr) if rows is None else rows
    oY, oU = oracle.linear_fwd(ow, d["x"], d["A"], d["B"], wl.r, wl.alpha, rows=sel)
    odX, odA, odB = oracle.linear_bwd(ow, d["x"], d["dy"], d["A"], d["B"], wl.r, wl.alpha, rows=sel,
                                      want_da="dA" in want, want_db="dB" in want)
    errs = {
        "Y": rel_fro(to_host(Y)[sel], oY),
        "U": rel_fro(to_host(U)[sel], oU),
        "dX": rel_fro(to_host(dX)[sel], odX),
    }
    if "dA" in want:
        errs["dA"] = rel_fro(to_host(dA), odA)
    if "dB" in want:
        errs["dB"] = rel_fro(to_host(dB), odB)
    return errs


def _check(errs, tol):
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, f"relative Frobenius errors above {tol}: {errs}"


def test_fp32_single_linear():
    wl = synth.workload("fp32_single_256")
    _check(_run_layer(wl, 0), TOL["fp32"])


@pytest.mark.parametrize("R", [0, 1, 7, 64, 130])
def test_fp32_ragged_rows(R):
    wl = synth.workload("fp32_single_256", R=R)
    if R == 0:
        d = layer_inputs(wl, 0)
        gw = q.qlora_quantize_nf4(to_dev_f32(d["W"]))
        A, B = to_dev_f32(d["A"]), to_dev_f32(d["B"])
        X = torch.empty((0, 256), device="cuda")
        Y, U = q.qlora_linear_fwd(gw, X, A, B, wl.alpha)
        dX, dA, dB = q.qlora_linear_bwd(gw, X, X[:, :256], A, B, wl.alpha)
        assert Y.shape == (0, 256) and float(dA.abs().sum()) == 0.0 and float(dB.abs().sum()) == 0.0
        return
    _check(_run_layer(wl, 0), TOL["fp32"])


def test_bf16_qwen_attention_full():
    wl = synth.workload("qwen3_0.6b_attn_qv")
    for li in range(len(wl.linears)):
        _check(_run_layer(wl, li), TOL["bf16"])


@pytest.mark.parametrize("R", [1, 16, 17, 31, 32, 48, 64, 100, 128, 130, 256, 1000])
def test_bf16_ragged_token_counts(R):
    # 16/32-token tiles (TMA loads of 4 and 2 K steps, adapter tile outside
    # the ring), 64..256-token tiles, split-K and not, ragged last tile
    wl = synth.workload("qwen3_0.6b_attn_qv", R=R)
    _check(_run_layer(wl, 1), TOL["bf16"])


@pytest.mark.parametrize("R", [24, 200])
def test_bf16_ragged_token_counts_wide_output(R):
    wl = synth.workload("qwen3_0.6b_attn_qv", R=R)
    _check(_run_layer(wl, 0), TOL["bf16"])


@pytest.mark.parametrize("R", [16, 4096])
def test_bf16_linear_is_deterministic(R):
    """Split-K partials and the side-product split partials are reduced in a
    fixed order: two runs on the same inputs agree bit for bit."""
    wl = synth.workload("qwen3_0.6b_attn_qv", R=R)
    d = layer_inputs(wl, 0)
    gw = q.qlora_quantize_nf4(to_dev_f32(d["W"]))
    A, B = to_dev_f32(d["A"]), to_dev_f32(d["B"])
    outs = []
    for _ in range(2):
        Y, U = q.qlora_linear_fwd(gw, d["xd"], A, B, wl.alpha)
        dX, dA, dB = q.qlora_linear_bwd(gw, d["xd"], d["dyd"], A, B, wl.alpha, U=U)
        torch.cuda.synchronize()
        outs.append([bf16_bits_of(Y), U.cpu().numpy(), bf16_bits_of(dX), dA.cpu().numpy(), dB.cpu().numpy()])
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b)


def test_bf16_identity_input_recovers_decoded_weight_bitwise():
    """X = I (R = I) and B = 0 give Y = bf16(W_hat)^T exactly; dY = I (R = O)
    and B = 0 give dX = bf16(W_hat) exactly: one nonzero product per output,
    so every decoded weight is checked bit for bit."""
    O, I = 256, 512
    W = synth.normal(3, (O, I), std=0.02)
    gw = q.qlora_quantize_nf4(to_dev_f32(W))
    ow = oracle.quantize_nf4(W)
    _assert_same_nf4(gw, ow)
    ref = torch.from_numpy(oracle.dequantize(ow)).to(torch.bfloat16)
    r = 8
    A = torch.zeros((r, I), device="cuda")
    Bz = torch.zeros((O, r), device="cuda")
    Xi = torch.eye(I, device="cuda", dtype=torch.bfloat16)
    Y, _ = q.qlora_linear_fwd(gw, Xi, A, Bz, 16.0)
    assert np.array_equal(bf16_bits_of(Y), bf16_bits_of(ref.t()))
    dYi = torch.eye(O, device="cuda", dtype=torch.bfloat16)
    dX, _, _ = q.qlora_linear_bwd(gw, None, dYi, A, Bz, 16.0, want_da=False, want_db=False)
    assert np.array_equal(bf16_bits_of(dX), bf16_bits_of(ref))


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("bits", [4, 8])
def test_bf16_identity_input_recovers_affine_weight_bitwise(bits, G):
    """4- and 8-bit affine weights in the tensor-core kernel: X = I (R = I)
    and B = 0 give Y = bf16(W_hat)^T exactly, dY = I gives dX = bf16(W_hat);
    every decoded weight (scale * code + bias of its group) checked bit for
    bit."""
    O, I = 256, 512
    W = synth.normal(5 + G + bits, (O, I), std=0.02)
    gw = q.qlora_quantize_affine(to_dev_f32(W), bits, G)
    ow = oracle.quantize_affine(W, bits, G)
    ref = torch.from_numpy(oracle.dequantize(ow)).to(torch.bfloat16)
    r = 8
    A = torch.zeros((r, I), device="cuda")
    Bz = torch.zeros((O, r), device="cuda")
    Xi = torch.eye(I, device="cuda", dtype=torch.bfloat16)
    Y, _ = q.qlora_linear_fwd(gw, Xi, A, Bz, 16.0)
    assert np.array_equal(bf16_bits_of(Y), bf16_bits_of(ref.t()))
    dYi = torch.eye(O, device="cuda", dtype=torch.bfloat16)
    dX, _, _ = q.qlora_linear_bwd(gw, None, dYi, A, Bz, 16.0, want_da=False, want_db=False)
    assert np.array_equal(bf16_bits_of(dX), bf16_bits_of(ref))


@pytest.mark.parametrize("fmt,bits,G", [("nf4", 4, 64), ("nf4_fp32scale", 4, 64), ("affine", 4, 32),
                                        ("affine", 8, 128)])
def test_bf16_identity_input_pre_decoded_bitwise(fmt, bits, G):
    """From 2048 tokens on 256-token tiles the input gradient decodes the
    weight to bf16 once per call and the GEMM reads that copy: dY = I (4096
    tokens, W 4096 x 1024) gives dX = bf16(W_hat) bit for bit, for every
    weight format; X = I (4096 tokens, W 1024 x 4096) checks the forward at
    the same size (Y = bf16(W_hat)^T)."""
    def quant(W):
        if fmt == "nf4":
            return q.qlora_quantize_nf4(to_dev_f32(W)), oracle.quantize_nf4(W)
        if fmt == "nf4_fp32scale":
            return q.qlora_quantize_nf4_fp32scale(to_dev_f32(W), 64), oracle.quantize_nf4_legacy(W, 64)
        return q.qlora_quantize_affine(to_dev_f32(W), bits, G), oracle.quantize_affine(W, bits, G)
    r = 8
    for O, I, fwd in ((1024, 4096, True), (4096, 1024, False)):
        W = synth.normal(40 + bits + G + O, (O, I), std=0.02)
        gw, ow = quant(W)
        ref = torch.from_numpy(oracle.dequantize(ow)).to(torch.bfloat16)
        A = torch.zeros((r, I), device="cuda")
        Bz = torch.zeros((O, r), device="cuda")
        if fwd:
            Xi = torch.eye(I, device="cuda", dtype=torch.bfloat16)
            Y, _ = q.qlora_linear_fwd(gw, Xi, A, Bz, 16.0)
            assert np.array_equal(bf16_bits_of(Y), bf16_bits_of(ref.t()))
        else:
            dYi = torch.eye(O, device="cuda", dtype=torch.bfloat16)
            dX, _, _ = q.qlora_linear_bwd(gw, None, dYi, A, Bz, 16.0, want_da=False, want_db=False)
            assert np.array_equal(bf16_bits_of(dX), bf16_bits_of(ref))


@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("R", [40, 100, 300, 4096])
@pytest.mark.parametrize("bits", [4, 8])
def test_bf16_affine_tensor_core_path(bits, G, R):
    """4- and 8-bit affine weights at many tokens run on the tensor-core
    kernel (split-K at 40 and 100 tokens, a ragged 300 over 128- and
    64-token tiles, 256-token tiles at 4096); 64 sampled rows."""
    wl = synth.workload("qwen3_0.6b_attn_qv", R=R)
    rows = synth.sample_rows(R, 64, seed=G + R + bits)
    _check(_run_layer(wl, 0, rows=rows, fmt="affine", bits=bits, G=G), TOL["bf16"])


def test_bf16_adapter_only_and_zero_alpha():
    wl = synth.workload("qwen3_0.6b_attn_qv", R=256)
    d = layer_inputs(wl, 1)
    gw = q.qlora_quantize_nf4(to_dev_f32(d["W"]))
    ow = oracle.quantize_nf4(d["W"])
    A, B = to_dev_f32(d["A"]), to_dev_f32(d["B"])
    Y0, _ = q.qlora_linear_fwd(gw, d["xd"], A, B, 0.0)
    oY0, _ = oracle.linear_fwd(ow, d["x"], d["A"], d["B"], wl.r, 0.0)
    assert rel_fro(to_host(Y0), oY0) <= TOL["bf16"]
    for r in (1, 16, 32, 64):
        A2 = to_dev_f32(synth.normal(50 + r, (r, 1024), std=0.02))
        B2 = to_dev_f32(synth.normal(60 + r, (1024, r), std=0.02))
        Y, U = q.qlora_linear_fwd(gw, d["xd"], A2, B2, 2.0 * r)
        dX, dA, dB = q.qlora_linear_bwd(gw, d["xd"], d["dyd"], A2, B2, 2.0 * r)  # U recomputed
        oY, _ = oracle.linear_fwd(ow, d["x"], A2.cpu().numpy(), B2.cpu().numpy(), r, 2.0 * r)
        odX, odA, odB = oracle.linear_bwd(ow, d["x"], d["dy"], A2.cpu().numpy(), B2.cpu().numpy(), r, 2.0 * r)
        _check({"Y": rel_fro(to_host(Y), oY), "dX": rel_fro(to_host(dX), odX),
                "dA": rel_fro(to_host(dA), odA), "dB": rel_fro(to_host(dB), odB)}, TOL["bf16"])


@pytest.mark.parametrize("name", ["bw_sweep_4096", "bw_sweep_12288"])
@pytest.mark.parametrize("R", [1, 2, 4, 8, 13, 16, 128])
def test_bf16_small_row_sweep_nf4(name, R):
    wl = synth.workload(name, R=R)
    _check(_run_layer(wl, 0, want=("Y", "dX")), TOL["bf16"])


@pytest.mark.parametrize("R", [9, 16])
def test_bf16_few_token_gemv_where_tiles_do_not_apply(R):
    """W 2048 x 1088 (I % 128 = 64: no tensor-core tiles) at 9 and 16 tokens:
    the few-token kernels with two 8-token MMA tiles, forward and dX,
    against the oracle (Y, U, dX; dA and dB by the side products)."""
    wl = synth.workload("qwen3_0.6b_attn_qv", R=R)
    wl.linears = [synth.Linear("odd_i", 2048, 1088)]
    _check(_run_layer(wl, 0), TOL["bf16"])


@pytest.mark.parametrize("name", ["bw_sweep_4096", "bw_sweep_12288"])
@pytest.mark.parametrize("R", [1, 16, 128])
@pytest.mark.parametrize("bits,G", [(4, 32), (4, 64), (4, 128), (8, 32), (8, 64), (8, 128)])
def test_bf16_small_row_sweep_affine(name, R, bits, G):
    """Affine weights at 1, 16 and 128 tokens against both sweep matrices:
    the single-token, the up-to-16-token and the many-token paths, for
    every (bits, G) of the sweep.  The 128-token case on the larger matrix
    compares 32 sampled rows (the oracle computes them one by one)."""
    wl = synth.workload(name, R=R)
    rows = synth.sample_rows(R, 32, seed=R + bits + G) if (R == 128 and name.endswith("12288")) else None
    _check(_run_layer(wl, 0, rows=rows, want=("Y", "dX"), fmt="affine", bits=bits, G=G), TOL["bf16"])


@pytest.mark.parametrize("R", [1, 5, 16])
@pytest.mark.parametrize("bits,G", [(4, 32), (4, 128), (8, 64)])
def test_fp32_small_row_affine(R, bits, G):
    """fp32 compute mode with affine weights at 1..16 tokens on W 4096x4096:
    the CUDA-core forward GEMV and the input-gradient GEMV (8 adjacent
    columns per thread up to 4 tokens, 4 above; 16 row splits summed in
    order)."""
    wl = synth.workload("bw_sweep_4096", R=R)
    wl.compute = "fp32"
    _check(_run_layer(wl, 0, want=("Y", "dX"), fmt="affine", bits=bits, G=G), TOL["fp32"])


@pytest.mark.parametrize("R", [1, 16, 64, 4096])
def test_bf16_fp32scale_format(R):
    """The legacy fp32-scale format through every bf16 path: the few-token
    GEMV (1, 16), the tensor-core kernel with split-K (64) and without (4096)."""
    wl = synth.workload("qwen3_0.6b_attn_qv", R=R)
    _check(_run_layer(wl, 0, fmt="nf4_fp32scale"), TOL["bf16"])


def test_fp32_fp32scale_format():
    wl = synth.workload("fp32_single_256")
    _check(_run_layer(wl, 0, fmt="nf4_fp32scale"), TOL["fp32"])


def test_merge_fp32scale_format():
    """Export of a legacy-format weight: B = 0 gives the dequantized matrix."""
    W = synth.normal(77, (256, 512), std=0.02)
    gw = q.qlora_quantize_nf4_fp32scale(to_dev_f32(W), 64)
    A = torch.randn((8, 512), device="cuda")
    Bz = torch.zeros((256, 8), device="cuda")
    out = q.qlora_merge(gw, A, Bz, 16.0)
    ref = oracle.dequantize(oracle.quantize_nf4_legacy(W, 64))
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("name,li", [("8b_mlp", 0), ("8b_mlp", 2), ("14b_layer", 1), ("14b_layer", 6)])
def test_bf16_full_size_sampled_rows(name, li):
    wl = synth.workload(name)
    rows = synth.sample_rows(wl.R, 64, seed=wl.wid)
    _check(_run_layer(wl, li, rows=rows), TOL["bf16"])


# ------------------------------------------------------- failure detection

def test_bounded_wait_reports_timeout_and_context_survives():
    assert q.qlora_selftest_wait_timeout(limit_us=2000) == 7  # QLORA_ERR_TIMEOUT
    W = to_dev_f32(synth.normal(8, (128, 128), std=0.02))
    gw = q.qlora_quantize_nf4(W)
    assert gw.codes.numel() == 128 * 64


def test_workspace_status_clean_after_tensor_core_calls():
    wl = synth.workload("qwen3_0.6b_attn_qv", R=512)
    d = layer_inputs(wl, 0)
    gw = q.qlora_quantize_nf4(to_dev_f32(d["W"]))
    A, B = to_dev_f32(d["A"]), to_dev_f32(d["B"])
    ws = q.workspace(q.qlora_linear_workspace_bytes(gw, 512, 8, 0, 1))
    n0 = q.qlora_kernel_launch_count()
    q.qlora_linear_fwd(gw, d["xd"], A, B, 16.0, ws=ws)
    assert q.qlora_workspace_status(ws) == 0
    assert q.qlora_kernel_launch_count() > n0


def test_kernel_timing_inside_cuda_graph():
    wl = synth.workload("qwen3_0.6b_attn_qv", R=512)
    d = layer_inputs(wl, 0)
    gw = q.qlora_quantize_nf4(to_dev_f32(d["W"]))
    A, B = to_dev_f32(d["A"]), to_dev_f32(d["B"])
    Y = torch.empty((512, 2048), dtype=torch.bfloat16, device="cuda")
    U = torch.empty((512, 8), device="cuda")
    ws = q.workspace(q.qlora_linear_workspace_bytes(gw, 512, 8, 0, 1))
    q.qlora_linear_fwd(gw, d["xd"], A, B, 16.0, Y=Y, U_out=U, ws=ws)  # first call outside capture
    torch.cuda.synchronize()
    q.qlora_kernel_timing_enable(8)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
        q.qlora_linear_fwd(gw, d["xd"], A, B, 16.0, Y=Y, U_out=U, ws=ws)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        recs = q.qlora_kernel_timing_collect(8)
        assert len(recs) == 1 and recs[0][0] == 0 and recs[0][1] > 0 and recs[0][2] > 0
    del g
    q.qlora_kernel_timing_enable(0)
    oY, _ = oracle.linear_fwd(oracle.quantize_nf4(d["W"]), d["x"], d["A"], d["B"], 8, 16.0)
    assert rel_fro(to_host(Y), oY) <= TOL["bf16"]

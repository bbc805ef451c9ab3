"""GPT-345M-shaped workload: all 96 linears as calibrated W8A8 (alpha 0.5).

Inputs come from a random-init bf16 forward (synthetic/gpt.py) over 8 x 1024
uniform token ids.  Every linear runs the whole path on the GPU through the C
ABI (calibrate on its own input, smooth, SSZ int8, per-token quantization,
GEMM + dequant); the oracle checks each one: the calibration and weight
maxima in full (bit-exact), the smoothing factor, and sampled output
channels / tokens for scales, codes and outputs.  A model-level forward with
every linear replaced reports the W8A8 error against the bf16 model.
"""
import numpy as np
import pytest
import torch

from tests.conftest import build_cuda_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    build_cuda_library()
    import w8a8_linear_layers_b200 as mod
    return mod


@pytest.fixture(scope="module")
def model():
    from synthetic import gpt
    weights, cap = gpt.linear_inputs(seed=0, device="cuda")
    return gpt, weights, cap


def _path(w, x, wt, alpha=0.5):
    M, K = x.shape
    N = wt.shape[0]
    d = dict(device="cuda")
    ax, aw, s, inv = (torch.empty(K, **d) for _ in range(4))
    qw = torch.empty(N, K, dtype=torch.int8, **d)
    sw = torch.empty(N, **d)
    qx = torch.empty(M, K, dtype=torch.int8, **d)
    sx = torch.empty(M, **d)
    y = torch.empty(M, N, dtype=torch.bfloat16, **d)
    w.sq_calib_absmax(x, ax)
    w.sq_smooth_fold(ax, wt, alpha, aw, s, inv)
    w.ssz_quant_weight(wt, s, 8, 20, qw, sw)
    w.quant_act_per_token(x, inv, qx, sx)
    w.w8a8_gemm_dequant(qx, sx, qw, sw, y)
    return dict(ax=ax, aw=aw, s=s, inv=inv, qw=qw, sw=sw, qx=qx, sx=sx, y=y)


def test_all_96_linears_against_oracle(w, orc, model):
    gpt, weights, cap = model
    assert len(cap) == 96
    rng = np.random.default_rng(0)
    worst = 0.0
    for (layer, name), x in sorted(cap.items()):
        wt = weights[(layer, name)]
        got = _path(w, x, wt)
        xf = x.float().cpu().numpy()
        wf = wt.float().cpu().numpy()
        ax = orc.calib_absmax(xf)
        np.testing.assert_array_equal(got["ax"].cpu().numpy(), ax)
        aw = orc.weight_col_absmax(wf)
        np.testing.assert_array_equal(got["aw"].cpu().numpy(), aw)
        s, inv_s = orc.smooth_factor(ax, aw, 0.5)
        np.testing.assert_allclose(got["s"].cpu().numpy(), s, rtol=1e-5, atol=0)
        rn = np.sort(rng.choice(wf.shape[0], 64, replace=False))
        rm = np.sort(rng.choice(xf.shape[0], 32, replace=False))
        wq = orc.ssz_quant_weight(wf[rn], bits=8, s=s)
        np.testing.assert_allclose(got["sw"].cpu().numpy()[rn], wq["scale"], rtol=1e-5, atol=0)
        assert np.mean(got["qw"].cpu().numpy()[rn] != wq["q"]) < 1e-5
        qx, sx = orc.quant_act_per_token(xf[rm], inv_s)
        np.testing.assert_allclose(got["sx"].cpu().numpy()[rm], sx, rtol=1e-5, atol=0)
        assert np.mean(got["qx"].cpu().numpy()[rm] != qx) < 1e-5
        y_ref = orc.bf16_bits_to_f32(orc.dequant(orc.gemm_i8(qx, wq["q"]), sx, wq["scale"]))
        y = got["y"].float().cpu().numpy()[np.ix_(rm, rn)]
        np.testing.assert_allclose(y, y_ref, rtol=1e-3, atol=1e-5)
        ref = (x[rm].float() @ wt[rn].float().t()).cpu().numpy()
        worst = max(worst, float(np.linalg.norm(y - ref) / np.linalg.norm(ref)))
    assert worst < 0.05, worst  # W8A8 vs the unquantized product, informational bound


def test_model_forward_with_w8a8_linears(w, model):
    gpt, weights, cap = model
    # calibrate each linear on the bf16 model's activations, then run the model
    # with every linear replaced by the quantized path
    layers = {}
    for key, x in cap.items():
        lin = w.W8A8Linear(weights[key], alpha=0.5)
        lin.calibrate(x)
        lin.quantize()
        layers[key] = lin
    toks = gpt.make_tokens(0)
    ref = gpt.forward(weights, toks).float()
    out = gpt.forward(weights, toks, linear=lambda layer, name, a, W: layers[(layer, name)].forward(a)).float()
    assert torch.isfinite(out).all()
    rel = (torch.linalg.norm(out - ref) / torch.linalg.norm(ref)).item()
    cos = torch.nn.functional.cosine_similarity(out.flatten(), ref.flatten(), dim=0).item()
    print("GPT-345M-shaped W8A8 forward: relative error %.4f, cosine %.5f" % (rel, cos))
    assert cos > 0.99

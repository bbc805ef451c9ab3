"""W8A8Linear with the next-row options: each configuration's forward equals
the explicit chain of library calls it stands for (bit for bit), and the
static-scale row sums equal the oracle's row sums of the same codes."""
import numpy as np
import pytest
import torch

import synthetic
from tests.test_parity_gpu import np32, w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


def _setup(M=96, K=512, N=384, seed=4):
    x, wt = synthetic.make_small(M, K, N, seed=seed)
    return x.cuda(), wt.cuda()


@pytest.mark.parametrize("weights", ["asym8", "int4"])
def test_module_weights_match_calls(w, weights):
    x, wt = _setup()
    lin = w.W8A8Linear(wt, alpha=0.5, weights=weights)
    lin.calibrate(x)
    lin.quantize()
    y = lin.forward(x)
    M, K = x.shape
    N = wt.shape[0]
    ax, aw, s, inv = (torch.empty(K, device="cuda") for _ in range(4))
    w.sq_calib_absmax(x, ax)
    w.sq_smooth_fold(ax, wt, 0.5, aw, s, inv)
    qw = torch.empty(N, K, dtype=torch.int8, device="cuda")
    sw = torch.empty(N, device="cuda")
    qx = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    yr = torch.empty_like(y)
    if weights == "asym8":
        ow = torch.empty(N, device="cuda")
        rs = torch.empty(M, dtype=torch.int32, device="cuda")
        w.ssz_quant_weight_asym(wt, s, 20, qw, sw, ow)
        w.quant_act_per_token_rowsum(x, inv, qx, sx, rs)
        w.w8a8_gemm_dequant_asym(qx, sx, rs, qw, sw, ow, yr)
    else:
        p = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
        w.ssz_quant_weight(wt, s, 4, 20, qw, sw)
        w.sq_pack_int4(qw, p)
        w.quant_act_per_token(x, inv, qx, sx)
        w.w4a8_gemm_dequant(qx, sx, p, sw, yr)
    assert torch.equal(y.view(torch.int16) if y.dtype == torch.bfloat16 else y,
                       yr.view(torch.int16) if yr.dtype == torch.bfloat16 else yr)


@pytest.mark.parametrize("weights", ["sym8", "asym8"])
def test_module_static_scales_match_calls(w, orc, weights):
    x, wt = _setup(seed=5)
    lin = w.W8A8Linear(wt, alpha=0.5, weights=weights, act_scales="static")
    lin.calibrate(x)
    lin.quantize()
    batches = [x[i * 32:(i + 1) * 32].contiguous() for i in range(3)]
    for b in batches:
        lin.calibrate_static(b)
    with pytest.raises(RuntimeError):
        w.W8A8Linear(wt, act_scales="static").forward(x)
    y = lin.forward(x)
    M, K = x.shape
    rng = torch.empty(1, device="cuda")
    axb = torch.empty(K, device="cuda")
    for i, b in enumerate(batches):
        w.sq_calib_absmax(b, axb)
        w.sq_static_range_update(axb, lin.inv_s, rng, first=(i == 0))
    assert torch.equal(rng, lin.range)
    qx = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    rs = torch.empty(M, dtype=torch.int32, device="cuda")
    w.quant_act_static(x, lin.inv_s, rng, qx, sx, rs)
    np.testing.assert_array_equal(rs.cpu().numpy(), orc.act_rowsum(qx.cpu().numpy()))
    yr = torch.empty_like(y)
    if weights == "asym8":
        w.w8a8_gemm_dequant_asym(qx, sx, rs, lin.qw, lin.sw, lin.ow, yr)
    else:
        w.w8a8_gemm_dequant(qx, sx, lin.qw, lin.sw, yr)
    assert torch.equal(y.float(), yr.float())


def test_module_forward_ln_matches_calls(w):
    x, wt = _setup(seed=6)
    K = x.shape[1]
    g = torch.rand(K, device="cuda") + 0.5
    b = torch.randn(K, device="cuda") * 0.1
    lin = w.W8A8Linear(wt, alpha=0.5)
    lin.calibrate(torch.nn.functional.layer_norm(x.float(), (K,), g, b).to(x.dtype))
    lin.quantize()
    y = lin.forward_ln(x, g, b, 1e-5)
    qx = torch.empty(x.shape, dtype=torch.int8, device="cuda")
    sx = torch.empty(x.shape[0], device="cuda")
    w.sq_layernorm_quant(x, g, b, 1e-5, lin.inv_s, qx, sx)
    yr = torch.empty_like(y)
    w.w8a8_gemm_dequant(qx, sx, lin.qw, lin.sw, yr)
    assert torch.equal(y.float(), yr.float())
    with pytest.raises(ValueError):
        w.W8A8Linear(wt, weights="asym8").forward_ln(x, g, b)


@pytest.mark.parametrize("weights,act", [("sym8", "dynamic"), ("int4", "dynamic"), ("asym8", "static")])
def test_graphed_forward_equals_eager(w, weights, act):
    x, wt = _setup(seed=7)
    lin = w.W8A8Linear(wt, alpha=0.5, weights=weights, act_scales=act)
    lin.calibrate(x)
    lin.quantize()
    if act == "static":
        lin.calibrate_static(x)
    g = lin.graphed(16)
    for seed in (1, 2):
        xi, _ = synthetic.make_small(16, x.shape[1], 8, seed=seed)
        g.x.copy_(xi.cuda())
        yg = g.replay().clone()
        ye = lin.forward(xi.cuda())
        assert torch.equal(yg.float(), ye.float())

"""GPU parity of the static activation scale path against the CPU oracle.

A per-tensor activation range calibrated offline as a moving average of each
batch's abs-max ("PaddleNLP GPT 量化感知训练（QAT）实战指南" section 六,
moving_average_abs_max; CUDA INT8 notes section 2.1 for range calibration and
saturation), then codes at the fixed scale S = range / 127.  Oracle inputs
come from the oracle or from the seeded generators, never from the GPU; the
range (a max and fp32 blends) and the codes must match bit for bit, the
linear's output within 1e-3 relative + 1e-5 absolute.
"""
import numpy as np
import pytest
import torch

import synthetic
from tests.test_parity_gpu import Guarded, make_x, np32, w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


def _inv_s(orc, xs, wt, alpha):
    ax = orc.calib_absmax(np.concatenate([np32(x) for x in xs]))
    _, inv = orc.smooth_factor(ax, orc.weight_col_absmax(np32(wt)), alpha)
    return inv


@pytest.mark.parametrize("K,rate,smooth", [(16, 0.9, False), (1040, 0.9, True), (4096, 0.9, True),
                                           (4096, 0.0, True), (4096, 1.0, True), (8192, 0.5, False)])
def test_static_range_bit_exact(w, orc, K, rate, smooth):
    batches = [make_x(64 + 17 * i, K, torch.bfloat16, seed=100 + i, scale=30.0 + 10 * i) for i in range(5)]
    inv = _inv_s(orc, batches, make_x(32, K, torch.bfloat16, seed=99, outliers=0) * 0.02, 0.5) if smooth else None
    inv_d = None if inv is None else torch.from_numpy(inv).cuda()
    rng = Guarded((1,), torch.float32)
    ax = torch.empty(K, device="cuda")
    for i, xb in enumerate(batches):
        w.sq_calib_absmax(xb.cuda(), ax)
        w.sq_static_range_update(ax, inv_d, rng.t, first=(i == 0), rate=rate)
    want = orc.static_range([np32(x) for x in batches], inv, rate=rate)
    assert rng.t.item() == float(want)
    assert rng.intact()


@pytest.mark.parametrize("M,K,dtype,frac", [
    (1, 16, torch.float32, 1.0), (7, 48, torch.bfloat16, 0.3), (300, 528, torch.bfloat16, 0.5),
    (129, 1040, torch.float32, 0.25), (2048, 4096, torch.bfloat16, 0.7), (33, 8192, torch.bfloat16, 1.2),
    (5, 32768, torch.float32, 0.5),
])
def test_quant_act_static_bit_exact(w, orc, M, K, dtype, frac):
    x = make_x(M, K, dtype, seed=M + K)
    inv = (np.random.default_rng(K).random(K) + 0.5).astype(np.float32)
    xs = np32(x) * inv[None, :]
    m = np.float32(np.abs(xs).max() * np.float32(frac))  # frac < 1: the top values saturate
    q = Guarded((M, K), torch.int8)
    sc = Guarded((M,), torch.float32)
    rng = torch.tensor([m], device="cuda")
    w.quant_act_static(x.cuda(), torch.from_numpy(inv).cuda(), rng, q.t, sc.t)
    np.testing.assert_array_equal(q.t.cpu().numpy(), orc.quant_act_static(np32(x), inv, m))
    assert np.all(sc.t.cpu().numpy() == orc.static_scale(m))
    assert q.intact() and sc.intact()


def test_quant_act_static_zero_range_and_no_scale_out(w, orc):
    x = make_x(9, 64, torch.bfloat16, seed=5)
    q = torch.full((9, 64), 7, dtype=torch.int8, device="cuda")
    w.quant_act_static(x.cuda(), None, torch.zeros(1, device="cuda"), q)
    assert not q.any()
    m = np.float32(3.0)
    w.quant_act_static(x.cuda(), None, torch.tensor([m], device="cuda"), q)
    np.testing.assert_array_equal(q.cpu().numpy(), orc.quant_act_static(np32(x), None, m))


@pytest.mark.parametrize("name", ["single_linear_16x256x128", "prefill_2048x4096x4096"])
def test_static_linear_end_to_end(w, orc, name):
    """Calibrate the range on 4 batches, quantize a fifth at the static scale,
    GEMM + dequant; the same chain in the oracle.  Reports the output error of
    the static and the per-token path against the unquantized product."""
    cfg = synthetic.CONFIGS[name]
    M = min(cfg.M, 512)
    # one draw (one set of outlier channels, as in a real model), split into
    # four calibration batches and the batch that is then quantized
    x_all, wt = synthetic.make_linear(cfg, seed=0, M=5 * M)
    calib = [x_all[i * M:(i + 1) * M].contiguous() for i in range(4)]
    x = x_all[4 * M:].contiguous()
    N, K = wt.shape
    dev = dict(device="cuda")
    # GPU chain: smoothing from the running calibration absmax over all batches
    ax, aw, s, inv = (torch.empty(K, **dev) for _ in range(4))
    for i, xb in enumerate(calib):
        w.sq_calib_absmax(xb.cuda(), ax, accumulate=(i > 0))
    w.sq_smooth_fold(ax, wt.cuda(), cfg.alpha, aw, s, inv)
    qw = torch.empty(N, K, dtype=torch.int8, **dev)
    sw = torch.empty(N, **dev)
    w.ssz_quant_weight(wt.cuda(), s, cfg.bits, cfg.max_iters, qw, sw)
    rng = torch.empty(1, **dev)
    axb = torch.empty(K, **dev)
    for i, xb in enumerate(calib):
        w.sq_calib_absmax(xb.cuda(), axb)
        w.sq_static_range_update(axb, inv, rng, first=(i == 0))
    qx = torch.empty(M, K, dtype=torch.int8, **dev)
    sx = torch.empty(M, **dev)
    w.quant_act_static(x.cuda(), inv, rng, qx, sx)
    ydt = torch.bfloat16 if cfg.out_dtype == "bf16" else torch.float32
    y = torch.empty(M, N, dtype=ydt, **dev)
    w.w8a8_gemm_dequant(qx, sx, qw, sw, y)
    # oracle chain (sampled output channels and tokens: the oracle is slow at full size)
    rows_n = np.sort(np.random.default_rng(1).choice(N, min(N, 256), replace=False))
    rows_m = np.sort(np.random.default_rng(2).choice(M, min(M, 64), replace=False))
    xs_np = [np32(b) for b in calib]
    ax_o = orc.calib_absmax(np.concatenate(xs_np))
    s_o, inv_o = orc.smooth_factor(ax_o, orc.weight_col_absmax(np32(wt)), cfg.alpha)
    np.testing.assert_allclose(inv.cpu().numpy(), inv_o, rtol=1e-5, atol=0)
    m_o = orc.static_range(xs_np, inv_o)
    assert abs(rng.item() - float(m_o)) <= 1e-5 * float(m_o)
    wq = orc.ssz_quant_weight(np32(wt)[rows_n], bits=cfg.bits, max_iters=cfg.max_iters, s=s_o)
    np.testing.assert_allclose(sw.cpu().numpy()[rows_n], wq["scale"], rtol=1e-5, atol=0)
    assert np.mean(qw.cpu().numpy()[rows_n] != wq["q"]) < 1e-5
    qx_o = orc.quant_act_static(np32(x)[rows_m], inv_o, m_o)
    assert np.mean(qx.cpu().numpy()[rows_m] != qx_o) < 1e-5
    S = orc.static_scale(m_o)
    y_o = orc.dequant(orc.gemm_i8(qx_o, wq["q"]), np.full(len(rows_m), S, np.float32), wq["scale"], out="f32")
    if ydt == torch.bfloat16:
        y_o = orc.bf16_bits_to_f32(orc.to_bf16_bits(y_o))
    yg = y.float().cpu().numpy()
    np.testing.assert_allclose(yg[np.ix_(rows_m, rows_n)], y_o, rtol=1e-3, atol=1e-5)
    # informational: static vs per-token error against the unquantized product
    ref = np32(x).astype(np.float64) @ np32(wt).astype(np.float64).T
    qd = torch.empty_like(qx)
    sd = torch.empty_like(sx)
    w.quant_act_per_token(x.cuda(), inv, qd, sd)
    yd = torch.empty_like(y)
    w.w8a8_gemm_dequant(qd, sd, qw, sw, yd)
    e_s = np.linalg.norm(yg - ref) / np.linalg.norm(ref)
    e_d = np.linalg.norm(yd.float().cpu().numpy() - ref) / np.linalg.norm(ref)
    print("%s: relative error static %.4g, per-token %.4g" % (name, e_s, e_d))
    assert e_s < 0.2 and e_d < 0.2

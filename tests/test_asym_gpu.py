"""GPU parity of the asymmetric int8 path against the CPU oracle.

"SSZ：权重量化算法说明" 迭代优化阶段 (asymmetric: scale and offset by least
squares) with MinMax min/max init; the dequant of CUDA INT8 notes sections
2.1 / 4.2 with the zero point carried as a weight-domain offset.  Oracle
inputs come from the oracle or the seeded generators, never from the GPU.
MinMax codes and every integer result (codes, row sums, accumulators) and the
dequant given its inputs must match bit for bit; searched scales and offsets
within 1e-5 relative; the weight codes bit for bit given the GPU's own
(scale, offset); outputs within 1e-3 relative + 1e-5 absolute.
"""
import numpy as np
import pytest
import torch

import synthetic
from tests.test_parity_gpu import Guarded, make_x, np32, w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


def _weights(N, K, dtype, seed, shift=0.0):
    g = torch.Generator().manual_seed(seed)
    wt = torch.randn(N, K, generator=g) * 0.02 + shift
    wt[:, torch.randperm(K, generator=g)[:3]] *= 8.0
    return wt.to(dtype)


@pytest.mark.parametrize("N,K,dtype,smooth,shift", [
    (1, 16, torch.float32, False, 0.0), (7, 48, torch.bfloat16, False, 0.01), (33, 1040, torch.bfloat16, True, 0.0),
    (64, 4096, torch.bfloat16, True, 0.005), (300, 528, torch.float32, True, -0.01), (8, 32768, torch.float32, False, 0.0),
])
def test_ssz_asym_parity(w, orc, N, K, dtype, smooth, shift):
    wt = _weights(N, K, dtype, seed=N + K, shift=shift)
    s = None
    if smooth:
        ax = np.abs(np.random.default_rng(K).standard_normal(K)).astype(np.float32) * 5 + 0.1
        s, _ = orc.smooth_factor(ax, orc.weight_col_absmax(np32(wt)), 0.5)
    q = Guarded((N, K), torch.int8)
    sc, off = Guarded((N,), torch.float32), Guarded((N,), torch.float32)
    mse = torch.empty(N, dtype=torch.float64, device="cuda")
    its = torch.empty(N, dtype=torch.int32, device="cuda")
    w.ssz_quant_weight_asym(wt.cuda(), None if s is None else torch.from_numpy(s).cuda(), 20, q.t, sc.t, off.t,
                            mse, its)
    ref = orc.ssz_quant_weight_asym(np32(wt), s=s)
    wf = np32(wt) if s is None else orc.scale_columns(np32(wt), s)
    S, m = sc.t.cpu().numpy(), off.t.cpu().numpy()
    np.testing.assert_allclose(S, ref["scale"], rtol=1e-5, atol=0)
    np.testing.assert_allclose(m, ref["offset"], rtol=1e-5, atol=1e-6 * np.abs(wf).max())
    # codes bit-exact given the GPU's (scale, offset)
    np.testing.assert_array_equal(q.t.cpu().numpy(), orc.weight_codes_asym(wf, S, m))
    # the reported error is the error at the returned (scale, offset)
    mse_ref = np.array([orc.channel_mse_asym(wf[n], S[n], m[n]) for n in range(N)])
    np.testing.assert_allclose(mse.cpu().numpy(), mse_ref, rtol=1e-9, atol=1e-300)
    np.testing.assert_allclose(mse.cpu().numpy(), ref["mse"], rtol=1e-6, atol=0)
    # rounds taken: equal wherever the search took the same path (a decision
    # at a rounding tie of the fp64 error may end a channel one round apart)
    assert np.mean(its.cpu().numpy() == ref["iters"]) > 0.99
    assert q.intact() and sc.intact() and off.intact()


def test_ssz_asym_minmax_is_bit_exact(w, orc):
    wt = _weights(40, 1024, torch.bfloat16, seed=3, shift=0.02)
    q = torch.empty(40, 1024, dtype=torch.int8, device="cuda")
    sc, off = torch.empty(40, device="cuda"), torch.empty(40, device="cuda")
    w.ssz_quant_weight_asym(wt.cuda(), None, 0, q, sc, off)
    ref = orc.ssz_quant_weight_asym(np32(wt), max_iters=0)
    np.testing.assert_array_equal(sc.cpu().numpy(), ref["scale"])
    np.testing.assert_array_equal(off.cpu().numpy(), ref["offset"])
    np.testing.assert_array_equal(q.cpu().numpy(), ref["q"])


@pytest.mark.parametrize("M,K,dtype", [(1, 16, torch.float32), (300, 528, torch.bfloat16),
                                       (2048, 4096, torch.bfloat16), (33, 8192, torch.bfloat16)])
def test_quant_rowsum_bit_exact(w, orc, M, K, dtype):
    x = make_x(M, K, dtype, seed=M + 7)
    inv = (np.random.default_rng(K).random(K) + 0.5).astype(np.float32)
    q = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    R = Guarded((M,), torch.int32)
    w.quant_act_per_token_rowsum(x.cuda(), torch.from_numpy(inv).cuda(), q, sx, R.t)
    qo, sxo = orc.quant_act_per_token(np32(x), inv)
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(R.t.cpu().numpy(), orc.act_rowsum(qo))
    assert R.intact()


@pytest.mark.parametrize("M,N,K,ydt", [
    (1, 8, 16, torch.bfloat16), (77, 264, 272, torch.float32), (128, 512, 1024, torch.bfloat16),
    (300, 520, 4096, torch.bfloat16), (1000, 1032, 2064, torch.float32),
    (128, 520, 4096, torch.bfloat16), (90, 264, 2080, torch.float32),  # 128-token decode tiles
])
def test_gemm_asym_bit_exact(w, orc, M, N, K, ydt):
    r = np.random.default_rng(M * N + K)
    qx = r.integers(-127, 128, (M, K)).astype(np.int8)
    qw = r.integers(-128, 128, (N, K)).astype(np.int8)
    sx = (r.random(M) * 0.05 + 1e-3).astype(np.float32)
    sw = (r.random(N) * 1e-3 + 1e-5).astype(np.float32)
    ow = (r.standard_normal(N) * 0.05).astype(np.float32)
    R = orc.act_rowsum(qx)
    y = Guarded((M, N), ydt)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    d = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    w.w8a8_gemm_dequant_asym(d(qx), d(sx), d(R), d(qw), d(sw), d(ow), y.t, acc)
    acc_o = orc.gemm_i8(qx, qw)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    if ydt == torch.bfloat16:
        yb = y.t.cpu().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(yb, orc.dequant_asym(acc_o, R, sx, sw, ow))
    else:
        np.testing.assert_array_equal(y.t.cpu().numpy(), orc.dequant_asym(acc_o, R, sx, sw, ow, out="f32"))
    assert y.intact()
    # without acc_out (M > 128: the output staged in shared memory and stored by TMA) the output is the same
    y2 = Guarded((M, N), ydt)
    w.w8a8_gemm_dequant_asym(d(qx), d(sx), d(R), d(qw), d(sw), d(ow), y2.t)
    assert torch.equal(y2.t, y.t) and y2.intact()


@pytest.mark.parametrize("name", ["single_linear_16x256x128", "prefill_2048x4096x4096"])
def test_asym_linear_end_to_end(w, orc, name):
    """Whole path with asymmetric weights on the GPU; the oracle checks
    sampled channels and tokens.  Reports the output error of the asymmetric
    and the symmetric weight path against the unquantized product."""
    cfg = synthetic.CONFIGS[name]
    x, wt = synthetic.make_linear(cfg, seed=0)
    M, K = x.shape
    N = wt.shape[0]
    dev = dict(device="cuda")
    ax, aw, s, inv = (torch.empty(K, **dev) for _ in range(4))
    w.sq_calib_absmax(x.cuda(), ax)
    w.sq_smooth_fold(ax, wt.cuda(), cfg.alpha, aw, s, inv)
    qw = torch.empty(N, K, dtype=torch.int8, **dev)
    sw, ow = torch.empty(N, **dev), torch.empty(N, **dev)
    w.ssz_quant_weight_asym(wt.cuda(), s, cfg.max_iters, qw, sw, ow)
    qx = torch.empty(M, K, dtype=torch.int8, **dev)
    sx = torch.empty(M, **dev)
    R = torch.empty(M, dtype=torch.int32, **dev)
    w.quant_act_per_token_rowsum(x.cuda(), inv, qx, sx, R)
    ydt = torch.bfloat16 if cfg.out_dtype == "bf16" else torch.float32
    y = torch.empty(M, N, dtype=ydt, **dev)
    w.w8a8_gemm_dequant_asym(qx, sx, R, qw, sw, ow, y)
    # oracle on sampled channels / tokens
    rows_n = np.sort(np.random.default_rng(1).choice(N, min(N, 256), replace=False))
    rows_m = np.sort(np.random.default_rng(2).choice(M, min(M, 64), replace=False))
    xf, wf = np32(x), np32(wt)
    ax_o = orc.calib_absmax(xf)
    s_o, inv_o = orc.smooth_factor(ax_o, orc.weight_col_absmax(wf), cfg.alpha)
    wq = orc.ssz_quant_weight_asym(wf[rows_n], max_iters=cfg.max_iters, s=s_o)
    np.testing.assert_allclose(sw.cpu().numpy()[rows_n], wq["scale"], rtol=1e-5, atol=0)
    wfo = orc.scale_columns(wf[rows_n], s_o)
    np.testing.assert_allclose(ow.cpu().numpy()[rows_n], wq["offset"], rtol=1e-5, atol=1e-6 * np.abs(wfo).max())
    np.testing.assert_array_equal(qw.cpu().numpy()[rows_n],
                                  orc.weight_codes_asym(wfo, sw.cpu().numpy()[rows_n], ow.cpu().numpy()[rows_n]))
    qx_o, sx_o = orc.quant_act_per_token(xf[rows_m], inv_o)
    assert np.mean(qx.cpu().numpy()[rows_m] != qx_o) < 1e-5
    R_o = orc.act_rowsum(qx_o)
    y_o = orc.dequant_asym(orc.gemm_i8(qx_o, wq["q"]), R_o, sx_o, wq["scale"], wq["offset"], out="f32")
    if ydt == torch.bfloat16:
        y_o = orc.bf16_bits_to_f32(orc.to_bf16_bits(y_o))
    yg = y.float().cpu().numpy()
    np.testing.assert_allclose(yg[np.ix_(rows_m, rows_n)], y_o, rtol=1e-3, atol=1e-5)
    # informational: asymmetric vs symmetric weights, against the unquantized product
    ref = xf[rows_m].astype(np.float64) @ wf.astype(np.float64).T
    qs = torch.empty_like(qw)
    ss = torch.empty_like(sw)
    w.ssz_quant_weight(wt.cuda(), s, 8, cfg.max_iters, qs, ss)
    ys = torch.empty_like(y)
    w.w8a8_gemm_dequant(qx, sx, qs, ss, ys)
    e_a = np.linalg.norm(yg[rows_m] - ref) / np.linalg.norm(ref)
    e_s = np.linalg.norm(ys.float().cpu().numpy()[rows_m] - ref) / np.linalg.norm(ref)
    print("%s: relative error asymmetric %.4g, symmetric %.4g" % (name, e_a, e_s))
    assert e_a < 0.1 and e_s < 0.1

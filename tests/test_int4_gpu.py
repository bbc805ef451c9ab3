"""GPU parity of the packed int4 weight path against the CPU oracle.

int4 per-channel symmetric SSZ codes ("SSZ：权重量化算法说明", 使用限制: int8
and int4 per_channel symmetric) packed two per byte, and the W4A8 GEMM that
unpacks them on chip.  Packing, accumulators and the dequantized output must
match the oracle bit for bit (the output given the codes and scales);
the whole int4 decode path within 1e-3 relative + 1e-5 absolute.
"""
import numpy as np
import pytest
import torch

import synthetic
from tests.test_parity_gpu import Guarded, make_x, np32, w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(1, 32), (7, 96), (300, 1056), (64, 8192)])
def test_pack_int4_bit_exact(w, orc, N, K):
    q = np.random.default_rng(N + K).integers(-8, 8, (N, K)).astype(np.int8)
    p = Guarded((N, K // 2), torch.uint8)
    w.sq_pack_int4(torch.from_numpy(q).cuda(), p.t)
    np.testing.assert_array_equal(p.t.cpu().numpy(), orc.pack_int4(q))
    assert p.intact()


@pytest.mark.parametrize("M,N,K,ydt", [
    (1, 8, 32, torch.bfloat16), (16, 264, 288, torch.float32), (77, 512, 1024, torch.bfloat16),
    (128, 1032, 2080, torch.float32), (300, 520, 4096, torch.bfloat16), (16, 2048, 8192, torch.bfloat16),
])
def test_w4a8_gemm_bit_exact(w, orc, M, N, K, ydt):
    r = np.random.default_rng(M * N + K)
    qx = r.integers(-127, 128, (M, K)).astype(np.int8)
    q4 = r.integers(-7, 8, (N, K)).astype(np.int8)
    q4[0, :] = -8  # the int4 extreme
    sx = (r.random(M) * 0.05 + 1e-3).astype(np.float32)
    sw = (r.random(N) * 1e-2 + 1e-5).astype(np.float32)
    d = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    p = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    w.sq_pack_int4(d(q4), p)
    y = Guarded((M, N), ydt)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    w.w4a8_gemm_dequant(d(qx), d(sx), p, d(sw), y.t, acc)
    acc_o = orc.gemm_i8(qx, orc.unpack_int4(orc.pack_int4(q4), K))
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    if ydt == torch.bfloat16:
        np.testing.assert_array_equal(y.t.cpu().view(torch.int16).numpy().view(np.uint16),
                                      orc.dequant(acc_o, sx, sw))
    else:
        np.testing.assert_array_equal(y.t.cpu().numpy(), orc.dequant(acc_o, sx, sw, out="f32"))
    assert y.intact()


# the decode kernel and the W4A8 kernel; K = 131040 is the largest the call
# accepts (16 * 128 * 8 * K just below 2^31) and ends in a partial k-block
@pytest.mark.parametrize("M,N,K", [(16, 256, 16384), (300, 256, 16384), (16, 16, 131040), (130, 16, 131040)])
def test_w4a8_extreme_accumulators(w, orc, M, N, K):
    """Largest |acc| the signed operands allow: a row of qx at -128 against
    codes at -8 (and at 7); acc exact, signs kept."""
    r = np.random.default_rng(M)
    qx = r.integers(-127, 128, (M, K)).astype(np.int8)
    qx[0, :] = -128
    qx[1, :] = 127
    q4 = r.integers(-8, 8, (N, K)).astype(np.int8)
    q4[0, :] = -8
    q4[1, :] = 7
    sx = np.full(M, 1e-6, np.float32)
    sw = np.full(N, 1e-3, np.float32)
    d = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    p = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    w.sq_pack_int4(d(q4), p)
    y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    w.w4a8_gemm_dequant(d(qx), d(sx), p, d(sw), y, acc)
    acc_o = orc.gemm_i8(qx, q4)
    assert acc_o[0, 0] == 128 * 8 * K and acc_o[1, 1] == 127 * 7 * K and acc_o[0, 1] == -128 * 7 * K
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    np.testing.assert_array_equal(y.cpu().numpy(), orc.dequant(acc_o, sx, sw, out="f32"))


def test_w4a8_equals_w8a8_on_the_same_codes(w):
    r = np.random.default_rng(7)
    M, N, K = 200, 1024, 4096
    qx = torch.from_numpy(r.integers(-127, 128, (M, K)).astype(np.int8)).cuda()
    q4 = torch.from_numpy(r.integers(-7, 8, (N, K)).astype(np.int8)).cuda()
    sx = torch.rand(M, device="cuda") * 0.01
    sw = torch.rand(N, device="cuda") * 0.01
    p = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    w.sq_pack_int4(q4, p)
    y4 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y8 = torch.empty_like(y4)
    w.w4a8_gemm_dequant(qx, sx, p, sw, y4)
    w.w8a8_gemm_dequant(qx, sx, q4, sw, y8)
    assert torch.equal(y4.view(torch.int16), y8.view(torch.int16))


def test_int4_decode_path_end_to_end(w, orc):
    """The decode workload with int4 weights: SSZ int4, pack, per-token
    activation codes, W4A8 GEMM; the oracle checks sampled channels."""
    cfg = synthetic.CONFIGS["decode_16x8192x28672"]
    assert cfg.bits == 4
    x, wt = synthetic.make_linear(cfg, seed=0)
    M, K = x.shape
    N = wt.shape[0]
    dev = dict(device="cuda")
    ax, aw, s, inv = (torch.empty(K, **dev) for _ in range(4))
    w.sq_calib_absmax(x.cuda(), ax)
    w.sq_smooth_fold(ax, wt.cuda(), cfg.alpha, aw, s, inv)
    q4 = torch.empty(N, K, dtype=torch.int8, **dev)
    sw = torch.empty(N, **dev)
    w.ssz_quant_weight(wt.cuda(), s, 4, cfg.max_iters, q4, sw)
    p = torch.empty(N, K // 2, dtype=torch.uint8, **dev)
    w.sq_pack_int4(q4, p)
    qx = torch.empty(M, K, dtype=torch.int8, **dev)
    sx = torch.empty(M, **dev)
    w.quant_act_per_token(x.cuda(), inv, qx, sx)
    y = torch.empty(M, N, dtype=torch.bfloat16, **dev)
    w.w4a8_gemm_dequant(qx, sx, p, sw, y)
    rows_n = np.sort(np.random.default_rng(1).choice(N, 256, replace=False))
    xf, wf = np32(x), np32(wt)
    ax_o = orc.calib_absmax(xf)
    s_o, inv_o = orc.smooth_factor(ax_o, orc.weight_col_absmax(wf), cfg.alpha)
    wq = orc.ssz_quant_weight(wf[rows_n], bits=4, max_iters=cfg.max_iters, s=s_o)
    np.testing.assert_allclose(sw.cpu().numpy()[rows_n], wq["scale"], rtol=1e-5, atol=0)
    assert np.mean(q4.cpu().numpy()[rows_n] != wq["q"]) < 1e-5
    np.testing.assert_array_equal(p.cpu().numpy()[rows_n], orc.pack_int4(q4.cpu().numpy()[rows_n]))
    qx_o, sx_o = orc.quant_act_per_token(xf, inv_o)
    assert np.mean(qx.cpu().numpy() != qx_o) < 1e-5
    y_o = orc.dequant(orc.gemm_i8(qx_o, wq["q"]), sx_o, wq["scale"], out="f32")
    y_o = orc.bf16_bits_to_f32(orc.to_bf16_bits(y_o))
    np.testing.assert_allclose(y.float().cpu().numpy()[:, rows_n], y_o, rtol=1e-3, atol=1e-5)

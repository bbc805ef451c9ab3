"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Stage-wise, every kernel is fed inputs and the oracle recomputes the stage
from the same inputs.  Integer results (codes, int32 accumulators) and exact
floating-point results (maxima, the dequant given acc/sx/sw) must match bit
for bit; smoothing factors and SSZ scales within 1e-5 relative; bf16/fp32
outputs within 1e-3 relative + 1e-5 absolute.  End to end, the whole path runs
from raw seeded inputs at every workload's full size, and the oracle checks
the same sampled rows/columns.  Output buffers carry guard bytes that must
survive every call.
"""
import os

import numpy as np
import pytest
import torch

import synthetic
from tests.conftest import build_cuda_library

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def w():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    build_cuda_library()
    import w8a8_linear_layers_b200 as mod
    assert mod.device_fault() == 0
    yield mod
    torch.cuda.synchronize()
    assert mod.device_fault() == 0


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


class Guarded:
    """A device tensor with 512 guard bytes on each side filled with 0xA5."""

    PAD = 512

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) if len(shape) else 1
        item = torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((n * item + 2 * self.PAD,), 0xA5, dtype=torch.uint8, device="cuda")
        self.t = self.raw[self.PAD:self.PAD + n * item].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.raw[:self.PAD] == 0xA5).all() and (self.raw[-self.PAD:] == 0xA5).all())


def make_x(M, K, dtype, seed=0, outliers=2, scale=40.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g)
    if outliers and K:
        x[:, torch.randperm(K, generator=g)[:outliers]] *= scale
    return x.to(dtype)


# --------------------------------------------------------------- step 1
@pytest.mark.parametrize("M,K,dtype", [
    (1, 16, torch.float32), (7, 48, torch.bfloat16), (33, 4096, torch.bfloat16), (16, 256, torch.float32),
    (300, 528, torch.bfloat16), (2048, 4096, torch.bfloat16), (5, 32768, torch.float32),
])
def test_calib_absmax_bit_exact(w, orc, M, K, dtype):
    x = make_x(M, K, dtype, seed=M + K)
    ax = Guarded((K,), torch.float32)
    w.sq_calib_absmax(x.cuda(), ax.t)
    np.testing.assert_array_equal(ax.t.cpu().numpy(), orc.calib_absmax(np32(x)))
    # running max over a second batch equals the max over both
    x2 = make_x(M + 3, K, dtype, seed=M + K + 1)
    w.sq_calib_absmax(x2.cuda(), ax.t, accumulate=True)
    np.testing.assert_array_equal(ax.t.cpu().numpy(), orc.calib_absmax(np.concatenate([np32(x), np32(x2)])))
    assert ax.intact()


def test_calib_absmax_empty_batch_writes_zeros(w):
    ax = torch.full((64,), 7.0, device="cuda")
    w.sq_calib_absmax(torch.empty(0, 64, device="cuda"), ax)
    assert (ax == 0).all()


# --------------------------------------------------------------- step 2
@pytest.mark.parametrize("N,K,dtype,alpha", [
    (13, 48, torch.float32, 0.5), (128, 256, torch.float32, 0.5), (4096, 4096, torch.bfloat16, 0.5),
    (301, 528, torch.bfloat16, 0.8), (64, 256, torch.bfloat16, 0.0), (64, 256, torch.bfloat16, 1.0),
])
def test_smooth_fold(w, orc, N, K, dtype, alpha):
    x = make_x(256, K, dtype, seed=K)
    wt = (torch.randn(N, K, generator=torch.Generator().manual_seed(N)) * 0.02).to(dtype)
    ax = orc.calib_absmax(np32(x))
    ax[0] = 0.0  # an empty activation channel: s must be 1
    aw_d, s_d, inv_d = (Guarded((K,), torch.float32) for _ in range(3))
    fold = Guarded((N, K), torch.float32)
    w.sq_smooth_fold(torch.from_numpy(ax).cuda(), wt.cuda(), alpha, aw_d.t, s_d.t, inv_d.t, fold.t)
    aw = orc.weight_col_absmax(np32(wt))
    np.testing.assert_array_equal(aw_d.t.cpu().numpy(), aw)
    s_ref, _ = orc.smooth_factor(ax, aw, alpha)
    s = s_d.t.cpu().numpy()
    assert s[0] == 1.0
    np.testing.assert_allclose(s, s_ref, rtol=1e-5, atol=0)
    assert np.mean(s == s_ref) > 0.999  # fp64 pow on both sides: ties are vanishingly rare
    np.testing.assert_array_equal(inv_d.t.cpu().numpy(), np.float32(1.0) / s)
    np.testing.assert_array_equal(fold.t.cpu().numpy(), orc.scale_columns(np32(wt), s))
    assert all(g.intact() for g in (aw_d, s_d, inv_d, fold))


@pytest.mark.parametrize("N,K,dtype,alpha", [(13, 48, torch.float32, 0.5), (4096, 4096, torch.bfloat16, 0.5),
                                             (301, 528, torch.bfloat16, 0.8)])
def test_smooth_factor_split(w, orc, N, K, dtype, alpha):
    """Step 2 split in two: the weight's column abs-max by sq_calib_absmax,
    then sq_smooth_factor -- the same s and 1/s as sq_smooth_fold, and the
    oracle's."""
    x = make_x(256, K, dtype, seed=K + 1)
    wt = (torch.randn(N, K, generator=torch.Generator().manual_seed(N + 1)) * 0.02).to(dtype)
    ax = orc.calib_absmax(np32(x))
    ax[1] = 0.0
    axd = torch.from_numpy(ax).cuda()
    aw, s1, inv1, aw2 = (torch.empty(K, device="cuda") for _ in range(4))
    s2, inv2 = Guarded((K,), torch.float32), Guarded((K,), torch.float32)
    w.sq_smooth_fold(axd, wt.cuda(), alpha, aw, s1, inv1)
    w.sq_calib_absmax(wt.cuda(), aw2)
    w.sq_smooth_factor(axd, aw2, alpha, s2.t, inv2.t)
    assert torch.equal(aw2, aw) and torch.equal(s2.t, s1) and torch.equal(inv2.t, inv1)
    s_ref, _ = orc.smooth_factor(ax, orc.weight_col_absmax(np32(wt)), alpha)
    np.testing.assert_allclose(s2.t.cpu().numpy(), s_ref, rtol=1e-5, atol=0)
    assert s2.intact() and inv2.intact()


# --------------------------------------------------------------- step 4
@pytest.mark.parametrize("M,K,dtype,smooth", [
    (1, 16, torch.float32, False), (5, 48, torch.bfloat16, True), (16, 256, torch.float32, True),
    (2048, 4096, torch.bfloat16, True), (33, 8192, torch.bfloat16, True), (3, 12304, torch.bfloat16, True),
    (2, 32768, torch.float32, True), (257, 1040, torch.bfloat16, False),
    # rows staged by bulk copies (M, K >= 1024): ragged token counts, fp32 rows of 16 KB
    (1500, 1040, torch.float32, True), (4099, 2064, torch.bfloat16, True), (1100, 4096, torch.float32, False),
    (1024, 8192, torch.bfloat16, True),
])
def test_quant_act_bit_exact(w, orc, M, K, dtype, smooth):
    x = make_x(M, K, dtype, seed=3 * M + K)
    if M > 2:
        x[1] = 0  # an all-zero token
    inv = (torch.rand(K, generator=torch.Generator().manual_seed(K)) * 4 + 0.05) if smooth else None
    q = Guarded((M, K), torch.int8)
    sx = Guarded((M,), torch.float32)
    w.quant_act_per_token(x.cuda(), None if inv is None else inv.cuda(), q.t, sx.t)
    q_ref, sx_ref = orc.quant_act_per_token(np32(x), None if inv is None else inv.numpy())
    np.testing.assert_array_equal(sx.t.cpu().numpy(), sx_ref)
    np.testing.assert_array_equal(q.t.cpu().numpy(), q_ref)
    assert q.intact() and sx.intact()


def test_quant_act_golden_ties(w):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "act_round_half_even.txt"))
            if l.strip() and not l.startswith("#")]
    vals = [float(a) for a, _ in rows]
    want = [int(b) for _, b in rows]
    K = 16 * ((len(vals) + 15) // 16)
    x = torch.zeros(1, K)
    x[0, :len(vals)] = torch.tensor(vals)
    q = torch.empty(1, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(1, device="cuda")
    w.quant_act_per_token(x.cuda(), None, q, sx)
    assert sx.item() == 1.0
    assert q[0, :len(vals)].cpu().tolist() == want


# --------------------------------------------------------------- step 3
def _ssz_check(w, orc, wt, s, bits, max_iters=20):
    N, K = wt.shape
    q = Guarded((N, K), torch.int8)
    sc = Guarded((N,), torch.float32)
    mse = torch.empty(N, dtype=torch.float64, device="cuda")
    its = torch.empty(N, dtype=torch.int32, device="cuda")
    w.ssz_quant_weight(wt.cuda(), None if s is None else s.cuda(), bits, max_iters, q.t, sc.t, mse, its)
    wf = np32(wt) if s is None else orc.scale_columns(np32(wt), s.numpy())
    ref = orc.ssz_quant_weight(wf, bits=bits, max_iters=max_iters)
    scale = sc.t.cpu().numpy()
    # scales within 1e-5 relative of the oracle's search
    np.testing.assert_allclose(scale, ref["scale"], rtol=1e-5, atol=0)
    # codes bit-exact given the GPU's scales
    np.testing.assert_array_equal(q.t.cpu().numpy(), orc.weight_codes(wf, scale, bits))
    # the reported error is the error at the returned scale
    mse_ref = np.array([orc.channel_mse(wf[n], scale[n], bits) for n in range(N)])
    np.testing.assert_allclose(mse.cpu().numpy(), mse_ref, rtol=1e-9, atol=1e-300)
    same = (scale == ref["scale"]) & (its.cpu().numpy() == ref["iters"])
    assert q.intact() and sc.intact()
    return same.mean()


@pytest.mark.parametrize("N,K,dtype,bits,smooth", [
    (5, 16, torch.float32, 8, False), (5, 16, torch.float32, 4, False), (128, 256, torch.float32, 8, True),
    (300, 4096, torch.bfloat16, 8, True), (300, 4096, torch.bfloat16, 4, True), (17, 528, torch.bfloat16, 8, True),
    (64, 1040, torch.bfloat16, 4, False), (2, 32768, torch.float32, 8, True), (40, 20000, torch.bfloat16, 8, True),
])
def test_ssz_parity(w, orc, N, K, dtype, bits, smooth):
    g = torch.Generator().manual_seed(N * 7 + K)
    wt = torch.randn(N, K, generator=g) * 0.02
    wt.view(-1)[torch.randperm(N * K, generator=g)[: max(1, N * K // 1000)]] *= 10
    if N > 3:
        wt[2] = 0.0          # all-zero channel: minimum scale, zero codes
        wt[3] = 1e-7         # tiny channel: floored scale, no least-squares codes
    wt = wt.to(dtype)
    s = (torch.rand(K, generator=g) * 3 + 0.2) if smooth else None
    assert _ssz_check(w, orc, wt, s, bits) > 0.999


def test_ssz_max_iters_zero_is_minmax(w, orc):
    wt = (torch.randn(64, 256) * 0.02).to(torch.bfloat16)
    assert _ssz_check(w, orc, wt, None, 8, max_iters=0) == 1.0


# --------------------------------------------------------------- step 5
def _gemm_case(M, N, K, seed, extreme=False):
    g = torch.Generator().manual_seed(seed)
    if extreme:
        qx = torch.full((M, K), 127, dtype=torch.int8)
        qw = torch.full((N, K), -127, dtype=torch.int8)
        qw[::2] = 127
    else:
        qx = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
        qw = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    sx = torch.rand(M, generator=g) * 0.05
    sw = torch.rand(N, generator=g) * 1e-3
    return qx, qw, sx, sw


@pytest.mark.parametrize("M,N,K,ydt", [
    (1, 16, 16, torch.bfloat16), (7, 24, 48, torch.bfloat16), (129, 264, 144, torch.bfloat16),
    (128, 256, 128, torch.bfloat16), (256, 512, 256, torch.float32), (16, 128, 256, torch.float32),
    (300, 520, 4096, torch.bfloat16), (1000, 2056, 1040, torch.bfloat16), (16, 28672, 512, torch.bfloat16),
    (200, 24, 64, torch.bfloat16), (130, 12, 48, torch.float32), (520, 392, 272, torch.float32),
    # 64 < M <= 128 with few column tiles and a long K: the decode kernel's
    # 128-token tiles (split K); then the one-CTA kernel with a short K
    (120, 1040, 4096, torch.bfloat16), (65, 264, 2048, torch.float32), (100, 264, 1024, torch.bfloat16),
])
def test_gemm_bit_exact(w, orc, M, N, K, ydt):
    qx, qw, sx, sw = _gemm_case(M, N, K, seed=M * 31 + N * 7 + K)
    y = Guarded((M, N), ydt)
    acc = Guarded((M, N), torch.int32)
    w.w8a8_gemm_dequant(qx.cuda(), sx.cuda(), qw.cuda(), sw.cuda(), y.t, acc.t)
    acc_ref = orc.gemm_i8(qx.numpy(), qw.numpy())
    np.testing.assert_array_equal(acc.t.cpu().numpy(), acc_ref)
    if ydt == torch.bfloat16:
        yb = y.t.cpu().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(yb, orc.dequant(acc_ref, sx.numpy(), sw.numpy(), out="bf16"))
    else:
        np.testing.assert_array_equal(y.t.cpu().numpy(), orc.dequant(acc_ref, sx.numpy(), sw.numpy(), out="f32"))
    assert y.intact() and acc.intact()
    # without acc_out the output is the same
    y2 = torch.empty(M, N, dtype=ydt, device="cuda")
    w.w8a8_gemm_dequant(qx.cuda(), sx.cuda(), qw.cuda(), sw.cuda(), y2)
    assert torch.equal(y2, y.t)


# the pair kernel at K = 8192; then K = 133136, the largest multiple of 16
# the call accepts (127 * 127 * K just below 2^31, a partial last k-block),
# on the one-CTA kernel (M <= 128) and the pair kernel
@pytest.mark.parametrize("M,N,K", [(130, 264, 8192), (100, 16, 133136), (130, 16, 133136)])
def test_gemm_extreme_codes_do_not_overflow(w, orc, M, N, K):
    qx, qw, sx, sw = _gemm_case(M, N, K, seed=5, extreme=True)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    w.w8a8_gemm_dequant(qx.cuda(), sx.cuda(), qw.cuda(), sw.cuda(), y, acc)
    a = acc.cpu().numpy()
    assert a[0, 0] == 127 * 127 * K and a[0, 1] == -127 * 127 * K
    np.testing.assert_array_equal(a, orc.gemm_i8(qx.numpy(), qw.numpy()))


# --------------------------------------------------------------- whole path
def run_path(w, x, wt, alpha, bits):
    """All five calls on the GPU; returns every intermediate on the host."""
    M, K = x.shape
    N = wt.shape[0]
    dev = dict(device="cuda")
    xd, wd = x.cuda(), wt.cuda()
    ax = torch.empty(K, **dev)
    aw, s, inv = (torch.empty(K, **dev) for _ in range(3))
    qw = torch.empty(N, K, dtype=torch.int8, **dev)
    sw = torch.empty(N, **dev)
    mse = torch.empty(N, dtype=torch.float64, **dev)
    its = torch.empty(N, dtype=torch.int32, **dev)
    qx = torch.empty(M, K, dtype=torch.int8, **dev)
    sx = torch.empty(M, **dev)
    y = torch.empty(M, N, dtype=x.dtype, **dev)
    w.sq_calib_absmax(xd, ax)
    w.sq_smooth_fold(ax, wd, alpha, aw, s, inv)
    w.ssz_quant_weight(wd, s, bits, 20, qw, sw, mse, its)
    w.quant_act_per_token(xd, inv, qx, sx)
    if bits == 8:
        w.w8a8_gemm_dequant(qx, sx, qw, sw, y)
    out = dict(ax=ax, aw=aw, s=s, inv_s=inv, qw=qw, sw=sw, iters=its, qx=qx, sx=sx, y=y)
    return {k: v.cpu() for k, v in out.items()}


def _sample(n, k, seed):
    if k >= n:
        return np.arange(n)
    return np.sort(np.random.default_rng(seed).choice(n, k, replace=False))


@pytest.mark.parametrize("name", synthetic.ORDER)
def test_end_to_end_workloads(w, orc, name):
    cfg = synthetic.CONFIGS[name]
    x, wt = synthetic.make_linear(cfg, seed=0)
    got = run_path(w, x, wt, cfg.alpha, cfg.bits)
    xf, wf = np32(x), np32(wt)
    ax = orc.calib_absmax(xf)
    np.testing.assert_array_equal(got["ax"].numpy(), ax)
    aw = orc.weight_col_absmax(wf)
    np.testing.assert_array_equal(got["aw"].numpy(), aw)
    s, inv_s = orc.smooth_factor(ax, aw, cfg.alpha)
    np.testing.assert_allclose(got["s"].numpy(), s, rtol=1e-5, atol=0)
    # sampled output channels and tokens (the oracle is slow at full size)
    rows_n = _sample(cfg.N, 512, 1)
    rows_m = _sample(cfg.M, 64, 2)
    wq = orc.ssz_quant_weight(wf[rows_n], bits=cfg.bits, s=s)
    np.testing.assert_allclose(got["sw"].numpy()[rows_n], wq["scale"], rtol=1e-5, atol=0)
    code_mismatch = np.mean(got["qw"].numpy()[rows_n] != wq["q"])
    assert code_mismatch < 1e-5
    qx, sx = orc.quant_act_per_token(xf[rows_m], inv_s)
    np.testing.assert_allclose(got["sx"].numpy()[rows_m], sx, rtol=1e-5, atol=0)
    assert np.mean(got["qx"].numpy()[rows_m] != qx) < 1e-5
    if cfg.bits == 8:
        acc = orc.gemm_i8(qx, wq["q"])
        y_ref = orc.dequant(acc, sx, wq["scale"], out="f32")
        if cfg.out_dtype == "bf16":
            y_ref = orc.bf16_bits_to_f32(orc.to_bf16_bits(y_ref))
        y = np32(got["y"])[np.ix_(rows_m, rows_n)]
        np.testing.assert_allclose(y, y_ref, rtol=1e-3, atol=1e-5)
    else:
        # the int4 decode workload also runs its int8 GEMM path
        qw8 = torch.empty(cfg.N, cfg.K, dtype=torch.int8, device="cuda")
        sw8 = torch.empty(cfg.N, device="cuda")
        w.ssz_quant_weight(wt.cuda(), got["s"].cuda(), 8, 20, qw8, sw8)
        y = torch.empty(cfg.M, cfg.N, dtype=torch.bfloat16, device="cuda")
        w.w8a8_gemm_dequant(got["qx"].cuda(), got["sx"].cuda(), qw8, sw8, y)
        acc = orc.gemm_i8(got["qx"].numpy()[rows_m], qw8.cpu().numpy()[rows_n])
        yb = y.cpu().view(torch.int16).numpy().view(np.uint16)[np.ix_(rows_m, rows_n)]
        np.testing.assert_array_equal(yb, orc.dequant(acc, got["sx"].numpy()[rows_m], sw8.cpu().numpy()[rows_n]))


# --------------------------------------------------------------- failure path
def test_bounded_wait_gives_up_and_context_survives(w, orc):
    assert w.device_fault() == 0
    w.selftest_bounded_wait(50)
    assert w.device_fault() == 6
    assert w.device_fault() == 0  # read-and-clear
    qx, qw, sx, sw = _gemm_case(64, 64, 64, seed=9)
    y = torch.empty(64, 64, dtype=torch.float32, device="cuda")
    w.w8a8_gemm_dequant(qx.cuda(), sx.cuda(), qw.cuda(), sw.cuda(), y)
    acc_ref = orc.gemm_i8(qx.numpy(), qw.numpy())
    np.testing.assert_array_equal(y.cpu().numpy(), orc.dequant(acc_ref, sx.numpy(), sw.numpy(), out="f32"))
    assert w.device_fault() == 0


def test_w8a8_linear_module_matches_calls(w):
    x, wt = synthetic.make_small(96, 512, 384, seed=4)
    lin = w.W8A8Linear(wt.cuda(), alpha=0.5)
    lin.calibrate(x.cuda())
    lin.quantize()
    y = lin.forward(x.cuda())
    ref = run_path(w, x, wt, 0.5, 8)
    assert torch.equal(y.cpu(), ref["y"])

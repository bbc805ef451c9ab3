"""GPU parity of the LayerNorm fused with smoothing and per-token
quantization (activation quantization fused upstream) against the oracle.

SmoothQuant page section 1 (the smoothing moves into the op that produces
X) and the CUDA INT8 notes 4.2 (fused kernel, no intermediate in memory).
Both sides compute the statistics as fp64 pairwise sums (the row padded
with zeros to a power of two, summed by recursive halving), so the
statistics, the scales and the int8 codes must match bit for bit.
"""
import numpy as np
import pytest
import torch

from tests.test_parity_gpu import Guarded, make_x, np32, w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,dtype,affine,smooth", [
    (1, 16, torch.float32, False, False), (7, 48, torch.bfloat16, True, False), (300, 528, torch.bfloat16, True, True),
    (129, 1040, torch.float32, True, True), (2048, 4096, torch.bfloat16, True, True),
    (33, 8192, torch.bfloat16, False, True), (5, 16384, torch.float32, True, True),
    (64, 3072, torch.bfloat16, True, True), (17, 272, torch.float32, False, True),
])
def test_layernorm_quant_parity(w, orc, M, K, dtype, affine, smooth):
    h = make_x(M, K, dtype, seed=M + K, scale=20.0)
    r = np.random.default_rng(K)
    g = (r.random(K) + 0.5).astype(np.float32) if affine else None
    b = (r.standard_normal(K) * 0.1).astype(np.float32) if affine else None
    inv = (r.random(K) * 2 + 0.1).astype(np.float32) if smooth else None
    d = lambda a: None if a is None else torch.from_numpy(a).cuda()  # noqa: E731
    q = Guarded((M, K), torch.int8)
    sx = Guarded((M,), torch.float32)
    w.sq_layernorm_quant(h.cuda(), d(g), d(b), 1e-5, d(inv), q.t, sx.t)
    qo, sxo, _ = orc.layernorm_quant(np32(h), g, b, 1e-5, inv)
    np.testing.assert_array_equal(sx.t.cpu().numpy(), sxo)
    np.testing.assert_array_equal(q.t.cpu().numpy(), qo)
    assert q.intact() and sx.intact()


@pytest.mark.parametrize("K", [16, 48, 1024, 4096])
def test_layernorm_quant_order_sensitive_rows(w, orc, K):
    """Rows whose fp64 sums depend on the summation order (entries of
    magnitude 2^53 beside small ones): the codes and scales still match the
    oracle's pairwise tree bit for bit."""
    r = np.random.default_rng(K + 5)
    h = (r.standard_normal((6, K)) * 4.0).astype(np.float32)
    big = np.float32(2.0 ** 53)
    for t in range(6):
        cols = r.choice(K, 4, replace=False)
        h[t, cols[:2]] = big
        h[t, cols[2:]] = -big
        h[t, r.choice(K, 3, replace=False)] += np.float32(0.5)
    inv = (r.random(K) + 0.5).astype(np.float32)
    q = Guarded((6, K), torch.int8)
    sx = Guarded((6,), torch.float32)
    w.sq_layernorm_quant(torch.from_numpy(h).cuda(), None, None, 1e-5, torch.from_numpy(inv).cuda(), q.t, sx.t)
    qo, sxo, _ = orc.layernorm_quant(h, None, None, 1e-5, inv)
    np.testing.assert_array_equal(sx.t.cpu().numpy(), sxo)
    np.testing.assert_array_equal(q.t.cpu().numpy(), qo)
    assert q.intact() and sx.intact()


def test_layernorm_quant_constant_rows_and_eps_zero(w, orc):
    h = torch.full((4, 64), 2.5, dtype=torch.bfloat16)
    q = torch.full((4, 64), 9, dtype=torch.int8, device="cuda")
    sx = torch.full((4,), 7.0, device="cuda")
    w.sq_layernorm_quant(h.cuda(), None, None, 1e-5, None, q, sx)
    assert not q.any() and not sx.any()
    x = make_x(16, 256, torch.float32, seed=3)
    w.sq_layernorm_quant(x.cuda(), None, None, 0.0, None, q.new_empty(16, 256), sx.new_empty(16))

"""GPU parity of the few-token GEMM kernel (M <= 64 tokens) against the CPU
oracle.

Same operation as the other GEMM kernels (CUDA INT8 notes sections 3.2 and
4.2: integer product with the dequant fused): the weight tile is the MMA's
128-row operand and the tokens the narrow one, and where N / 128 tiles are too
few for the SMs the K dimension is split over a thread-block cluster of 2, 4
or 8 CTAs whose int32 partials are summed through distributed shared memory.
Accumulators and outputs must match the oracle bit for bit at every token
width (16, 32, 64), every split, ragged M, N and K, with int8, asymmetric
int8 and packed int4 weights.
"""
import numpy as np
import pytest
import torch

from tests.test_parity_gpu import Guarded, w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


def split_of(N, K, sms=148):
    """The K split the launcher picks (largest power of two <= 8 with
    ceil(N/128) x S <= 2 x SMs and S <= ceil(K/128))."""
    tiles, kb, s = -(-N // 128), -(-K // 128), 1
    while s < 8 and tiles * 2 * s <= 2 * sms and 2 * s <= kb:
        s *= 2
    return s


def _case(M, N, K, seed, extreme=False):
    r = np.random.default_rng(seed)
    if extreme:
        qx = np.full((M, K), 127, np.int8)
        qw = np.full((N, K), 127, np.int8)
        qw[1::2] = -127
    else:
        qx = r.integers(-127, 128, (M, K)).astype(np.int8)
        qw = r.integers(-127, 128, (N, K)).astype(np.int8)
    sx = (r.random(M) * 0.05 + 1e-3).astype(np.float32)
    sw = (r.random(N) * 1e-3 + 1e-5).astype(np.float32)
    return qx, qw, sx, sw


def _d(a):
    return torch.from_numpy(a).cuda()


DECODE_SHAPES = [
    # M, N, K, output dtype                      split  token tile
    (1, 8, 4096, torch.bfloat16),               # 8      16
    (5, 264, 1040, torch.float32),              # 8      16 (9 k-blocks over 8 CTAs)
    (16, 136, 272, torch.bfloat16),             # 2      16
    (17, 1024, 2048, torch.bfloat16),           # 8      32
    (32, 11008, 512, torch.float32),            # 2      32
    (48, 5120, 1024, torch.float32),            # 4      64
    (33, 4096, 8192, torch.bfloat16),           # 8      64
    (64, 28672, 1024, torch.bfloat16),          # 1      64
    (16, 28672, 8192, torch.bfloat16),          # 1      16 (the decode workload)
]


@pytest.mark.parametrize("M,N,K,ydt", DECODE_SHAPES)
def test_decode_gemm_bit_exact(w, orc, M, N, K, ydt):
    qx, qw, sx, sw = _case(M, N, K, seed=M * 7 + N + K)
    y = Guarded((M, N), ydt)
    acc = Guarded((M, N), torch.int32)
    w.w8a8_gemm_dequant(_d(qx), _d(sx), _d(qw), _d(sw), y.t, acc.t)
    acc_o = orc.gemm_i8(qx, qw)
    np.testing.assert_array_equal(acc.t.cpu().numpy(), acc_o)
    if ydt == torch.bfloat16:
        np.testing.assert_array_equal(y.t.cpu().view(torch.int16).numpy().view(np.uint16),
                                      orc.dequant(acc_o, sx, sw, out="bf16"))
    else:
        np.testing.assert_array_equal(y.t.cpu().numpy(), orc.dequant(acc_o, sx, sw, out="f32"))
    assert y.intact() and acc.intact()
    y2 = torch.empty(M, N, dtype=ydt, device="cuda")
    w.w8a8_gemm_dequant(_d(qx), _d(sx), _d(qw), _d(sw), y2)  # without acc_out
    assert torch.equal(y2, y.t)


def test_decode_split_covers_every_width():
    """The shapes above reach every split and every token tile."""
    splits = {split_of(N, K) for _, N, K, _ in DECODE_SHAPES}
    tiles = {16 if M <= 16 else 32 if M <= 32 else 64 for M, _, _, _ in DECODE_SHAPES}
    assert splits == {1, 2, 4, 8} and tiles == {16, 32, 64}
    assert split_of(8, 4096) == 8 and split_of(136, 272) == 2 and split_of(28672, 8192) == 1


@pytest.mark.parametrize("M,N,K", [(1, 264, 8192), (64, 128, 133120)])
def test_decode_extreme_codes_do_not_overflow(w, orc, M, N, K):
    """|acc| up to 127 * 127 * K with the partials of a split K summed."""
    qx, qw, sx, sw = _case(M, N, K, seed=3, extreme=True)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    w.w8a8_gemm_dequant(_d(qx), _d(sx), _d(qw), _d(sw), y, acc)
    a = acc.cpu().numpy()
    assert a[0, 0] == 127 * 127 * K and a[0, 1] == -127 * 127 * K
    np.testing.assert_array_equal(a, orc.gemm_i8(qx, qw))


@pytest.mark.parametrize("M,N,K,ydt", [(1, 8, 16, torch.bfloat16), (16, 264, 4096, torch.float32),
                                       (40, 520, 1040, torch.bfloat16), (16, 28672, 1024, torch.bfloat16)])
def test_decode_gemm_asym_bit_exact(w, orc, M, N, K, ydt):
    r = np.random.default_rng(M + N + K)
    qx = r.integers(-127, 128, (M, K)).astype(np.int8)
    qw = r.integers(-128, 128, (N, K)).astype(np.int8)
    sx = (r.random(M) * 0.05 + 1e-3).astype(np.float32)
    sw = (r.random(N) * 1e-3 + 1e-5).astype(np.float32)
    ow = (r.standard_normal(N) * 0.05).astype(np.float32)
    R = orc.act_rowsum(qx)
    y = Guarded((M, N), ydt)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    w.w8a8_gemm_dequant_asym(_d(qx), _d(sx), _d(R), _d(qw), _d(sw), _d(ow), y.t, acc)
    acc_o = orc.gemm_i8(qx, qw)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    if ydt == torch.bfloat16:
        np.testing.assert_array_equal(y.t.cpu().view(torch.int16).numpy().view(np.uint16),
                                      orc.dequant_asym(acc_o, R, sx, sw, ow))
    else:
        np.testing.assert_array_equal(y.t.cpu().numpy(), orc.dequant_asym(acc_o, R, sx, sw, ow, out="f32"))
    assert y.intact()


@pytest.mark.parametrize("M,N,K,ydt", [(1, 8, 32, torch.bfloat16), (16, 264, 4096, torch.float32),
                                       (33, 1032, 2080, torch.bfloat16), (64, 4096, 8192, torch.bfloat16),
                                       (16, 28672, 8192, torch.bfloat16)])
def test_decode_w4a8_bit_exact(w, orc, M, N, K, ydt):
    r = np.random.default_rng(M * N + K)
    qx = r.integers(-127, 128, (M, K)).astype(np.int8)
    q4 = r.integers(-8, 8, (N, K)).astype(np.int8)
    sx = (r.random(M) * 0.05 + 1e-3).astype(np.float32)
    sw = (r.random(N) * 1e-2 + 1e-5).astype(np.float32)
    p = torch.empty(N, K // 2, dtype=torch.uint8, device="cuda")
    w.sq_pack_int4(_d(q4), p)
    y = Guarded((M, N), ydt)
    acc = torch.empty(M, N, dtype=torch.int32, device="cuda")
    w.w4a8_gemm_dequant(_d(qx), _d(sx), p, _d(sw), y.t, acc)
    acc_o = orc.gemm_i8(qx, orc.unpack_int4(orc.pack_int4(q4), K))
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    if ydt == torch.bfloat16:
        np.testing.assert_array_equal(y.t.cpu().view(torch.int16).numpy().view(np.uint16),
                                      orc.dequant(acc_o, sx, sw))
    else:
        np.testing.assert_array_equal(y.t.cpu().numpy(), orc.dequant(acc_o, sx, sw, out="f32"))
    assert y.intact()


@pytest.mark.parametrize("M", [1, 16, 64])
def test_decode_equals_wide_tile_kernel(w, M):
    """Tokens 1..64 (decode kernel) and the same rows inside a 65..128-token
    batch (the 128 x 256 tile kernel) give the same outputs."""
    N, K = 1024, 4096
    qx, qw, sx, sw = _case(128, N, K, seed=M)
    big = torch.empty(128, N, dtype=torch.bfloat16, device="cuda")
    w.w8a8_gemm_dequant(_d(qx), _d(sx), _d(qw), _d(sw), big)
    small = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    w.w8a8_gemm_dequant(_d(qx[:M].copy()), _d(sx[:M].copy()), _d(qw), _d(sw), small)
    assert torch.equal(small.view(torch.int16), big[:M].view(torch.int16))

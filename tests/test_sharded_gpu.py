"""GPU pieces of the K-sharded (row-parallel) linear, against the oracle and
against the unsharded path (ranks emulated on one GPU: each shard's kernels
run in turn and the MAX / SUM exchange is taken on the device between them;
no kernel waits on another)."""
import numpy as np
import pytest
import torch

from tests.test_parity_gpu import Guarded, make_x, np32, w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,dtype", [(1, 16, torch.float32), (77, 528, torch.bfloat16), (300, 4096, torch.bfloat16)])
def test_quant_act_given_scale_bit_exact(w, orc, M, K, dtype):
    x = make_x(M, K, dtype, seed=M + K)
    inv = (np.random.default_rng(K).random(K) + 0.5).astype(np.float32)
    _, sx = orc.quant_act_per_token(np32(x), inv)
    sx = (sx * np.float32(0.7)).astype(np.float32)  # narrower than each row: saturation
    sx[0] = 0.0
    q = Guarded((M, K), torch.int8)
    w.quant_act_given_scale(x.cuda(), torch.from_numpy(inv).cuda(), torch.from_numpy(sx).cuda(), q.t)
    np.testing.assert_array_equal(q.t.cpu().numpy(), orc.quant_act_given_scale(np32(x), inv, sx))
    assert q.intact()


@pytest.mark.parametrize("M,N,ydt", [(1, 4, torch.float32), (77, 264, torch.bfloat16), (300, 1028, torch.float32)])
def test_dequant_bit_exact(w, orc, M, N, ydt):
    r = np.random.default_rng(M * N)
    acc = r.integers(-2**30, 2**30, (M, N)).astype(np.int32)
    sx = (r.random(M) * 1e-3).astype(np.float32)
    sw = (r.random(N) * 1e-3).astype(np.float32)
    y = Guarded((M, N), ydt)
    w.sq_dequant(torch.from_numpy(acc).cuda(), torch.from_numpy(sx).cuda(), torch.from_numpy(sw).cuda(), y.t)
    if ydt == torch.bfloat16:
        np.testing.assert_array_equal(y.t.cpu().view(torch.int16).numpy().view(np.uint16), orc.dequant(acc, sx, sw))
    else:
        np.testing.assert_array_equal(y.t.cpu().numpy(), orc.dequant(acc, sx, sw, out="f32"))
    assert y.intact()


def test_row_parallel_emulated_equals_unsharded(w):
    from w8a8_linear_layers_b200.distributed import KernelOps
    ops = KernelOps(w)
    M, K, N = 256, 4096, 1024
    x = make_x(M, K, torch.bfloat16, seed=9).cuda()
    inv = torch.rand(K, device="cuda") + 0.5
    qw = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda")
    sw = torch.rand(N, device="cuda") * 1e-3
    # unsharded
    qx = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    w.quant_act_per_token(x, inv, qx, sx)
    y_full = torch.empty(M, N, device="cuda")
    w.w8a8_gemm_dequant(qx, sx, qw, sw, y_full)
    # four shards of K
    cuts = [0, 1024, 1536, 3072, 4096]
    parts = [(x[:, a:b].contiguous(), inv[a:b].contiguous(), qw[:, a:b].contiguous()) for a, b in zip(cuts, cuts[1:])]
    sx_g = torch.stack([ops.per_token_scales(xs, iv) for xs, iv, _ in parts]).amax(0)
    assert torch.equal(sx_g, sx)
    acc = sum(ops.gemm_acc(ops.quant_given(xs, iv, sx_g), q, sx_g, sw) for xs, iv, q in parts)
    y = torch.empty(M, N, device="cuda")
    ops.dequant(acc.to(torch.int32), sx_g, sw, y)
    assert torch.equal(y, y_full)


@pytest.mark.parametrize("G", [2, 3])
def test_ssz_by_output_channel_blocks_equals_unsharded(w, G):
    """SSZ on each rank's block of output channels (ranks emulated in turn)
    concatenates to the unsharded search: codes, scales and rounds bit for
    bit (the channels are independent)."""
    import synthetic
    from w8a8_linear_layers_b200.distributed import shard_rows
    x, wt = synthetic.make_small(64, 1040, 203, seed=11, w_outliers=20)
    wt = wt.cuda()
    N, K = wt.shape
    s = torch.rand(K, device="cuda") + 0.5
    q, sc, its = (torch.empty(N, K, dtype=torch.int8, device="cuda"), torch.empty(N, device="cuda"),
                  torch.empty(N, dtype=torch.int32, device="cuda"))
    w.ssz_quant_weight(wt, s, 8, 20, q, sc, iters_out=its)
    for r in range(G):
        a, b = shard_rows(N, G, r)
        qr, sr, ir = (torch.empty(b - a, K, dtype=torch.int8, device="cuda"), torch.empty(b - a, device="cuda"),
                      torch.empty(b - a, dtype=torch.int32, device="cuda"))
        w.ssz_quant_weight(wt[a:b].contiguous(), s, 8, 20, qr, sr, iters_out=ir)
        assert torch.equal(qr, q[a:b]) and torch.equal(sr, sc[a:b]) and torch.equal(ir, its[a:b])


def test_column_parallel_blocks_equal_unsharded_columns(w):
    """The column-parallel linear's per-rank products (ranks emulated in
    turn, each on its block of output channels) are the unsharded output's
    columns, bit for bit."""
    from w8a8_linear_layers_b200.distributed import KernelOps, column_parallel_linear, shard_rows
    M, K, N, G = 300, 1024, 1032, 3
    x = make_x(M, K, torch.bfloat16, seed=12).cuda()
    inv = torch.rand(K, device="cuda") + 0.5
    qw = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda")
    sw = torch.rand(N, device="cuda") * 1e-3
    qx, sx = torch.empty(M, K, dtype=torch.int8, device="cuda"), torch.empty(M, device="cuda")
    w.quant_act_per_token(x, inv, qx, sx)
    y_full = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    w.w8a8_gemm_dequant(qx, sx, qw, sw, y_full)
    ops = KernelOps(w)
    for r in range(G):
        a, b = shard_rows(N, G, r)
        assert (b - a) % 8 == 0  # bf16 output rows of 16 bytes
        y_r = torch.empty(M, b - a, dtype=torch.bfloat16, device="cuda")
        column_parallel_linear(x, inv, qw[a:b].contiguous(), sw[a:b].contiguous(), y_r, ops=ops)
        assert torch.equal(y_r, y_full[:, a:b])

"""Multi-rank path on CPU (gloo, world size 2).

The data-parallel calibration exchange (MAX all-reduce of the per-channel
activation absmax) must give every rank the absmax of the global batch,
bit-identically, so that every replica derives the same smoothing factor and
the same SSZ-quantized weight.  Max-over-ranks timing is checked too, and a
rank that leaves before the collective makes the other fail with an error
within the process-group timeout instead of hanging.
"""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=20):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))


def _calibration_worker(rank, world, port, outdir):
    _init(rank, world, port)
    try:
        import oracle
        import synthetic
        from w8a8_linear_layers_b200 import distributed as wdist
        # each rank: its own token batch (seed = rank), the same weight
        x, wt = synthetic.make_small(24 + 8 * rank, 64, 40, seed=rank)
        _, wt0 = synthetic.make_small(24, 64, 40, seed=0)
        ax = torch.from_numpy(oracle.calib_absmax(x.float().numpy()))
        wdist.allreduce_calibration(ax)
        s, inv_s = oracle.smooth_factor(ax.numpy(), oracle.weight_col_absmax(wt0.float().numpy()), 0.5)
        q = oracle.ssz_quant_weight(wt0.float().numpy(), bits=8, s=s)
        t = wdist.max_over_ranks(float(rank + 1))
        np.savez(os.path.join(outdir, "rank%d.npz" % rank), ax=ax.numpy(), s=s, scale=q["scale"], q=q["q"],
                 t=np.array([t]))
    finally:
        dist.destroy_process_group()


def test_calibration_allreduce_matches_global_batch():
    import oracle
    import synthetic
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_calibration_worker, args=(2, _free_port(), d), nprocs=2, join=True)
        r0 = np.load(os.path.join(d, "rank0.npz"))
        r1 = np.load(os.path.join(d, "rank1.npz"))
    x0, _ = synthetic.make_small(24, 64, 40, seed=0)
    x1, _ = synthetic.make_small(32, 64, 40, seed=1)
    glob = oracle.calib_absmax(np.concatenate([x0.float().numpy(), x1.float().numpy()]))
    for r in (r0, r1):
        np.testing.assert_array_equal(r["ax"], glob)          # exact: MAX is order-free
        assert r["t"][0] == 2.0                                # max over ranks
    for k in ("s", "scale", "q"):
        np.testing.assert_array_equal(r0[k], r1[k])           # identical replicas


def _dropout_worker(rank, world, port, outdir):
    _init(rank, world, port, timeout_s=3)
    from w8a8_linear_layers_b200 import distributed as wdist
    if rank == 1:
        # leaves between steps, without joining the next collective
        dist.destroy_process_group()
        return
    ax = torch.ones(16)
    try:
        wdist.allreduce_calibration(ax)
        status = "no error"
    except Exception as e:  # gloo: timeout or connection closed
        status = "error: " + type(e).__name__
    with open(os.path.join(outdir, "status.txt"), "w") as f:
        f.write(status)


def test_rank_leaving_fails_the_collective_instead_of_hanging():
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_dropout_worker, args=(2, _free_port(), d), nprocs=2, join=True)
        status = open(os.path.join(d, "status.txt")).read()
    assert status.startswith("error"), status


def test_single_rank_helpers_are_noops():
    from w8a8_linear_layers_b200 import distributed as wdist
    ax = torch.arange(8, dtype=torch.float32)
    wdist.allreduce_calibration(ax)
    assert torch.equal(ax, torch.arange(8, dtype=torch.float32))
    assert wdist.max_over_ranks(3.5) == 3.5
    assert wdist.world_size() == 1


# ------------------------------------------------------------ K-sharded linear
class _OracleOps:
    """The kernels of the K-sharded linear, computed by the CPU oracle (this
    checks the exchange itself: MAX of scales, exact SUM of products)."""

    def __init__(self, oracle):
        self.o = oracle

    def per_token_scales(self, x, inv_s):
        return torch.from_numpy(self.o.quant_act_per_token(x.numpy(), inv_s.numpy())[1].copy())

    def quant_given(self, x, inv_s, sx):
        return torch.from_numpy(self.o.quant_act_given_scale(x.numpy(), inv_s.numpy(), sx.numpy()))

    def gemm_acc(self, qx, qw, sx, sw):
        return torch.from_numpy(self.o.gemm_i8(qx.numpy(), qw.numpy()))

    def dequant(self, acc, sx, sw, y):
        y.copy_(torch.from_numpy(self.o.dequant(acc.numpy(), sx.numpy(), sw.numpy(), out="f32")))

    def ssz(self, w_rows, s, bits, max_iters, q_out, scale_out, iters_out):
        r = self.o.ssz_quant_weight(w_rows.float().numpy(), bits=bits, max_iters=max_iters,
                                    s=None if s is None else s.numpy())
        q_out.copy_(torch.from_numpy(r["q"]))
        scale_out.copy_(torch.from_numpy(r["scale"]))
        iters_out.copy_(torch.from_numpy(r["iters"]))

    def quant_act(self, x, inv_s, qx, sx):
        q, s = self.o.quant_act_per_token(x.float().numpy(), None if inv_s is None else inv_s.numpy())
        qx.copy_(torch.from_numpy(q))
        sx.copy_(torch.from_numpy(s))

    def gemm(self, qx, sx, qw, sw, y):
        acc = self.o.gemm_i8(qx.numpy(), qw.numpy())
        if y.dtype == torch.bfloat16:
            y.view(torch.int16).copy_(torch.from_numpy(self.o.dequant(acc, sx.numpy(), sw.numpy()).view(np.int16)))
        else:
            y.copy_(torch.from_numpy(self.o.dequant(acc, sx.numpy(), sw.numpy(), out="f32")))


def _row_parallel_worker(rank, world, port, outdir):
    _init(rank, world, port)
    try:
        import oracle
        from w8a8_linear_layers_b200 import distributed as wdist
        r = np.random.default_rng(0)
        K = 96
        x = (r.standard_normal((12, K)) * np.where(np.arange(K) % 17 == 0, 30.0, 1.0)).astype(np.float32)
        inv = (r.random(K) + 0.5).astype(np.float32)
        qw = r.integers(-127, 128, (24, K)).astype(np.int8)
        sw = (r.random(24) * 0.01).astype(np.float32)
        cut = [0, 48, 96][rank:rank + 2]
        sl = slice(cut[0], cut[1])
        y = torch.empty(12, 24)
        wdist.row_parallel_linear(torch.from_numpy(x[:, sl].copy()), torch.from_numpy(inv[sl].copy()),
                                  torch.from_numpy(qw[:, sl].copy()), torch.from_numpy(sw), y,
                                  ops=_OracleOps(oracle))
        np.save(os.path.join(outdir, "y%d.npy" % rank), y.numpy())
    finally:
        dist.destroy_process_group()


def test_row_parallel_linear_equals_unsharded():
    import oracle
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_row_parallel_worker, args=(2, port, d), nprocs=2, join=True)
        ys = [np.load(os.path.join(d, "y%d.npy" % r)) for r in range(2)]
    r = np.random.default_rng(0)
    K = 96
    x = (r.standard_normal((12, K)) * np.where(np.arange(K) % 17 == 0, 30.0, 1.0)).astype(np.float32)
    inv = (r.random(K) + 0.5).astype(np.float32)
    qw = r.integers(-127, 128, (24, K)).astype(np.int8)
    sw = (r.random(24) * 0.01).astype(np.float32)
    q, sx = oracle.quant_act_per_token(x, inv)
    want = oracle.dequant(oracle.gemm_i8(q, qw), sx, sw, out="f32")
    for y in ys:
        np.testing.assert_array_equal(y, want)


# ------------------------------------------------- N-sharded SSZ and linear
def _sharded_inputs():
    import synthetic
    x, wt = synthetic.make_small(20, 96, 37, seed=5, w_outliers=4)  # N = 37: blocks of 19 and 18
    K = 96
    inv = (np.random.default_rng(6).random(K) + 0.5).astype(np.float32)
    s = (np.float32(1.0) / inv).astype(np.float32)
    return x, wt, s, inv


def _sharded_worker(rank, world, port, outdir):
    _init(rank, world, port)
    try:
        import oracle
        from w8a8_linear_layers_b200 import distributed as wdist
        x, wt, s, inv = _sharded_inputs()
        N, K = wt.shape
        ops = _OracleOps(oracle)
        # SSZ split by output channel, all-gathered
        q = torch.empty(N, K, dtype=torch.int8)
        sc = torch.empty(N)
        its = torch.empty(N, dtype=torch.int32)
        wdist.ssz_quant_weight_sharded(wt.float(), torch.from_numpy(s), 8, 20, q, sc, its, ops=ops)
        # column-parallel linear on this rank's block of the gathered weight
        a, b = wdist.shard_rows(N, world, rank)
        y_shard = torch.empty(x.shape[0], b - a, dtype=torch.bfloat16)
        y_full = torch.empty(x.shape[0], N, dtype=torch.bfloat16)
        wdist.column_parallel_linear(x.float(), torch.from_numpy(inv), q[a:b].contiguous(), sc[a:b].contiguous(),
                                     y_shard, y_full, ops=ops)
        np.savez(os.path.join(outdir, "rank%d.npz" % rank), q=q.numpy(), sc=sc.numpy(), its=its.numpy(),
                 y=y_full.view(torch.int16).numpy(), ys=y_shard.view(torch.int16).numpy(), a=a, b=b)
    finally:
        dist.destroy_process_group()


def test_shard_rows_cover_every_row_once():
    from w8a8_linear_layers_b200.distributed import shard_rows
    for n in (1, 7, 37, 4096, 11008):
        for g in (1, 2, 3, 8):
            blocks = [shard_rows(n, g, r) for r in range(g)]
            assert blocks[0][0] == 0 and blocks[-1][1] == n
            assert all(blocks[i][1] == blocks[i + 1][0] for i in range(g - 1))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1


def test_sharded_ssz_and_column_parallel_equal_unsharded():
    """SSZ split by output channel over 2 ranks and all-gathered equals the
    unsharded search (codes, scales, rounds bit for bit); the column-parallel
    linear's gathered output equals the unsharded linear's, and each rank's
    block equals its columns."""
    import oracle
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_sharded_worker, args=(2, _free_port(), d), nprocs=2, join=True)
        rs = [np.load(os.path.join(d, "rank%d.npz" % r)) for r in range(2)]
    x, wt, s, inv = _sharded_inputs()
    ref = oracle.ssz_quant_weight(wt.float().numpy(), bits=8, max_iters=20, s=s)
    qx, sx = oracle.quant_act_per_token(x.float().numpy(), inv)
    y_ref = oracle.dequant(oracle.gemm_i8(qx, ref["q"]), sx, ref["scale"]).view(np.int16)
    for r in rs:
        np.testing.assert_array_equal(r["q"], ref["q"])
        np.testing.assert_array_equal(r["sc"], ref["scale"])
        np.testing.assert_array_equal(r["its"], ref["iters"])
        np.testing.assert_array_equal(r["y"], y_ref)
        np.testing.assert_array_equal(r["ys"], y_ref[:, int(r["a"]):int(r["b"])])

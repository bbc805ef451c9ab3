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

"""Stream order with the per-inference kernels launched back to back: the
activation quantization and the GEMMs may be scheduled before their
predecessor finishes, but must wait for it before touching memory.  Here
every linear reuses ONE code/scale buffer and ONE output buffer chain, so
a kernel that started early would overwrite codes the previous GEMM still
reads, or read codes not yet written.  Eager launches and a CUDA-graph
capture of the same sequence must both give each linear's output exactly."""
import pytest
import torch

import synthetic
from tests.test_parity_gpu import w  # noqa: F401  (w: module fixture)

pytestmark = pytest.mark.gpu


def _layers(w, n, M, K, N, weights):
    out = []
    for i in range(n):
        x, wt = synthetic.make_small(M, K, N, seed=100 + i)
        lin = w.W8A8Linear(wt.cuda(), alpha=0.5, weights=weights)
        lin.calibrate(x.cuda())
        lin.quantize()
        out.append((lin, x.cuda()))
    return out


@pytest.mark.parametrize("weights", ["sym8", "int4"])
@pytest.mark.parametrize("M,K,N", [(4096, 1024, 1024), (16, 4096, 2048), (2000, 512, 768)])
def test_back_to_back_linears_share_buffers(w, M, K, N, weights):
    layers = _layers(w, 6, M, K, N, weights)
    refs = [lin.forward(x).clone() for lin, x in layers]
    qx = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sx = torch.empty(M, device="cuda")
    ys = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for _ in layers]

    def chain():
        for (lin, x), y in zip(layers, ys):
            w.quant_act_per_token(x, lin.inv_s, qx, sx)     # overwrites the codes the previous GEMM read
            lin._gemm(qx, sx, None, y)

    for y in ys:
        y.zero_()
    chain()
    torch.cuda.synchronize()
    for y, ref in zip(ys, refs):
        assert torch.equal(y, ref)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        chain()  # kernel attributes set outside the capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        chain()
    for rep in range(3):
        for y in ys:
            y.zero_()
        g.replay()
        torch.cuda.synchronize()
        for y, ref in zip(ys, refs):
            assert torch.equal(y, ref)
    del g

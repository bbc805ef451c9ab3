"""HostStreamer / W8A8Linear.forward_host: activations in pinned host memory,
the copies in and out overlapped with the kernels chunk by chunk.  Per-token
quantization and the GEMM treat rows independently, so the chunked output
must equal the resident forward's bit for bit, for every weight format and
for a ragged last chunk."""
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w():
    from tests.conftest import build_cuda_library
    build_cuda_library()
    import w8a8_linear_layers_b200 as w
    return w


@pytest.mark.parametrize("weights,M,K,N,chunk", [
    ("sym8", 1000, 512, 384, 256), ("int4", 777, 1024, 256, 300), ("asym8", 600, 256, 512, 128),
    ("sym8", 90, 4096, 1024, 2048),
])
def test_forward_host_equals_resident(w, weights, M, K, N, chunk):
    x, wt = synthetic.make_small(M, K, N, seed=M + K)
    lin = w.W8A8Linear(wt.cuda(), alpha=0.5, weights=weights)
    lin.calibrate(x.cuda())
    lin.quantize()
    y_dev = lin.forward(x.cuda())
    xh = x.pin_memory()
    yh = torch.empty(M, N, dtype=lin.out_dtype).pin_memory()
    lin.forward_host(xh, yh, chunk_rows=chunk)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(yh, y_dev.cpu())


def test_streamer_runs_several_jobs_through_shared_slots(w):
    """Two linears of different shapes through one streamer (two slots)."""
    layers, outs = [], []
    for i, (M, K, N) in enumerate(((513, 256, 128), (700, 512, 256))):
        x, wt = synthetic.make_small(M, K, N, seed=10 + i)
        lin = w.W8A8Linear(wt.cuda(), alpha=0.5)
        lin.calibrate(x.cuda())
        lin.quantize()
        layers.append((lin, x))
        outs.append(lin.forward(x.cuda()).cpu())
    st = w.HostStreamer("cuda", 200, 512, 256, torch.bfloat16, torch.bfloat16, slots=2)
    jobs, hosts = [], []
    for lin, x in layers:
        yh = torch.empty(x.shape[0], lin.N, dtype=torch.bfloat16).pin_memory()
        hosts.append(yh)
        jobs.append((x.pin_memory(), yh, lambda xc, qx, sx, yc, lin=lin: lin._forward_into(xc, qx, sx, None, yc)))
    st.run(jobs)
    torch.cuda.current_stream().synchronize()
    for yh, ref in zip(hosts, outs):
        assert torch.equal(yh, ref)

"""Linears over activations that live in pinned host memory, with the
host<->device copies overlapped with the computation.

The tokens of every job are cut into chunks of at most `chunk_rows` rows
that flow through three CUDA streams: the host->device copy of one chunk,
the per-inference kernels of the previous chunk (the job's function, on the
caller's stream) and the device->host copy of the one before run at once,
on the two copy engines and the SMs, through `slots` device buffers used in
rotation.  Per-token quantization and the GEMM treat rows independently, so
the chunked result equals the whole-batch one bit for bit.  Memory plumbing
only: the computation is the job's function (library calls).
"""
from __future__ import annotations

from typing import Callable, Iterable

import torch

# fn(x, qx, sx, y): the per-inference kernels of one chunk -- x [r, K] input
# rows on the device, qx [r, K] int8 and sx [r] fp32 scratch for the codes
# and scales, y [r, N] output rows -- enqueued on the current stream
ChunkFn = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor], None]


class HostStreamer:
    """Device buffers and copy streams for chunked host-resident linears
    (see the module docstring).  max_k / max_n: the largest K and N of the
    jobs it will run; x_dtype / y_dtype: their element types."""

    def __init__(self, device, chunk_rows: int, max_k: int, max_n: int, x_dtype: torch.dtype,
                 y_dtype: torch.dtype, slots: int = 3):
        if chunk_rows <= 0 or slots < 2:
            raise ValueError("chunk_rows must be positive and slots at least 2")
        self.device = torch.device(device)
        self.rows = chunk_rows
        self.max_k, self.max_n = max_k, max_n
        self.slots = [dict(x=torch.empty(chunk_rows * max_k, device=self.device, dtype=x_dtype),
                           qx=torch.empty(chunk_rows * max_k, device=self.device, dtype=torch.int8),
                           sx=torch.empty(chunk_rows, device=self.device, dtype=torch.float32),
                           y=torch.empty(chunk_rows * max_n, device=self.device, dtype=y_dtype))
                      for _ in range(slots)]
        self.s_in = torch.cuda.Stream(device=self.device)
        self.s_out = torch.cuda.Stream(device=self.device)

    def run(self, jobs: Iterable[tuple[torch.Tensor, torch.Tensor, ChunkFn]], stream=None) -> None:
        """Enqueue every job (x_host [M, K] pinned, y_host [M, N] pinned, fn):
        y_host receives fn applied to x_host, chunk by chunk.  Returns once
        everything is enqueued; `stream` (default: the current one) waits for
        the last copy, so an event recorded on it afterwards marks the end."""
        stream = stream or torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(stream)
        self.s_in.wait_event(start)
        self.s_out.wait_event(start)
        n_slots = len(self.slots)
        x_free = [None] * n_slots  # per slot: the compute that last read its x and codes
        y_free = [None] * n_slots  # per slot: the copy that last read its y
        k = 0
        for x_host, y_host, fn in jobs:
            M, K = x_host.shape
            N = y_host.shape[1]
            if K > self.max_k or N > self.max_n or y_host.shape[0] != M:
                raise ValueError("job shape (%d, %d) -> %d outside this streamer's buffers" % (M, K, N))
            for r0 in range(0, M, self.rows):
                r = min(self.rows, M - r0)
                si = k % n_slots
                sl = self.slots[si]
                x = sl["x"][: r * K].view(r, K)
                y = sl["y"][: r * N].view(r, N)
                with torch.cuda.stream(self.s_in):
                    if x_free[si] is not None:
                        self.s_in.wait_event(x_free[si])
                    x.copy_(x_host[r0:r0 + r], non_blocking=True)
                    ev_in = torch.cuda.Event()
                    ev_in.record(self.s_in)
                stream.wait_event(ev_in)
                if y_free[si] is not None:
                    stream.wait_event(y_free[si])
                with torch.cuda.stream(stream):
                    fn(x, sl["qx"][: r * K].view(r, K), sl["sx"][:r], y)
                ev_c = torch.cuda.Event()
                ev_c.record(stream)
                x_free[si] = ev_c
                with torch.cuda.stream(self.s_out):
                    self.s_out.wait_event(ev_c)
                    y_host[r0:r0 + r].copy_(y, non_blocking=True)
                    ev_o = torch.cuda.Event()
                    ev_o.record(self.s_out)
                y_free[si] = ev_o
                k += 1
        stream.wait_stream(self.s_out)

"""Seeded synthetic inputs for the W8A8 linear path.

This module holds no arithmetic of the method: it only draws the inputs
(LLM-shaped activations with outlier channels, small-std weights), so that the
CUDA path, the CPU oracle, the tests and the benchmark all see the same data.
It imports neither the CUDA package nor the oracle.

Recipe (every config, torch CPU generator with the given seed, default 0):
draw in fp32 and in this order -- X = randn(M, K); the X outlier channels
randperm(K)[:n_x] whose whole columns are multiplied by the outlier factor;
W = randn(N, K) * std; for configs with weight outliers, randperm(N*K)[:n_w]
individual weights multiplied by 10 -- then cast to the config's input dtype
(bf16 with round-to-nearest-even).

The pages measure on whole models and datasets (ResNet50/BERT-base on a T4,
GPT-345M on LAMBADA); those are not available, and these synthetic linears of
the same shapes stand in for them.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LinearConfig:
    name: str
    M: int          # tokens
    K: int          # input channels
    N: int          # output channels
    in_dtype: str   # "f32" | "bf16"
    out_dtype: str  # "f32" | "bf16"
    alpha: float
    x_outliers: int         # number of outlier input channels
    x_outlier_scale: float
    w_std: float
    w_outliers: int = 0     # number of individual outlier weights (x10)
    bits: int = 8
    max_iters: int = 20


def _r(x: float) -> int:
    return int(round(x))


# The four single-linear workloads (sizes from the workload list the build
# follows; outlier counts are round(fraction * channels)).
CONFIGS = {
    "single_linear_16x256x128": LinearConfig(
        "single_linear_16x256x128", 16, 256, 128, "f32", "f32", 0.5, 4, 50.0, 0.02),
    "prefill_2048x4096x4096": LinearConfig(
        "prefill_2048x4096x4096", 2048, 4096, 4096, "bf16", "bf16", 0.5,
        _r(0.01 * 4096), 40.0, 0.02),
    "mlp_up_8192x4096x11008": LinearConfig(
        "mlp_up_8192x4096x11008", 8192, 4096, 11008, "bf16", "bf16", 0.8,
        _r(0.01 * 4096), 60.0, 0.02, w_outliers=_r(0.001 * 11008 * 4096)),
    "decode_16x8192x28672": LinearConfig(
        "decode_16x8192x28672", 16, 8192, 28672, "bf16", "bf16", 0.5,
        _r(0.005 * 8192), 50.0, 0.015, bits=4),
}
ORDER = list(CONFIGS)


def make_linear(cfg: LinearConfig | str, seed: int = 0, M: int | None = None):
    """Draw (x, w) for a config on the CPU.  M overrides the token count (the
    draw order is unchanged, so a smaller M is not a prefix of the full X)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    M = cfg.M if M is None else M
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, cfg.K, generator=g, dtype=torch.float32)
    if cfg.x_outliers:
        idx = torch.randperm(cfg.K, generator=g)[: cfg.x_outliers]
        x[:, idx] *= cfg.x_outlier_scale
    w = torch.randn(cfg.N, cfg.K, generator=g, dtype=torch.float32) * cfg.w_std
    if cfg.w_outliers:
        widx = torch.randperm(cfg.N * cfg.K, generator=g)[: cfg.w_outliers]
        w.view(-1)[widx] *= 10.0
    if cfg.in_dtype == "bf16":
        x = x.to(torch.bfloat16)
        w = w.to(torch.bfloat16)
    return x, w


def make_small(M: int, K: int, N: int, seed: int = 0, in_dtype: str = "bf16",
               x_outliers: int = 2, x_outlier_scale: float = 40.0, w_std: float = 0.02,
               w_outliers: int = 0):
    """A small LLM-shaped linear (same recipe) for ragged-shape parity cases."""
    cfg = LinearConfig("small", M, K, N, in_dtype, in_dtype, 0.5, min(x_outliers, K),
                       x_outlier_scale, w_std, w_outliers=w_outliers)
    return make_linear(cfg, seed)


def flush_buffer(device, nbytes: int = 512 << 20) -> torch.Tensor:
    """A buffer larger than the 126 MB L2, written between timed iterations."""
    return torch.empty(nbytes, dtype=torch.uint8, device=device)

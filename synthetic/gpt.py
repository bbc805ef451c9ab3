"""GPT-345M-shaped activations for the W8A8 linears (input synthesis only).

A random-init decoder (24 layers, hidden 1024, 16 heads, FFN 4096, vocab
50304, learned positions up to 1024; weights N(0, 0.02), biases 0, LayerNorm
gamma 1 / beta 0, GELU, causal attention) runs one bf16 forward over a batch
of 8 x 1024 uniform token ids and records the input of every linear layer:
per layer QKV (fused [3072 x 1024]), proj [1024 x 1024], fc1 [4096 x 1024],
fc2 [1024 x 4096] -- 96 linears.  This is plain PyTorch used to produce
realistic inputs for the path under test; it holds none of the method's
arithmetic.  Trained weights and the evaluation data the pages use
(GPT-345M on LAMBADA) are not available here; this stands in for them.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as F

LAYERS, HIDDEN, HEADS, FFN, VOCAB, MAXPOS = 24, 1024, 16, 4096, 50304, 1024
BATCH, SEQ = 8, 1024
LINEARS = ("qkv", "proj", "fc1", "fc2")
SHAPES = {"qkv": (3 * HIDDEN, HIDDEN), "proj": (HIDDEN, HIDDEN), "fc1": (FFN, HIDDEN), "fc2": (HIDDEN, FFN)}


def make_weights(seed: int = 0, device="cpu", dtype=torch.bfloat16):
    """Random-init weights: {(layer, name): W [N, K]} plus embeddings."""
    g = torch.Generator().manual_seed(seed)
    w = {"wte": (torch.randn(VOCAB, HIDDEN, generator=g) * 0.02).to(device, dtype),
         "wpe": (torch.randn(MAXPOS, HIDDEN, generator=g) * 0.02).to(device, dtype)}
    for layer in range(LAYERS):
        for name in LINEARS:
            N, K = SHAPES[name]
            w[(layer, name)] = (torch.randn(N, K, generator=g) * 0.02).to(device, dtype)
    return w


def make_tokens(seed: int = 0, batch: int = BATCH, seq: int = SEQ):
    g = torch.Generator().manual_seed(seed + 1)
    return torch.randint(0, VOCAB, (batch, seq), generator=g)


@torch.no_grad()
def forward(weights, tokens, linear=None, capture=None, layers=LAYERS):
    """bf16 forward.  `linear(layer, name, x2d, W)` computes each linear
    (default x W^T); `capture` (dict) receives every linear's input [B*T, K];
    `layers` < 24 stops after that many layers (input synthesis for a sample)."""
    dev = weights["wte"].device
    B, T = tokens.shape
    x = weights["wte"][tokens.to(dev)] + weights["wpe"][:T][None]
    lin = linear or (lambda layer, name, a, W: a @ W.t())

    def run(layer, name, a):
        a2 = a.reshape(-1, a.shape[-1]).contiguous()
        if capture is not None:
            capture[(layer, name)] = a2
        return lin(layer, name, a2, weights[(layer, name)]).reshape(*a.shape[:-1], -1)

    for layer in range(layers):
        h = F.layer_norm(x, (HIDDEN,))
        qkv = run(layer, "qkv", h)
        q, k, v = qkv.split(HIDDEN, dim=-1)
        hd = HIDDEN // HEADS
        q, k, v = (t.reshape(B, T, HEADS, hd).transpose(1, 2) for t in (q, k, v))
        att = F.scaled_dot_product_attention(q, k, v, is_causal=True)
        att = att.transpose(1, 2).reshape(B, T, HIDDEN)
        x = x + run(layer, "proj", att)
        h = F.layer_norm(x, (HIDDEN,))
        x = x + run(layer, "fc2", F.gelu(run(layer, "fc1", h)))
    return F.layer_norm(x, (HIDDEN,))


def linear_inputs(seed: int = 0, device="cuda"):
    """(weights, {(layer, name): X [8192, K] bf16}) on `device`."""
    w = make_weights(seed, device)
    cap = {}
    forward(w, make_tokens(seed), capture=cap)
    return w, cap


def flops_per_pass() -> float:
    """2 M N K summed over the 96 linears for one batch."""
    M = BATCH * SEQ
    return float(sum(2 * M * N * K for (N, K) in SHAPES.values()) * LAYERS)


assert math.isclose(flops_per_pass(), 2 * 8192 * 24 * (3072 * 1024 + 1024 * 1024 + 4096 * 1024 + 1024 * 4096))

"""Seeded synthetic inputs shared by the CUDA path (tests, bench, smoke) and the oracle's
tests.

This module holds random draws only -- no routing or attention arithmetic -- so that
both sides of a parity check see bit-identical inputs without sharing any of the
method.  Distributions follow the workloads: Q, K, V and the router input x_Q are
N(0, 1) rounded to bf16, router weights N(0, 0.02) in bf16 with zero biases, and fixed
FA/SA layer masks come from a seeded permutation of the layers.

All draws use torch's default CPU generator (``torch.Generator``) with an
explicit seed per tensor and a fixed chunk size, so a tensor is the same on every
machine that runs the same torch build.
"""

from __future__ import annotations

import torch

_CHUNK = 1 << 24  # elements per draw; part of the definition of every tensor below


def normal_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """CPU bf16 tensor of N(0, std^2) draws, seeded, drawn in fixed-size chunks."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    numel = 1
    for s in shape:
        numel *= int(s)
    out = torch.empty(numel, dtype=torch.bfloat16)
    for start in range(0, numel, _CHUNK):
        n = min(_CHUNK, numel - start)
        x = torch.randn(n, generator=gen, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[start:start + n] = x.to(torch.bfloat16)
    return out.view(*[int(s) for s in shape])


def layer_seed(base: int, layer: int, which: int) -> int:
    """Distinct seed per (workload, layer, tensor kind)."""
    return int(base) * 1_000_003 + int(layer) * 101 + int(which)


# tensor kinds for layer_seed
Q, K, V, K_NEW, V_NEW, Q_DECODE, XQ = 1, 2, 3, 4, 5, 6, 7


def router_weights(hidden: int, rank: int, n_layers: int, seed: int):
    """Layer-router parameters in the (out, in) convention: W1 [rank][hidden],
    b1 [rank], W2 [n_layers][rank], b2 [n_layers].  Weights N(0, 0.02), biases 0."""
    w1 = normal_bf16((rank, hidden), seed * 7 + 1, std=0.02)
    w2 = normal_bf16((n_layers, rank), seed * 7 + 2, std=0.02)
    b1 = torch.zeros(rank, dtype=torch.bfloat16)
    b2 = torch.zeros(n_layers, dtype=torch.bfloat16)
    return w1, b1, w2, b2


def fixed_sa_layers(n_layers: int, n_sa: int, seed: int) -> list:
    """Indices of the layers routed to SA in a fixed mask: the first n_sa entries of a
    seeded permutation of the layers."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    perm = torch.randperm(n_layers, generator=gen)
    return sorted(int(x) for x in perm[:n_sa])


def fa_bits_from_sa_layers(batch: int, n_layers: int, sa_layers) -> torch.Tensor:
    """[batch][n_layers] bool, True = FA, the same for every sequence."""
    bits = torch.ones(batch, n_layers, dtype=torch.bool)
    for layer in sa_layers:
        bits[:, layer] = False
    return bits


def pack_bits_u32(bits: torch.Tensor) -> torch.Tensor:
    """Pack [B][n_layers] bools into int32 words laid out as the uint32 mask the
    library reads (bit l % 32 of word l // 32).  A fixed mask is an input, so the
    packing lives with the inputs."""
    batch, n_layers = bits.shape
    n_words = (n_layers + 31) // 32
    words = [[0] * n_words for _ in range(batch)]
    for b in range(batch):
        for layer in range(n_layers):
            if bool(bits[b, layer]):
                words[b][layer // 32] |= 1 << (layer % 32)
    # reinterpret as signed int32 for torch storage
    flat = [w - (1 << 32) if w >= (1 << 31) else w for row in words for w in row]
    return torch.tensor(flat, dtype=torch.int32).view(batch, n_words)


def random_seq_lens(batch: int, low: int, high: int, seed: int) -> torch.Tensor:
    """Seeded ragged lengths in [low, high]."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    return torch.randint(low, high + 1, (batch,), generator=gen, dtype=torch.int64)

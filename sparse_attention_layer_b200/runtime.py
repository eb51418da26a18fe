"""Per-model state of the hybrid-attention hot path: one contiguous bf16 KV cache per
layer ([B][Hkv][cap][d] for K and V, plus int32 seq_len[B]), the device-side FA/SA
mask written by the router at prefill and reused by every decode step, and the
decode workspace.  PyTorch only allocates the memory; every step runs in libflux.
"""

from __future__ import annotations

import torch

from . import flux
from .flux import AttnCfg


class LayerCache:
    def __init__(self, cfg: AttnCfg, batch: int, capacity: int, device):
        shape = (batch, cfg.n_kv_heads, capacity, cfg.head_dim)
        self.k = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.v = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.seq_len = torch.zeros(batch, dtype=torch.int32, device=device)

    def reset(self, lengths=None):
        if lengths is None:
            self.seq_len.zero_()
        else:
            self.seq_len.copy_(torch.as_tensor(lengths, dtype=torch.int32))


class HybridAttention:
    """Router + per-layer FA/SA attention over per-layer KV caches."""

    def __init__(self, cfg: AttnCfg, batch: int, capacity: int, device="cuda", layers=None):
        self.cfg = cfg
        self.batch = batch
        self.capacity = capacity
        self.device = torch.device(device)
        n = cfg.n_layers if layers is None else layers
        self.caches = [LayerCache(cfg, batch, capacity, self.device) for _ in range(n)]
        self.fa_mask = torch.zeros(batch, cfg.mask_words, dtype=torch.int32, device=self.device)
        self.workspace = torch.empty(flux.flux_decode_workspace_size(cfg, batch),
                                     dtype=torch.uint8, device=self.device)

    def route(self, w1, b1, w2, b2, xq, pool_len: int = 100, tau: float = 0.0, logits=None):
        flux.flux_route(w1, b1, w2, b2, xq, pool_len, tau, self.fa_mask, logits)

    def set_mask(self, packed_words: torch.Tensor):
        self.fa_mask.copy_(packed_words)

    def prefill_layer(self, layer: int, q, k_new, v_new, out, cache_index=None):
        c = self.caches[layer if cache_index is None else cache_index]
        flux.flux_kv_append(self.cfg, c.k, c.v, c.seq_len, k_new, v_new)
        flux.flux_prefill(self.cfg, layer, self.fa_mask, q, c.k, c.v, c.seq_len, out)

    def decode_layer(self, layer: int, q, k_new, v_new, out, cache_index=None):
        c = self.caches[layer if cache_index is None else cache_index]
        flux.flux_kv_append(self.cfg, c.k, c.v, c.seq_len, k_new, v_new)
        flux.flux_decode(self.cfg, layer, self.fa_mask, q, c.k, c.v, c.seq_len, out,
                         self.workspace)

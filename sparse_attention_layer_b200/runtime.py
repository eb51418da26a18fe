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


class RingCache:
    """An SA layer's decode-time cache after eviction: sink rows plus a ring of
    ring_rows recent rows ([B][Hkv][sink + ring_rows][d]); seq_len counts positions."""

    def __init__(self, cfg: AttnCfg, batch: int, ring_rows: int, device):
        shape = (batch, cfg.n_kv_heads, cfg.sink + ring_rows, cfg.head_dim)
        self.k = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.v = torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.seq_len = torch.zeros(batch, dtype=torch.int32, device=device)
        self.ring_rows = ring_rows

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
        self.workspace = flux.new_decode_workspace(cfg, batch, self.device)

    def route(self, w1, b1, w2, b2, xq, pool_len: int = 100, tau: float = 0.0, logits=None):
        flux.flux_route(w1, b1, w2, b2, xq, pool_len, tau, self.fa_mask, logits)

    def set_mask(self, packed_words: torch.Tensor):
        self.fa_mask.copy_(packed_words)

    def prefill_layer(self, layer: int, q, k_new, v_new, out, cache_index=None):
        c = self.caches[layer if cache_index is None else cache_index]
        flux.flux_kv_append(self.cfg, c.k, c.v, c.seq_len, k_new, v_new)
        flux.flux_prefill(self.cfg, layer, self.fa_mask, q, c.k, c.v, c.seq_len, out)

    def prefill_layer_chunked(self, layer: int, q, k_new, v_new, out, chunk: int = 16384):
        """Prefill a long prompt in chunks of `chunk` tokens (Table 6 of the paper page
        runs its SA kernel with chunk 16384): each chunk appends its K/V rows, then its
        queries attend everything before them.  With chunk a multiple of 128 the
        result equals a one-shot prefill bit for bit (same tiles, same order).
        q/out [B][S][Hq][d], k_new/v_new [B][S][Hkv][d]."""
        c = self.caches[layer]
        seq = q.shape[1]
        for c0 in range(0, seq, chunk):
            c1 = min(seq, c0 + chunk)
            qc = q[:, c0:c1].contiguous()
            oc = out[:, c0:c1] if q.shape[0] == 1 else torch.empty_like(qc)
            flux.flux_kv_append(self.cfg, c.k, c.v, c.seq_len, k_new[:, c0:c1].contiguous(),
                                v_new[:, c0:c1].contiguous())
            flux.flux_prefill(self.cfg, layer, self.fa_mask, qc, c.k, c.v, c.seq_len, oc)
            if q.shape[0] != 1:
                out[:, c0:c1].copy_(oc)

    def decode_layer(self, layer: int, q, k_new, v_new, out, cache_index=None):
        """One decode step of one layer: append the new K/V row and attend, one launch."""
        c = self.caches[layer if cache_index is None else cache_index]
        if isinstance(c, RingCache):
            flux.flux_decode_append_ring(self.cfg, layer, self.fa_mask, q, k_new, v_new, c.k,
                                         c.v, c.seq_len, out, self.workspace)
            return
        flux.flux_decode_append(self.cfg, layer, self.fa_mask, q, k_new, v_new, c.k, c.v,
                                c.seq_len, out, self.workspace)

    def sa_layers(self) -> list:
        """Layers every sequence routes to SA (reads the mask once, after routing:
        routing is decided at prefill and reused by every decode step)."""
        words = self.fa_mask.cpu()
        out = []
        for layer in range(self.cfg.n_layers):
            bits = [(int(words[b, layer // 32]) >> (layer % 32)) & 1 for b in range(self.batch)]
            if not any(bits):
                out.append(layer)
        return out

    def evict_sa_layers(self, ring_rows: int = 0) -> int:
        """After prefill: move the cache of every all-SA layer into a ring cache of
        sink + ring_rows rows (ring_rows defaults to the window) and free the full
        cache.  Returns the bytes of KV cache freed."""
        ring_rows = ring_rows or self.cfg.window
        freed = 0
        for layer in self.sa_layers():
            full = self.caches[layer]
            if isinstance(full, RingCache):
                continue
            ring = RingCache(self.cfg, self.batch, ring_rows, self.device)
            flux.flux_kv_compact_ring(self.cfg, full.k, full.v, full.seq_len, ring.k, ring.v)
            ring.seq_len.copy_(full.seq_len)
            freed += (full.k.numel() + full.v.numel() - ring.k.numel() - ring.v.numel()) * 2
            self.caches[layer] = ring
        return freed

    def kv_bytes(self) -> int:
        """Bytes of KV cache currently held (K and V of every layer)."""
        return sum((c.k.numel() + c.v.numel()) * 2 for c in self.caches)


class DecodeStepGraph:
    """One decode step over every layer (KV append + FA/SA decode per layer) captured in
    a CUDA graph and replayed once per generated token.

    Capture is possible because no call allocates, synchronises or reads device state
    on the host: routes come from the device-side mask and lengths from seq_len, which
    the captured appends advance on every replay.  q, k_new, v_new and o are the
    static input/output buffers ([L][B][Hq][d], [L][B][1][Hkv][d] twice, [L][B][Hq][d]);
    refill them in place between replays.  Run one eager step first (per-device
    one-time set-up of the library happens outside the capture).
    """

    def __init__(self, model: HybridAttention, q, k_new, v_new, o):
        self.buffers = (q, k_new, v_new, o)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            for layer in range(len(model.caches)):
                model.decode_layer(layer, q[layer], k_new[layer], v_new[layer], o[layer])

    def replay(self):
        self.graph.replay()

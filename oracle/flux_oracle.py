"""FP64 CPU oracle for the Flux Attention hot path (router, KV append, FA/SA attention).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run this
module.  The product package ``sparse_attention_layer_b200`` never imports it and has
no CPU fallback: without its CUDA library it raises.

Everything here is the plain definition, in float64, on arrays that hold the exact
bf16 input values.  Nothing is blocked, fused, split or reordered beyond what each
definition states; library primitives (a matmul, a mean, an exp) serve as steps.

Sources (all pages are about "Flux Attention: Context-Aware Hybrid Attention for
Efficient LLMs Inference", arXiv 2604.07394):

* Figure 2 caption: a Layer Router reads the query hidden states x_Q and sends every
  layer to Full Attention (FA) or Sparse Attention (SA).
* Figure 8 caption: the router pools only a truncated window of L tokens taken at
  the two sequence boundaries (prefix and suffix); L = 100 works best, "Full" is the
  untruncated alternative.
* Table 19 caption: the router produces a soft FA probability per layer, which is
  made a hard FA/SA choice at inference.
* Table 3 (Flux Attention row): routing is decided at prefill and reused for decode.
* Table 6 and Figure 1 caption: SA is streaming attention -- attention-sink tokens
  plus a local window -- run by a block-sparse kernel (block 64, sink 128).
* Tables 15/16: the model sparsity ratio Omega_MSR is the fraction of layers on SA.

Readings taken where the pages are silent:

* SA visibility is block-granular: key block jb is visible from query position t
  (query block qb = t // block) iff jb < sink/block or jb >= qb - window/block + 1,
  always with causality j <= t.  Sink and window are one set union.
* Router: mean-pool over the boundary tokens (first ceil(L/2), last floor(L/2); all
  tokens when L = 0 or S <= L), then Linear(h->r), ReLU, Linear(r->n_layers).
  Weights are stored in the (out, in) convention of a linear layer.
* Hard decision: FA iff logit > tau (strict; ties go to SA), i.e. sigmoid(z) > 1/2
  for tau = 0.  Bit l of the packed mask word l // 32 is 1 for FA.
* Attention: softmax(q k^T / sqrt(d)) v over the visible keys, no bias, no cap;
  query head h reads KV head h // (Hq / Hkv) (grouped-query sharing).
* Prefill queries are the last n_q positions of the cache; a decode step is the
  prefill row at t = seq_len - 1 after the new token has been appended.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
against closed forms, a library attention routine, hand-derived golden values under
``tests/golden/`` and invariants; none is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------------------
# Router (Figure 2, Figure 8, Table 19 caption)
# --------------------------------------------------------------------------------------


def pool_token_indices(seq_len: int, pool_len: int) -> np.ndarray:
    """Token positions the router averages over.

    Figure 8 (pooling window size): only L boundary tokens are kept, split between the
    prefix and the suffix of the sequence.  pool_len <= 0 means "Full" (every token);
    a sequence no longer than L is pooled whole.
    """
    if pool_len <= 0 or seq_len <= pool_len:
        return np.arange(seq_len, dtype=np.int64)
    n_prefix = (pool_len + 1) // 2
    n_suffix = pool_len // 2
    return np.concatenate(
        [np.arange(n_prefix, dtype=np.int64),
         np.arange(seq_len - n_suffix, seq_len, dtype=np.int64)])


def router_pool(xq: np.ndarray, pool_len: int) -> np.ndarray:
    """Mean of x_Q over the boundary tokens.  xq: [B][S][h] -> [B][h]."""
    idx = pool_token_indices(xq.shape[1], pool_len)
    return xq[:, idx, :].mean(axis=1)


def router_logits(pooled: np.ndarray, w1: np.ndarray, b1: np.ndarray,
                  w2: np.ndarray, b2: np.ndarray) -> np.ndarray:
    """Two-layer MLP of the Layer Router (Figure 2): z = W2 relu(W1 p + b1) + b2.

    w1: [r][h], b1: [r], w2: [n_layers][r], b2: [n_layers]; pooled: [B][h].
    Returns the per-layer FA logits z: [B][n_layers].
    """
    hidden = np.maximum(pooled @ w1.T + b1, 0.0)
    return hidden @ w2.T + b2


def router_fa_bits(logits: np.ndarray, tau: float) -> np.ndarray:
    """Hard FA/SA decision per layer (Table 19 caption's soft FA probability made
    binary): True = FA iff z > tau."""
    return logits > tau


def pack_fa_mask(fa_bits: np.ndarray) -> np.ndarray:
    """Pack [B][n_layers] booleans into uint32 words: bit (l % 32) of word l // 32."""
    batch, n_layers = fa_bits.shape
    n_words = (n_layers + 31) // 32
    out = np.zeros((batch, n_words), dtype=np.uint32)
    for b in range(batch):
        for layer in range(n_layers):
            if fa_bits[b, layer]:
                out[b, layer // 32] |= np.uint32(1) << np.uint32(layer % 32)
    return out


def omega_msr(fa_bits: np.ndarray) -> np.ndarray:
    """Model sparsity ratio (Tables 15/16): fraction of layers routed to SA."""
    n_layers = fa_bits.shape[-1]
    return 1.0 - fa_bits.sum(axis=-1) / n_layers


def router(xq, w1, b1, w2, b2, pool_len: int, tau: float):
    """Whole router: pooled input, logits, FA bits and the packed mask."""
    pooled = router_pool(xq, pool_len)
    logits = router_logits(pooled, w1, b1, w2, b2)
    bits = router_fa_bits(logits, tau)
    return {"pooled": pooled, "logits": logits, "fa_bits": bits,
            "fa_mask": pack_fa_mask(bits)}


def router_error_bound(xq, w1, b1, w2, b2, pool_len: int,
                       unit_roundoff: float = 2.0 ** -53) -> np.ndarray:
    """Worst-case |z_computed - z_exact| for any evaluation order of the router in a
    floating-point format with the given unit roundoff (2^-53: fp64, 2^-24: fp32).

    Standard forward error bounds for sums and dot products (gamma_n = n u / (1 - n u)),
    carried through the mean, the first layer, the 1-Lipschitz ReLU and the second
    layer.  A logit whose distance to tau exceeds this bound has a hard decision that
    no implementation in that format can flip.  Returns [B][n_layers].
    """
    u = unit_roundoff

    def gamma(n):
        return n * u / (1.0 - n * u)

    idx = pool_token_indices(xq.shape[1], pool_len)
    n = len(idx)
    absx = np.abs(xq[:, idx, :]).sum(axis=1) / n
    pooled = xq[:, idx, :].mean(axis=1)
    e_pool = gamma(n + 2) * absx
    h = w1.shape[1]
    pre = pooled @ w1.T + b1
    abs_terms1 = (np.abs(pooled) + e_pool) @ np.abs(w1).T + np.abs(b1)
    e_pre = gamma(h + 1) * abs_terms1 + e_pool @ np.abs(w1).T
    hidden = np.maximum(pre, 0.0)
    r = w2.shape[1]
    abs_terms2 = (np.abs(hidden) + e_pre) @ np.abs(w2).T + np.abs(b2)
    return gamma(r + 1) * abs_terms2 + e_pre @ np.abs(w2).T


# --------------------------------------------------------------------------------------
# Visibility masks (Table 6: streaming SA with sink + local window in KV blocks)
# --------------------------------------------------------------------------------------


def fa_key_visible(t, j):
    """Causal full attention: key j is visible from query position t iff j <= t."""
    return j <= t


def sa_key_visible(t, j, block: int, sink: int, window: int):
    """Streaming SA visibility, block-granular reading.

    The first sink/block key blocks (attention sinks) and the window/block key blocks
    ending at the query's own block stay visible; causality applies inside.
    """
    n_sink = sink // block
    n_win = window // block
    qb = t // block
    jb = j // block
    return (j <= t) & ((jb < n_sink) | (jb >= qb - n_win + 1))


def sa_key_visible_token_granular(t, j, sink: int, window: int):
    """Alternative token-granular reading, kept only to bound the difference:
    j < sink or t - j < window, with causality."""
    return (j <= t) & ((j < sink) | (t - j < window))


def visible_mask(is_fa: bool, q_pos: np.ndarray, n_keys: int, block: int,
                 sink: int, window: int) -> np.ndarray:
    """Dense boolean mask [len(q_pos)][n_keys] for one layer's route."""
    t = np.asarray(q_pos, dtype=np.int64)[:, None]
    j = np.arange(n_keys, dtype=np.int64)[None, :]
    if is_fa:
        return fa_key_visible(t, j)
    return sa_key_visible(t, j, block, sink, window)


def sa_visible_key_blocks(qb: int, n_key_blocks: int, block: int, sink: int,
                          window: int) -> set:
    """Key blocks holding at least one key visible from some query of query block qb,
    found by testing every (query, key) pair of the two blocks against the mask."""
    out = set()
    t = np.arange(qb * block, (qb + 1) * block, dtype=np.int64)[:, None]
    for jb in range(n_key_blocks):
        j = np.arange(jb * block, (jb + 1) * block, dtype=np.int64)[None, :]
        if sa_key_visible(t, j, block, sink, window).any():
            out.add(jb)
    return out


def key_tiles_of_rows(is_fa: bool, q_pos: np.ndarray, tile: int, block: int, sink: int,
                      window: int):
    """Key tiles of `tile` keys that a block-sparse kernel must visit for the query rows
    q_pos taken together, from the dense mask: the tiles holding a key visible from at
    least one row, and, of those, the tiles where some (row, key) pair is not visible
    (the kernel has to mask inside them).  Returns (visited, masked) as sorted lists."""
    q_pos = np.asarray(q_pos, dtype=np.int64)
    n_tiles = int(q_pos.max()) // tile + 1
    mask = visible_mask(is_fa, q_pos, n_tiles * tile, block, sink, window)
    per_tile = mask.reshape(len(q_pos), n_tiles, tile)
    visited = [kt for kt in range(n_tiles) if per_tile[:, kt, :].any()]
    masked = [kt for kt in visited if not per_tile[:, kt, :].all()]
    return visited, masked


# --------------------------------------------------------------------------------------
# Attention (Table 6: FA dense path and SA streaming path; grouped-query KV sharing)
# --------------------------------------------------------------------------------------


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray,
                     return_probs: bool = False):
    """softmax(q k^T / sqrt(d) restricted to mask) v for one head.

    q: [n_q][d], k, v: [n_keys][d], mask: [n_q][n_keys] (every row has a visible key).
    """
    d = q.shape[1]
    scores = (q @ k.T) / math.sqrt(d)
    scores = np.where(mask, scores, -np.inf)
    row_max = scores.max(axis=1, keepdims=True)
    weights = np.where(mask, np.exp(scores - row_max), 0.0)
    probs = weights / weights.sum(axis=1, keepdims=True)
    out = probs @ v
    if return_probs:
        return out, probs
    return out


def attention_layer(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                    seq_len: np.ndarray, is_fa: np.ndarray, block: int, sink: int,
                    window: int, rows=None, heads=None) -> np.ndarray:
    """One layer of hybrid attention over a per-layer KV cache.

    q: [B][n_q][Hq][d] (queries are the last n_q positions, t = seq_len[b] - n_q + i)
    k_cache, v_cache: [B][Hkv][cap][d]; seq_len: [B]; is_fa: [B] route bit of this
    layer (Table 3: one choice per layer, decided at prefill).
    rows / heads restrict the output to sampled query rows / query heads; the
    result is [B][len(rows)][len(heads)][d].
    """
    batch, n_q, n_qh, d = q.shape
    n_kvh = k_cache.shape[1]
    group = n_qh // n_kvh
    rows = np.arange(n_q) if rows is None else np.asarray(rows)
    heads = np.arange(n_qh) if heads is None else np.asarray(heads)
    out = np.zeros((batch, len(rows), len(heads), d), dtype=np.float64)
    for b in range(batch):
        n_keys = int(seq_len[b])
        q_pos = n_keys - n_q + rows
        mask = visible_mask(bool(is_fa[b]), q_pos, n_keys, block, sink, window)
        for hi, h in enumerate(heads):
            kvh = h // group
            out[b, :, hi, :] = masked_attention(
                q[b, rows, h, :], k_cache[b, kvh, :n_keys, :],
                v_cache[b, kvh, :n_keys, :], mask)
    return out


def decode_attention(q: np.ndarray, k_cache, v_cache, seq_len, is_fa, block, sink,
                     window, heads=None) -> np.ndarray:
    """One decode step (Table 3: decode reuses the prefill route).  The new token's
    K/V is already in the cache, so its position is seq_len - 1.  q: [B][Hq][d]."""
    out = attention_layer(q[:, None], k_cache, v_cache, seq_len, is_fa, block, sink,
                          window, heads=heads)
    return out[:, 0]


# --------------------------------------------------------------------------------------
# KV cache append (contiguous per-layer cache [B][Hkv][cap][d])
# --------------------------------------------------------------------------------------


def kv_append(k_cache: np.ndarray, v_cache: np.ndarray, seq_len: np.ndarray,
              k_new: np.ndarray, v_new: np.ndarray):
    """Write n new rows per sequence at positions [seq_len, seq_len + n) and advance
    seq_len.  k_new, v_new: [B][n][Hkv][d].  A sequence whose rows would pass the
    capacity is left untouched and reported in the returned overflow flags."""
    k_out = k_cache.copy()
    v_out = v_cache.copy()
    len_out = np.array(seq_len, dtype=np.int64).copy()
    cap = k_cache.shape[2]
    n_new = k_new.shape[1]
    overflow = np.zeros(len(len_out), dtype=bool)
    for b in range(len(len_out)):
        start = int(len_out[b])
        if start + n_new > cap:
            overflow[b] = True
            continue
        for i in range(n_new):
            k_out[b, :, start + i, :] = k_new[b, i]
            v_out[b, :, start + i, :] = v_new[b, i]
        len_out[b] = start + n_new
    return k_out, v_out, len_out, overflow


# --------------------------------------------------------------------------------------
# SA-layer KV eviction: sink rows plus a ring of recent rows (Tables 15/16 report the
# persistent decode-time KV saving of layers routed to SA)
# --------------------------------------------------------------------------------------


def ring_slot(p, sink: int, ring_rows: int):
    """Physical row of logical position p in an SA ring cache of sink + ring_rows rows:
    sink positions stay in place, later positions cycle through the ring."""
    p = np.asarray(p, dtype=np.int64)
    return np.where(p < sink, p, sink + (p - sink) % ring_rows)


def ring_retained_positions(seq_len: int, sink: int, ring_rows: int) -> np.ndarray:
    """Logical positions an SA ring cache holds after seq_len rows were written: the sink
    rows and the last ring_rows positions past the sink."""
    head = np.arange(min(sink, seq_len), dtype=np.int64)
    tail = np.arange(max(sink, seq_len - ring_rows), seq_len, dtype=np.int64)
    return np.concatenate([head, tail])


def kv_compact_ring(k_cache: np.ndarray, v_cache: np.ndarray, seq_len: np.ndarray,
                    sink: int, ring_rows: int):
    """Move a full cache [B][Hkv][cap][d] into ring caches [B][Hkv][sink + ring_rows][d]:
    every retained position p goes to ring_slot(p).  Slots that hold no position stay
    zero here (their content is unspecified in the library)."""
    batch, hkv, _, d = k_cache.shape
    k_ring = np.zeros((batch, hkv, sink + ring_rows, d), dtype=k_cache.dtype)
    v_ring = np.zeros_like(k_ring)
    for b in range(batch):
        pos = ring_retained_positions(int(seq_len[b]), sink, ring_rows)
        slots = ring_slot(pos, sink, ring_rows)
        for h in range(hkv):
            k_ring[b, h, slots] = k_cache[b, h, pos]
            v_ring[b, h, slots] = v_cache[b, h, pos]
    return k_ring, v_ring


def kv_append_ring(k_ring: np.ndarray, v_ring: np.ndarray, seq_len: np.ndarray,
                   k_new: np.ndarray, v_new: np.ndarray, sink: int, ring_rows: int):
    """Append n rows per sequence at logical positions [seq_len, seq_len + n) into ring
    caches and advance seq_len (rings never run out of room)."""
    k_out, v_out = k_ring.copy(), v_ring.copy()
    len_out = np.array(seq_len, dtype=np.int64).copy()
    for b in range(len(len_out)):
        for i in range(k_new.shape[1]):
            slot = int(ring_slot(len_out[b] + i, sink, ring_rows))
            k_out[b, :, slot] = k_new[b, i]
            v_out[b, :, slot] = v_new[b, i]
        len_out[b] += k_new.shape[1]
    return k_out, v_out, len_out

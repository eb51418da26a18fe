"""Workload shapes for the hybrid-attention hot path (shapes and seeds only).

* TINY: 2 layers (layer 0 FA, layer 1 SA), 8 query / 2 KV heads, head_dim 64,
  1024-token prompt, SA block 64 with sink 64 and window 256, router 512 -> 64 -> 2,
  prefill then 16 decode steps.
* LLAMA_PREFILL: Llama-3.1-8B attention shape (32 layers, 32 / 8 heads, head_dim 128),
  8192-token prompt, router 4096 -> 256 -> 32, SA sink 128 + window 2048 in 128-key
  blocks, router seed chosen for 16 SA layers.
* LLAMA_DECODE: the same shape decoding 16 sequences at a 32768-token context for 256
  steps, with a fixed seeded mask of 16 SA layers.
* QWEN_PREFILL: Qwen3-4B attention shape (36 layers, 32 / 8 heads, head_dim 128),
  131072-token prompt, router 2560 -> 256 -> 36, SA sink 128 + window 4096, router
  seed chosen for 22 SA layers.
* SWEEP: Llama shape over contexts x decode batches x SA-layer fractions.

The router seeds of LLAMA_PREFILL (10) and QWEN_PREFILL (19) are the first seeds whose
random-init router sends exactly 16 of 32 and 22 of 36 layers to SA at tau = 0 (the
"~50%" and "~60%" SA workloads); a seed search over the fp64 oracle recorded them with
the resulting bits, and the test suite checks these constants against that record.
"""

from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq: int                 # prompt length (prefill) or context before decode
    block: int
    sink: int
    window: int
    router_hidden: int
    router_rank: int
    pool_len: int = 100      # boundary pooling window; 0 = whole sequence
    tau: float = 0.0
    decode_steps: int = 0
    data_seed: int = 0
    router_seed: int = 0
    fixed_sa_layers: tuple = ()  # non-empty: use this mask instead of the router
    target_sa_layers: int = -1   # router seed is searched for this SA count

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def capacity(self) -> int:
        """KV cache capacity per sequence: the prompt plus every decode step."""
        return self.seq + self.decode_steps


# first router seeds giving exactly the target number of SA layers (see the module text)
LLAMA_PREFILL_ROUTER_SEED = 10
QWEN_PREFILL_ROUTER_SEED = 19


TINY = Workload(
    name="tiny_hybrid", batch=1, n_layers=2, n_q_heads=8, n_kv_heads=2, head_dim=64,
    seq=1024, block=64, sink=64, window=256, router_hidden=512, router_rank=64,
    decode_steps=16, data_seed=11, router_seed=5, fixed_sa_layers=(1,))

LLAMA_PREFILL = Workload(
    name="llama31_8b_prefill_8k", batch=1, n_layers=32, n_q_heads=32, n_kv_heads=8,
    head_dim=128, seq=8192, block=128, sink=128, window=2048, router_hidden=4096,
    router_rank=256, data_seed=21, router_seed=LLAMA_PREFILL_ROUTER_SEED,
    target_sa_layers=16)

LLAMA_DECODE = Workload(
    name="llama31_8b_decode_b16_32k", batch=16, n_layers=32, n_q_heads=32, n_kv_heads=8,
    head_dim=128, seq=32768, block=128, sink=128, window=2048, router_hidden=4096,
    router_rank=256, decode_steps=256, data_seed=31, router_seed=0,
    fixed_sa_layers=(), target_sa_layers=16)

QWEN_PREFILL = Workload(
    name="qwen3_4b_prefill_128k", batch=1, n_layers=36, n_q_heads=32, n_kv_heads=8,
    head_dim=128, seq=131072, block=128, sink=128, window=4096, router_hidden=2560,
    router_rank=256, data_seed=41, router_seed=QWEN_PREFILL_ROUTER_SEED,
    target_sa_layers=22)

# decode config's fixed mask: the first 16 entries of a seeded permutation of 32 layers
LLAMA_DECODE_MASK_SEED = 2604

SWEEP_CONTEXTS = (4096, 16384, 32768, 65536, 131072)
SWEEP_BATCHES = (1, 8, 32)
SWEEP_SA_FRACTIONS = (0.0, 0.25, 0.5, 0.75, 1.0)

ALL = {w.name: w for w in (TINY, LLAMA_PREFILL, LLAMA_DECODE, QWEN_PREFILL)}

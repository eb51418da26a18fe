"""Shared plumbing of the GPU parity tests: build seeded inputs, run them through the
C-ABI binding, run the same inputs through the oracle, compare.

Tolerances (bf16 attention outputs with fp32 accumulation): max-abs <= 2e-2 and
relative L2 <= 1e-2 against the fp64 oracle.  Router bits and block indices are
compared exactly.
"""

import numpy as np
import torch

from oracle import flux_oracle as orc
from sparse_attention_layer_b200 import flux, inputs
from sparse_attention_layer_b200.flux import AttnCfg

MAX_ABS = 2e-2
REL_L2 = 1e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64)


def assert_close(got: np.ndarray, want: np.ndarray, what: str = ""):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = float(np.abs(got - want).max()) if got.size else 0.0
    denom = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(got - want)) / denom if denom > 0 else float(np.linalg.norm(got))
    assert err <= MAX_ABS and rel <= REL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {rel:.3e}"
    return err, rel


def mask_words(batch: int, n_layers: int, fa_rows) -> torch.Tensor:
    """fa_rows[b] = list of FA layer indices for sequence b -> packed int32 words."""
    bits = torch.zeros(batch, n_layers, dtype=torch.bool)
    for b, layers in enumerate(fa_rows):
        for layer in layers:
            bits[b, layer] = True
    return inputs.pack_bits_u32(bits)


class CacheCase:
    """One layer's cache filled with `ctx[b]` seeded rows, mirrored on host for the
    oracle.  Rows past the filled length hold NaN bit patterns on the device to show
    that no kernel reads them into a result."""

    def __init__(self, cfg: AttnCfg, ctx, capacity: int, seed: int):
        self.cfg = cfg
        self.batch = len(ctx)
        self.capacity = capacity
        shape = (self.batch, cfg.n_kv_heads, capacity, cfg.head_dim)
        self.k_host = inputs.normal_bf16(shape, inputs.layer_seed(seed, 0, inputs.K))
        self.v_host = inputs.normal_bf16(shape, inputs.layer_seed(seed, 0, inputs.V))
        nan = torch.full((), float("nan"), dtype=torch.bfloat16)
        for b, n in enumerate(ctx):
            self.k_host[b, :, n:] = nan
            self.v_host[b, :, n:] = nan
        self.k = self.k_host.cuda()
        self.v = self.v_host.cuda()
        self.seq_len = torch.tensor(list(ctx), dtype=torch.int32, device="cuda")

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor):
        """Append through the library and mirror the rows into the host copy."""
        start = self.seq_len.cpu().tolist()
        flux.flux_kv_append(self.cfg, self.k, self.v, self.seq_len, k_new.cuda(), v_new.cuda())
        n = k_new.shape[1]
        for b in range(self.batch):
            self.k_host[b, :, start[b]:start[b] + n] = k_new[b].transpose(0, 1)
            self.v_host[b, :, start[b]:start[b] + n] = v_new[b].transpose(0, 1)


def oracle_layer(case: CacheCase, q_host: torch.Tensor, is_fa, rows=None, heads=None):
    """Oracle attention for q_host [B][n_q][Hq][d] over case's host cache, one sequence
    at a time (bounds host memory at full size)."""
    cfg = case.cfg
    lens = case.seq_len.cpu().numpy().astype(np.int64)
    outs = []
    for b in range(case.batch):
        n_keys = int(lens[b])
        kc = case.k_host[b:b + 1, :, :n_keys].float().numpy().astype(np.float64)
        vc = case.v_host[b:b + 1, :, :n_keys].float().numpy().astype(np.float64)
        q = q_host[b:b + 1].float().numpy().astype(np.float64)
        outs.append(orc.attention_layer(q, kc, vc, lens[b:b + 1], np.asarray(is_fa)[b:b + 1],
                                        cfg.block, cfg.sink, cfg.window, rows=rows,
                                        heads=heads))
    return np.concatenate(outs, axis=0)


def sample_rows(n_q: int, q_start: int, cfg: AttnCfg, n_random: int, seed: int):
    """First/last rows, rows at block and sink/window boundaries, plus seeded random."""
    rows = {0, n_q - 1, min(n_q - 1, 1), max(0, n_q - 2)}
    for edge in (cfg.block, cfg.sink, cfg.sink + cfg.window, cfg.window, 128, 2 * cfg.block):
        for d in (-1, 0, 1):
            r = edge + d - q_start
            if 0 <= r < n_q:
                rows.add(r)
    g = np.random.default_rng(seed)
    rows.update(int(x) for x in g.integers(0, n_q, n_random))
    return np.array(sorted(rows))

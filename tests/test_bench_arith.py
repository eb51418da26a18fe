"""The roofline arithmetic of bench.py, checked against the oracle's visibility masks:
the algorithmic bytes of a decode launch and the algorithmic flops of a prefill launch
count exactly the visible (query, key) pairs of the route, never the dense work SA
avoids.  CPU only."""

import importlib.util
import os
from types import SimpleNamespace

import numpy as np
import pytest

from oracle import flux_oracle as fo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def cfg(block=128, sink=128, window=2048, hq=32, hkv=8, d=128):
    return SimpleNamespace(block=block, sink=sink, window=window, n_q_heads=hq, n_kv_heads=hkv,
                           head_dim=d)


@pytest.mark.parametrize("fa", [True, False])
@pytest.mark.parametrize("T", [1, 100, 2176, 2177, 4097, 32769])
def test_decode_bytes_count_visible_keys(bench, fa, T):
    c = cfg()
    w = SimpleNamespace(batch=3)
    t = T - 1  # the decode query sits at the last position after the append
    mask = fo.visible_mask(fa, np.array([t]), T, c.block, c.sink, c.window)
    n_vis = int(mask.sum())
    want = 2 * 2 * w.batch * c.n_kv_heads * c.head_dim * n_vis + 2 * 2 * w.batch * c.n_q_heads * c.head_dim
    assert bench.decode_bytes_per_layer(w, c, T, fa) == want


@pytest.mark.parametrize("fa", [True, False])
@pytest.mark.parametrize("geom", [(64, 64, 256), (128, 128, 512)])
@pytest.mark.parametrize("S", [1, 130, 700])
def test_prefill_flops_count_visible_pairs(bench, fa, geom, S):
    block, sink, window = geom
    c = cfg(block=block, sink=sink, window=window, hq=4, hkv=2, d=64)
    mask = fo.visible_mask(fa, np.arange(S), S, block, sink, window)
    want = 4.0 * c.head_dim * c.n_q_heads * float(mask.sum())
    assert bench.prefill_flops_per_layer(c, S, fa) == want


def test_llama_decode_and_prefill_figures(bench):
    """The figures the bench reports for the Llama decode and prefill workloads."""
    c = cfg()
    w = SimpleNamespace(batch=16)
    fa = bench.decode_bytes_per_layer(w, c, 32769, True)
    sa = bench.decode_bytes_per_layer(w, c, 32769, False)
    assert fa == 2 * 2 * 16 * 8 * 128 * 32769 + 2 * 2 * 16 * 32 * 128
    # sink block + the query's own block (1 key so far) + 15 earlier window blocks
    assert sa == 2 * 2 * 16 * 8 * 128 * (128 + 1 + 15 * 128) + 2 * 2 * 16 * 32 * 128
    # causal FA over 8192 tokens: sum of (t + 1) visible keys per query row
    assert bench.prefill_flops_per_layer(c, 8192, True) == 4.0 * 128 * 32 * 8192 * 8193 / 2


def test_fused_append_adds_the_new_rows(bench):
    """A flux_decode_append launch also writes one K and one V row per (sequence, KV head)."""
    c = cfg()
    w = SimpleNamespace(batch=16)
    for fa in (True, False):
        plain = bench.decode_bytes_per_layer(w, c, 32769, fa)
        fused = bench.decode_bytes_per_layer(w, c, 32769, fa, append=True)
        assert fused - plain == 2 * 2 * 16 * 8 * 128

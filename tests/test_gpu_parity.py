"""GPU parity: the CUDA path, called through the C ABI (ctypes binding), against the
fp64 oracle on the same seeded inputs.

Small cases span several 128-row tiles with ragged tails; full-size cases (the Llama
and Qwen workloads, in the launch configuration the benchmark times) compare sampled
rows the oracle computes one by one.  Router bits and SA block indices must match
exactly; attention outputs within max-abs 2e-2 and relative L2 1e-2.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import flux_oracle as orc
from sparse_attention_layer_b200 import configs, flux, inputs
from sparse_attention_layer_b200.flux import AttnCfg
from tests.gpu_cases import CacheCase, assert_close, f64, mask_words, oracle_layer, sample_rows

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.fixture(autouse=True)
def _status_clean():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    flux.flux_get_device_status()
    yield


def cfg_of(w: configs.Workload) -> AttnCfg:
    return AttnCfg(w.n_layers, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.sink, w.window)


# ------------------------------------------------------------------------- router


def _route(w1, b1, w2, b2, xq, pool_len, tau):
    batch, n_layers = xq.shape[0], w2.shape[0]
    mask = torch.zeros(batch, (n_layers + 31) // 32, dtype=torch.int32, device="cuda")
    logits = torch.zeros(batch, n_layers, dtype=torch.float64, device="cuda")
    flux.flux_route(w1.cuda(), None if b1 is None else b1.cuda(), w2.cuda(),
                    None if b2 is None else b2.cuda(), xq.cuda(), pool_len, tau, mask, logits)
    torch.cuda.synchronize()
    return mask.cpu(), logits.cpu().numpy()


def _check_router(xq, w1, b1, w2, b2, pool_len, tau):
    mask, z_gpu = _route(w1, b1, w2, b2, xq, pool_len, tau)
    x64 = [t.float().numpy().astype(np.float64) for t in (xq, w1, b1, w2, b2)]
    res = orc.router(*x64, pool_len, tau)
    bound = orc.router_error_bound(*x64, pool_len)
    # logits agree within the fp64 evaluation-order bound (both sides fp64)
    assert (np.abs(z_gpu - res["logits"]) <= bound).all()
    decided = np.abs(res["logits"] - tau) > bound
    gpu_bits = ((mask.numpy().view(np.uint32)[:, np.arange(w2.shape[0]) // 32]
                 >> (np.arange(w2.shape[0]) % 32)) & 1).astype(bool)
    # unique decisions bit-exact; any undecidable one must follow the GPU's own logit
    assert (gpu_bits[decided] == res["fa_bits"][decided]).all()
    assert (gpu_bits[~decided] == (z_gpu[~decided] > tau)).all()
    if decided.all():
        assert (mask.numpy().view(np.uint32) == res["fa_mask"]).all()
    return gpu_bits, res


def test_router_toy_golden():
    g = json.load(open(os.path.join(GOLDEN, "router_toy.json")))
    pad = 8  # the library wants hidden % 8 == 0: zero columns leave the logits unchanged
    xq = torch.zeros(1, 4, pad)
    xq[:, :, :4] = torch.tensor(g["xq"], dtype=torch.float32)
    w1 = torch.zeros(2, pad)
    w1[:, :4] = torch.tensor(g["w1"], dtype=torch.float32)
    b1 = torch.tensor(g["b1"]); w2 = torch.tensor(g["w2"]); b2 = torch.tensor(g["b2"])
    bf = lambda t: t.to(torch.bfloat16)  # noqa: E731
    for case in g["cases"]:
        mask, z = _route(bf(w1), bf(b1), bf(w2), bf(b2), bf(xq), case["pool_len"], g["tau"])
        assert np.allclose(z, case["logits"], atol=1e-9)
        assert mask.numpy().view(np.uint32).tolist() == case["mask_words"]


@pytest.mark.parametrize("pool_len", [100, 0, 7])
def test_router_tiny(pool_len):
    w = configs.TINY
    xq = inputs.normal_bf16((2, w.seq, w.router_hidden), inputs.layer_seed(w.data_seed, 0, inputs.XQ))
    w1, b1, w2, b2 = inputs.router_weights(w.router_hidden, w.router_rank, w.n_layers, w.router_seed)
    _check_router(xq, w1, b1, w2, b2, pool_len, w.tau)


def test_router_nonzero_bias_and_threshold():
    xq = inputs.normal_bf16((3, 300, 256), 77)
    w1 = inputs.normal_bf16((40, 256), 78, std=0.05)
    w2 = inputs.normal_bf16((37, 40), 79, std=0.05)  # 37 layers: two mask words
    b1 = inputs.normal_bf16((40,), 80, std=0.01)
    b2 = inputs.normal_bf16((37,), 81, std=0.01)
    _check_router(xq, w1, b1, w2, b2, 100, 0.003)


@pytest.mark.parametrize("name", ["llama31_8b_prefill_8k", "qwen3_4b_prefill_128k"])
def test_router_full_size(name):
    w = configs.ALL[name]
    seeds = json.load(open(os.path.join(GOLDEN, "router_seeds.json")))[name]
    xq = inputs.normal_bf16((w.batch, w.seq, w.router_hidden),
                            inputs.layer_seed(w.data_seed, 0, inputs.XQ))
    w1, b1, w2, b2 = inputs.router_weights(w.router_hidden, w.router_rank, w.n_layers,
                                           seeds["router_seed"])
    bits, res = _check_router(xq, w1, b1, w2, b2, w.pool_len, w.tau)
    assert bits[0].astype(int).tolist() == seeds["fa_bits"]
    assert int((~bits).sum()) == w.target_sa_layers


# ------------------------------------------------------------------ SA block indices


@pytest.mark.parametrize("block,sink,window", [(64, 64, 256), (128, 128, 2048), (128, 128, 4096),
                                               (64, 0, 64), (128, 256, 128), (64, 128, 256)])
def test_sa_block_ranges_exact(block, sink, window):
    cfg = AttnCfg(2, 8, 2, 64, block, sink, window)
    n_qb = 80
    ranges = torch.zeros(n_qb, 3, dtype=torch.int32, device="cuda")
    flux.flux_sa_block_ranges(cfg, n_qb, ranges)
    r = ranges.cpu().numpy()
    for qb in range(n_qb):
        got = set(range(0, r[qb, 0])) | set(range(r[qb, 1], r[qb, 2]))
        want = orc.sa_visible_key_blocks(qb, qb + 1, block, sink, window)
        assert got == want, (qb, r[qb].tolist(), sorted(want))


def _tile_plan(cfg, layer, mask, seq_len, capacity, n_q):
    n_mt = (n_q + 127) // 128
    max_tiles = (capacity + 127) // 128
    tiles = torch.empty(len(seq_len), n_mt, max_tiles, dtype=torch.int32, device="cuda")
    seq = torch.tensor(seq_len, dtype=torch.int32, device="cuda")
    flux.flux_prefill_tile_plan(cfg, layer, mask, seq, capacity, n_q, tiles)
    torch.cuda.synchronize()
    assert flux.flux_get_device_status() == 0
    return tiles.cpu().numpy()


def _check_tile_plan(cfg, tiles, b, m, q_start, n_q, fa):
    """Query tile m of sequence b: the kernel's visited tiles (in visiting order) and the
    ones it masks equal the oracle's sets from the dense visibility mask."""
    rows = q_start + np.arange(m * 128, min(n_q, (m + 1) * 128))
    want_vis, want_msk = orc.key_tiles_of_rows(fa, rows, 128, cfg.block, cfg.sink, cfg.window)
    row = tiles[b, m]
    n = int((row >= 0).sum())
    assert (row[n:] == -1).all() and (row[:n] >= 0).all()
    got = row[:n]
    got_vis = (got & ~flux.FLUX_TILE_MASKED).tolist()
    got_msk = [int(e & ~flux.FLUX_TILE_MASKED) for e in got if e & flux.FLUX_TILE_MASKED]
    assert got_vis == want_vis, (b, m, got_vis, want_vis)
    assert got_msk == want_msk, (b, m, got_msk, want_msk)


@pytest.mark.parametrize("block,sink,window", [
    (64, 0, 64), (64, 64, 256), (64, 128, 256), (64, 128, 2048), (64, 128, 4096),
    (128, 0, 128), (128, 128, 128), (128, 128, 2048), (128, 256, 1024), (128, 128, 4096)])
def test_prefill_tile_plan_exact(block, sink, window):
    """SA block indices of the prefill kernel, exactly: the 128-key tiles it visits for
    every 128-query tile, and the tiles it masks, equal the oracle's (tiles holding a key
    some row of the query tile sees; of those, tiles with a pair some row does not see).
    One-shot and chunked prompts (queries after a prefix), ragged last tile, per-sequence
    routes in one batch."""
    cfg = AttnCfg(2, 8, 2, 128, block, sink, window)
    n_q = 3000                                  # 23 full query tiles + 56 rows
    q_starts = [0, 77, 4096, 5000]
    seq_len = [qs + n_q for qs in q_starts]
    capacity = max(seq_len) + 5
    fa_rows = [[], [0], [1], []]                # layer 0: SA, FA, SA, SA; layer 1: SA, SA, FA, SA
    mask = mask_words(len(seq_len), cfg.n_layers, fa_rows).cuda()
    for layer in (0, 1):
        tiles = _tile_plan(cfg, layer, mask, seq_len, capacity, n_q)
        for b, qs in enumerate(q_starts):
            for m in range(tiles.shape[1]):
                _check_tile_plan(cfg, tiles, b, m, qs, n_q, layer in fa_rows[b])


@pytest.mark.parametrize("name", ["llama31_8b_prefill_8k", "qwen3_4b_prefill_128k"])
def test_prefill_tile_plan_full_size(name):
    """The full-size prompts' tile schedules, exactly, for the SA route on every query tile
    of the Llama prompt and on sampled query tiles of the 131072-token Qwen prompt (the FA
    route checked on sampled tiles)."""
    w = configs.ALL[name]
    cfg = cfg_of(w)
    for fa in (False, True):
        mask = mask_words(1, cfg.n_layers, [[3] if fa else []]).cuda()
        tiles = _tile_plan(cfg, 3, mask, [w.seq], w.seq, w.seq)
        n_mt = tiles.shape[1]
        if n_mt <= 64 and not fa:
            ms = range(n_mt)
        else:
            g = np.random.default_rng(7)
            ms = sorted({0, 1, 15, 16, 17, 31, 32, 33, n_mt - 1} | set(g.integers(0, n_mt, 12).tolist()))
        for m in ms:
            _check_tile_plan(cfg, tiles, 0, m, 0, w.seq, fa)


# ------------------------------------------------------------------------ KV append


def test_kv_append_exact_and_capacity():
    cfg = AttnCfg(2, 8, 2, 64, 64, 64, 256)
    batch, cap = 3, 40
    k = torch.zeros(batch, 2, cap, 64, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    seq = torch.tensor([0, 30, 38], dtype=torch.int32, device="cuda")
    kn = inputs.normal_bf16((batch, 5, 2, 64), 5)
    vn = inputs.normal_bf16((batch, 5, 2, 64), 6)
    flux.flux_kv_append(cfg, k, v, seq, kn.cuda(), vn.cuda())
    assert flux.flux_get_device_status() == flux.FLUX_DEVICE_CAPACITY
    k2, v2, s2, over = orc.kv_append(np.zeros((batch, 2, cap, 64)), np.zeros((batch, 2, cap, 64)),
                                     np.array([0, 30, 38]), f64(kn), f64(vn))
    assert seq.cpu().tolist() == s2.tolist() and over.tolist() == [False, False, True]
    assert np.array_equal(f64(k), k2) and np.array_equal(f64(v), v2)
    # bit-exact copy, including the byte patterns
    assert torch.equal(k[1, :, 30:35].cpu().view(torch.int16), kn[1].transpose(0, 1).view(torch.int16))


# --------------------------------------------------------------------------- decode


def _decode_case(cfg, ctx, fa_per_seq, steps, seed, capacity=None, layer=0):
    batch = len(ctx)
    cap = capacity or (max(ctx) + steps + 8)
    case = CacheCase(cfg, ctx, cap, seed)
    fa_rows = [[layer] if fa else [] for fa in fa_per_seq]
    mask = mask_words(batch, cfg.n_layers, fa_rows).cuda()
    ws = flux.new_decode_workspace(cfg, batch)
    for step in range(steps):
        kn = inputs.normal_bf16((batch, 1, cfg.n_kv_heads, cfg.head_dim), seed * 31 + step * 3 + 1)
        vn = inputs.normal_bf16((batch, 1, cfg.n_kv_heads, cfg.head_dim), seed * 31 + step * 3 + 2)
        q = inputs.normal_bf16((batch, cfg.n_q_heads, cfg.head_dim), seed * 31 + step * 3 + 3)
        case.append(kn, vn)
        o = torch.empty(batch, cfg.n_q_heads, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
        flux.flux_decode(cfg, layer, mask, q.cuda(), case.k, case.v, case.seq_len, o, ws)
        torch.cuda.synchronize()
        want = oracle_layer(case, q[:, None], fa_per_seq)[:, 0]
        assert_close(f64(o), want, f"decode step {step}")
    assert flux.flux_get_device_status() == 0


def test_decode_tiny_config():
    """Tiny workload: 1024-token context, layer 0 FA and layer 1 SA, 16 decode steps."""
    w = configs.TINY
    cfg = cfg_of(w)
    for layer, fa in ((0, True), (1, False)):
        _decode_case(cfg, [w.seq], [fa], w.decode_steps, seed=100 + layer, layer=layer)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_decode_groups_and_head_dims(d, group):
    cfg = AttnCfg(3, 2 * group, 2, d, 64, 64, 192)
    _decode_case(cfg, [700, 1, 64, 333, 4000], [True, False, True, False, False], 2,
                 seed=7 + group + d, layer=2)


def test_decode_ragged_edges():
    """Contexts shorter than the sink, exactly one block, one key past the window."""
    cfg = AttnCfg(1, 8, 2, 128, 128, 128, 256)
    ctx = [0, 5, 127, 128, 383, 384, 385, 9000]
    _decode_case(cfg, ctx, [False] * len(ctx), 1, seed=3)
    _decode_case(cfg, ctx, [True] * len(ctx), 1, seed=4)


def test_decode_empty_sequence_writes_zeros():
    cfg = AttnCfg(1, 4, 1, 64, 64, 64, 64)
    k = torch.zeros(2, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([0, 0], dtype=torch.int32, device="cuda")
    mask = torch.zeros(2, 1, dtype=torch.int32, device="cuda")
    ws = flux.new_decode_workspace(cfg, 2)
    o = torch.full((2, 4, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    q = torch.ones(2, 4, 64, dtype=torch.bfloat16, device="cuda")
    flux.flux_decode(cfg, 0, mask, q, k, k, seq, o, ws)
    torch.cuda.synchronize()
    assert (o == 0).all()


def test_decode_bad_length_flag():
    cfg = AttnCfg(1, 4, 1, 64, 64, 64, 64)
    k = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([17], dtype=torch.int32, device="cuda")  # past capacity 16
    mask = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    ws = flux.new_decode_workspace(cfg, 1)
    o = torch.empty(1, 4, 64, dtype=torch.bfloat16, device="cuda")
    flux.flux_decode(cfg, 0, mask, torch.ones_like(o), k, k, seq, o, ws)
    assert flux.flux_get_device_status() & flux.FLUX_DEVICE_BAD_LENGTH


# -------------------------------------------------------------------------- prefill


def _prefill_case(cfg, q_start, n_q, fa_per_seq, seed, layer=0, rows=None, heads=None,
                  capacity=None):
    batch = len(q_start)
    cap = capacity or (max(q_start) + n_q + 5)
    case = CacheCase(cfg, q_start, cap, seed)
    kn = inputs.normal_bf16((batch, n_q, cfg.n_kv_heads, cfg.head_dim), seed * 17 + 1)
    vn = inputs.normal_bf16((batch, n_q, cfg.n_kv_heads, cfg.head_dim), seed * 17 + 2)
    q = inputs.normal_bf16((batch, n_q, cfg.n_q_heads, cfg.head_dim), seed * 17 + 3)
    case.append(kn, vn)
    fa_rows = [[layer] if fa else [] for fa in fa_per_seq]
    mask = mask_words(batch, cfg.n_layers, fa_rows).cuda()
    o = torch.empty(batch, n_q, cfg.n_q_heads, cfg.head_dim, dtype=torch.bfloat16, device="cuda")
    flux.flux_prefill(cfg, layer, mask, q.cuda(), case.k, case.v, case.seq_len, o)
    torch.cuda.synchronize()
    assert flux.flux_get_device_status() == 0
    want = oracle_layer(case, q, fa_per_seq, rows=rows, heads=heads)
    got = o.cpu()
    if rows is not None:
        got = got[:, torch.as_tensor(rows)]
    if heads is not None:
        got = got[:, :, torch.as_tensor(heads)]
    return assert_close(f64(got), want, "prefill")


def test_prefill_tiny_config():
    """Tiny workload prefill: 1024 tokens, layer 0 FA, layer 1 SA (block 64)."""
    w = configs.TINY
    cfg = cfg_of(w)
    _prefill_case(cfg, [0], w.seq, [True], seed=200, layer=0)
    _prefill_case(cfg, [0], w.seq, [False], seed=201, layer=1)


@pytest.mark.parametrize("fa", [True, False])
@pytest.mark.parametrize("d", [64, 128])
def test_prefill_ragged_tail(fa, d):
    cfg = AttnCfg(1, 4, 2, d, 128, 128, 256)
    _prefill_case(cfg, [0], 1000, [fa], seed=300 + d + fa)   # 1000 = 7 tiles + 104 rows


@pytest.mark.parametrize("block", [64, 128])
def test_prefill_chunked_and_mixed_batch(block):
    """Queries after an existing prefix (chunked prefill), per-sequence routes, ragged
    lengths in one batch."""
    cfg = AttnCfg(2, 8, 2, 128, block, block, 4 * block)
    _prefill_case(cfg, [0, 300, 1024, 77], 700, [False, True, False, True], seed=400 + block,
                  layer=1)


@pytest.mark.parametrize("group", [1, 2, 8])
def test_prefill_groups(group):
    cfg = AttnCfg(1, 2 * group, 2, 64, 64, 0, 128)   # no sink
    _prefill_case(cfg, [0], 600, [False], seed=500 + group)


def test_prefill_short_sequences():
    cfg = AttnCfg(1, 4, 1, 128, 128, 128, 128)
    for n_q in (1, 2, 127, 128, 129):
        _prefill_case(cfg, [0], n_q, [False], seed=600 + n_q)
        _prefill_case(cfg, [0], n_q, [True], seed=700 + n_q)


# ------------------------------------------------------------ full-size workloads


@pytest.mark.parametrize("fa", [True, False])
def test_prefill_llama_full_size(fa):
    """Llama-3.1-8B shape, 8192-token prompt, one FA and one SA layer; sampled rows."""
    w = configs.LLAMA_PREFILL
    cfg = cfg_of(w)
    rows = sample_rows(w.seq, 0, cfg, 40, seed=1)
    _prefill_case(cfg, [0], w.seq, [fa], seed=800 + fa, rows=rows, heads=[0, 5, 17, 31],
                  capacity=w.seq)


@pytest.mark.parametrize("fa", [True, False])
def test_prefill_qwen_full_size(fa):
    """Qwen3-4B shape, 131072-token prompt, SA window 4096; sampled rows."""
    w = configs.QWEN_PREFILL
    cfg = cfg_of(w)
    rows = sample_rows(w.seq, 0, cfg, 16, seed=2)
    _prefill_case(cfg, [0], w.seq, [fa], seed=900 + fa, rows=rows, heads=[0, 31],
                  capacity=w.seq)


@pytest.mark.parametrize("fa", [True, False])
def test_prefill_llama_128k(fa):
    """The sweep's longest prefill point in the Llama geometry (block 128, sink 128,
    window 2048): a 131072-token prompt, sampled rows."""
    w = configs.LLAMA_PREFILL
    cfg = cfg_of(w)
    seq = 131072
    rows = sample_rows(seq, 0, cfg, 16, seed=3)
    _prefill_case(cfg, [0], seq, [fa], seed=950 + fa, rows=rows, heads=[0, 31],
                  capacity=seq)


def test_decode_llama_full_size():
    """Llama-3.1-8B decode: 16 sequences at 32768 context, FA and SA layers."""
    w = configs.LLAMA_DECODE
    cfg = cfg_of(w)
    ctx = [w.seq] * w.batch
    _decode_case(cfg, ctx, [True] * w.batch, 1, seed=1000, capacity=w.capacity(), layer=3)
    _decode_case(cfg, ctx, [False] * w.batch, 2, seed=1001, capacity=w.capacity(), layer=4)


@pytest.mark.parametrize("fa", [True, False])
def test_decode_llama_batch1_128k(fa):
    """Llama-3.1-8B heads, one sequence at a 131072-token context (the sweep's longest
    point at batch 1): the 8 (sequence, KV head) pairs are each cut over ~18 CTAs."""
    cfg = AttnCfg(32, 32, 8, 128, 128, 128, 2048)
    _decode_case(cfg, [131072], [fa], 2, seed=1200 + fa, layer=9)


def test_decode_split_cap_single_pair():
    """One KV head, 8 query heads, a 131072-token FA context and SA beside it: a single
    pair of 1025 stages is dealt to ~61 CTAs, the most the split planner allows."""
    cfg = AttnCfg(1, 8, 1, 128, 128, 128, 2048)
    _decode_case(cfg, [131072, 131000], [True, False], 1, seed=1210)


def test_decode_llama_batch32_32k():
    """Llama-3.1-8B decode at the sweep's batch 32 x 32768 context, mixed routes."""
    cfg = AttnCfg(32, 32, 8, 128, 128, 128, 2048)
    ctx = [32768] * 32
    fa = [b % 2 == 0 for b in range(32)]
    _decode_case(cfg, ctx, fa, 1, seed=1220, layer=17)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_pages_sa_geometry(d):
    """The pages' SA kernel geometry (Table 6: block 64, sink 128) with a 2048-token
    window, Llama heads, head_dim 64 and 128: 16 sequences at a 32768-token context,
    SA and FA sequences in one batch, across a block boundary."""
    cfg = AttnCfg(32, 32, 8, d, 64, 128, 2048)
    ctx = [32768 - 2] * 8 + [32768 + 61] * 8
    fa = [b % 4 == 0 for b in range(16)]
    _decode_case(cfg, ctx, fa, 3, seed=1230 + d, layer=5)


@pytest.mark.parametrize("d,group", [(128, 4), (64, 8), (128, 1)])
def test_decode_append_equals_append_then_decode(d, group):
    """flux_decode_append (one launch) equals flux_kv_append + flux_decode bit for bit --
    outputs, cache rows and lengths -- over several steps with ragged lengths, an empty
    sequence and mixed routes; a sequence without room writes zeros, keeps its rows and
    length and sets the capacity flag.  The fused outputs also match the oracle."""
    cfg = AttnCfg(2, 2 * group, 2, d, 64, 64, 256)
    cap = 2003
    ctx = [0, 1, 63, 64, 700, 2000, 1999, cap]   # the last one has no room
    fa = [False, True, False, True, False, False, True, False]
    batch = len(ctx)
    sep, fused = CacheCase(cfg, ctx, cap, 77), CacheCase(cfg, ctx, cap, 77)
    mask = mask_words(batch, cfg.n_layers, [[1] if f else [] for f in fa]).cuda()
    ws_a, ws_b = flux.new_decode_workspace(cfg, batch), flux.new_decode_workspace(cfg, batch)
    room = [c < cap for c in ctx]
    for step in range(3):
        kn = inputs.normal_bf16((batch, 1, cfg.n_kv_heads, d), 4000 + step).cuda()
        vn = inputs.normal_bf16((batch, 1, cfg.n_kv_heads, d), 4100 + step).cuda()
        q = inputs.normal_bf16((batch, cfg.n_q_heads, d), 4200 + step).cuda()
        o_sep = torch.empty_like(q)
        o_fused = torch.full_like(q, float("nan"))
        flux.flux_kv_append(cfg, sep.k, sep.v, sep.seq_len, kn, vn)
        flux.flux_decode(cfg, 1, mask, q, sep.k, sep.v, sep.seq_len, o_sep, ws_a)
        assert flux.flux_get_device_status() == flux.FLUX_DEVICE_CAPACITY
        flux.flux_decode_append(cfg, 1, mask, q, kn, vn, fused.k, fused.v, fused.seq_len, o_fused,
                                ws_b)
        torch.cuda.synchronize()
        assert flux.flux_get_device_status() == flux.FLUX_DEVICE_CAPACITY
        r = torch.tensor(room)
        assert torch.equal(o_fused[r], o_sep[r]), f"step {step}"
        assert (o_fused[~r] == 0).all()
        assert torch.equal(fused.seq_len, sep.seq_len)
        assert torch.equal(fused.k.view(torch.int16), sep.k.view(torch.int16))
        assert torch.equal(fused.v.view(torch.int16), sep.v.view(torch.int16))
        # mirror the appends on the host copy for the oracle
        for b in range(batch):
            if room[b]:
                t = ctx[b] + step
                fused.k_host[b, :, t] = kn[b, 0].cpu()
                fused.v_host[b, :, t] = vn[b, 0].cpu()
    want = oracle_layer(fused, q.cpu()[:, None], fa)[:, 0]
    rr = np.array(room)
    assert_close(f64(o_fused)[rr], want[rr], "fused decode vs oracle")
    assert (ws_a[:4352] == 0).all() and (ws_b[:4352] == 0).all()  # counters back at zero


def test_decode_append_ring_equals_separate_calls():
    """flux_decode_append_ring equals flux_kv_append_ring + flux_decode_ring bit for bit,
    and the full-cache fused decode too, across a ring wrap."""
    cfg = AttnCfg(1, 8, 2, 128, 64, 128, 256)
    ring_rows = 256
    ctx = [1, 131, 383, 385, 1000]
    batch = len(ctx)
    case_a, k_ra, v_ra, len_a = _ring_setup(cfg, ctx, ring_rows, seed=31)
    case_b, k_rb, v_rb, len_b = _ring_setup(cfg, ctx, ring_rows, seed=31)
    mask = mask_words(batch, 1, [[] for _ in ctx]).cuda()
    ws = [flux.new_decode_workspace(cfg, batch) for _ in range(3)]
    for step in range(70):   # crosses a block boundary and wraps the ring
        kn = inputs.normal_bf16((batch, 1, 2, 128), 5000 + step).cuda()
        vn = inputs.normal_bf16((batch, 1, 2, 128), 5100 + step).cuda()
        q = inputs.normal_bf16((batch, 8, 128), 5200 + step).cuda()
        o_sep, o_fused, o_full = (torch.empty_like(q) for _ in range(3))
        flux.flux_kv_append_ring(cfg, k_ra, v_ra, len_a, kn, vn)
        flux.flux_decode_ring(cfg, 0, mask, q, k_ra, v_ra, len_a, o_sep, ws[0])
        flux.flux_decode_append_ring(cfg, 0, mask, q, kn, vn, k_rb, v_rb, len_b, o_fused, ws[1])
        flux.flux_decode_append(cfg, 0, mask, q, kn, vn, case_b.k, case_b.v, case_b.seq_len,
                                o_full, ws[2])
        torch.cuda.synchronize()
        assert torch.equal(o_fused, o_sep) and torch.equal(o_full, o_sep), f"step {step}"
        assert torch.equal(len_a, len_b) and torch.equal(k_ra.view(torch.int16), k_rb.view(torch.int16))
    assert flux.flux_get_device_status() == 0


def test_decode_workspace_shared_across_geometries():
    """One zero-filled workspace serves calls of different batches, routes and split plans
    in turn (its arrival counters sit at fixed offsets and return to zero)."""
    cfg = AttnCfg(1, 32, 8, 128, 128, 128, 2048)
    ws = flux.new_decode_workspace(cfg, 16)
    for seed, ctx, fa in ((1, [40000], [True]), (2, [3000] * 16, [False] * 16),
                          (3, [33000] * 4, [True, False, True, True]), (4, [500, 90000], [True, True])):
        case = CacheCase(cfg, ctx, max(ctx) + 1, 1300 + seed)
        mask = mask_words(len(ctx), 1, [[0] if f else [] for f in fa]).cuda()
        q = inputs.normal_bf16((len(ctx), 32, 128), 1400 + seed).cuda()
        o = torch.empty_like(q)
        flux.flux_decode(cfg, 0, mask, q, case.k, case.v, case.seq_len, o, ws)
        torch.cuda.synchronize()
        assert (ws[:4352] == 0).all(), seed
        want = oracle_layer(case, q.cpu()[:, None], fa)[:, 0]
        assert_close(f64(o), want, f"shared workspace call {seed}")
    assert flux.flux_get_device_status() == 0


def test_decode_append_batch_limit():
    """1024 sequences (the decode batch limit: the per-sequence length table and stage
    prefix fill the kernel's shared-memory tables), ragged lengths from 0 to 600, mixed
    routes, the fused append; outputs against the oracle and lengths advanced by one."""
    cfg = AttnCfg(2, 8, 2, 64, 64, 64, 256)
    batch = 1024
    ctx = inputs.random_seq_lens(batch, 0, 600, seed=31).tolist()
    cap = 608
    case = CacheCase(cfg, ctx, cap, seed=1240)
    fa = [(b * 7) % 3 == 0 for b in range(batch)]
    mask = mask_words(batch, cfg.n_layers, [[1] if f else [] for f in fa]).cuda()
    ws = flux.new_decode_workspace(cfg, batch)
    kn = inputs.normal_bf16((batch, 1, 2, 64), 1241)
    vn = inputs.normal_bf16((batch, 1, 2, 64), 1242)
    q = inputs.normal_bf16((batch, 8, 64), 1243)
    o = torch.empty(batch, 8, 64, dtype=torch.bfloat16, device="cuda")
    flux.flux_decode_append(cfg, 1, mask, q.cuda(), kn.cuda(), vn.cuda(), case.k, case.v,
                            case.seq_len, o, ws)
    torch.cuda.synchronize()
    assert flux.flux_get_device_status() == 0
    assert case.seq_len.cpu().tolist() == [c + 1 for c in ctx]
    for b in range(batch):
        case.k_host[b, :, ctx[b]] = kn[b, 0]
        case.v_host[b, :, ctx[b]] = vn[b, 0]
    want = oracle_layer(case, q[:, None], fa)[:, 0]
    assert_close(f64(o), want, "decode at batch 1024")
    assert (ws[:4352] == 0).all()


def test_decode_graph_replay_matches_eager():
    """A decode step captured as a CUDA graph replays to the outputs of the eager calls
    (lengths and routes are read on the device, so the graph serves every step)."""
    from sparse_attention_layer_b200.runtime import DecodeStepGraph, HybridAttention
    cfg = AttnCfg(3, 8, 2, 128, 128, 128, 256)
    batch, ctx, steps = 3, 700, 4
    mask = mask_words(batch, 3, [[0], [0, 2], []]).cuda()
    models = [HybridAttention(cfg, batch, ctx + steps, "cuda") for _ in range(2)]
    for m in models:
        m.set_mask(mask)
        for layer, c in enumerate(m.caches):
            c.k.copy_(inputs.normal_bf16(c.k.shape, 50 + layer).cuda())
            c.v.copy_(inputs.normal_bf16(c.v.shape, 60 + layer).cuda())
            c.seq_len.fill_(ctx)
    q = torch.zeros(3, batch, 8, 128, dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros(3, batch, 1, 2, 128, dtype=torch.bfloat16, device="cuda")
    vn = torch.zeros_like(kn)
    o = torch.zeros_like(q)
    eager_m, graph_m = models
    # one eager step on the graph model first (one-time set-up), then undo its append
    for layer in range(3):
        graph_m.decode_layer(layer, q[layer], kn[layer], vn[layer], o[layer])
    for c in graph_m.caches:
        c.seq_len.fill_(ctx)
    g = DecodeStepGraph(graph_m, q, kn, vn, o)
    for step in range(steps):
        q.copy_(inputs.normal_bf16(q.shape, 70 + step).cuda())
        kn.copy_(inputs.normal_bf16(kn.shape, 80 + step).cuda())
        vn.copy_(inputs.normal_bf16(vn.shape, 90 + step).cuda())
        o_e = torch.empty_like(o)
        for layer in range(3):
            eager_m.decode_layer(layer, q[layer], kn[layer], vn[layer], o_e[layer])
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_e), f"step {step}"
    assert [int(c.seq_len[0]) for c in graph_m.caches] == [ctx + steps] * 3


# ------------------------------------------------------ SA ring caches (KV eviction)


def _ring_setup(cfg, ctx, ring_rows, seed):
    case = CacheCase(cfg, ctx, max(ctx) + 200, seed)
    rows = cfg.sink + ring_rows
    k_ring = torch.zeros(len(ctx), cfg.n_kv_heads, rows, cfg.head_dim, dtype=torch.bfloat16,
                         device="cuda")
    v_ring = torch.zeros_like(k_ring)
    flux.flux_kv_compact_ring(cfg, case.k, case.v, case.seq_len, k_ring, v_ring)
    ring_len = case.seq_len.clone()
    return case, k_ring, v_ring, ring_len


def _retained_equal(cfg, ring_rows, k_ring, full_host, lens):
    for b, T in enumerate(lens):
        pos = orc.ring_retained_positions(int(T), cfg.sink, ring_rows)
        slots = orc.ring_slot(pos, cfg.sink, ring_rows)
        got = k_ring[b][:, torch.as_tensor(slots)].cpu().view(torch.int16)
        want = full_host[b][:, torch.as_tensor(pos)].view(torch.int16)
        assert torch.equal(got, want), (b, T)


def test_ring_compact_and_append_exact():
    cfg = AttnCfg(1, 8, 2, 128, 64, 128, 256)
    ring_rows = 320
    ctx = [0, 50, 128, 300, 449, 450, 1000, 1777]
    case, k_ring, v_ring, ring_len = _ring_setup(cfg, ctx, ring_rows, seed=5)
    _retained_equal(cfg, ring_rows, k_ring, case.k_host, ctx)
    _retained_equal(cfg, ring_rows, v_ring, case.v_host, ctx)
    for step in range(3):
        kn = inputs.normal_bf16((len(ctx), 1, 2, 128), 300 + step)
        vn = inputs.normal_bf16((len(ctx), 1, 2, 128), 400 + step)
        flux.flux_kv_append_ring(cfg, k_ring, v_ring, ring_len, kn.cuda(), vn.cuda())
        case.append(kn, vn)
    lens = case.seq_len.cpu().tolist()
    assert ring_len.cpu().tolist() == lens
    _retained_equal(cfg, ring_rows, k_ring, case.k_host, lens)
    _retained_equal(cfg, ring_rows, v_ring, case.v_host, lens)
    assert flux.flux_get_device_status() == 0


@pytest.mark.parametrize("block,sink,window,ring_extra", [(64, 64, 256, 0), (128, 128, 512, 64),
                                                          (64, 0, 128, 0)])
def test_ring_decode_identical_to_full(block, sink, window, ring_extra):
    """Decode over the ring equals decode over the full cache bit for bit (same keys,
    same split plan) and the oracle within tolerance, across the ring's wrap-around."""
    cfg = AttnCfg(1, 8, 2, 128, block, sink, window)
    ring_rows = window + ring_extra
    ctx = [1, sink + 3, sink + window - 1, sink + window + 1, 3 * window + 17, 4000]
    case, k_ring, v_ring, ring_len = _ring_setup(cfg, ctx, ring_rows, seed=9)
    batch = len(ctx)
    mask = mask_words(batch, 1, [[] for _ in ctx]).cuda()
    ws = flux.new_decode_workspace(cfg, batch)
    for step in range(block + 3):   # crosses a block boundary and wraps the ring
        kn = inputs.normal_bf16((batch, 1, 2, 128), 500 + step)
        vn = inputs.normal_bf16((batch, 1, 2, 128), 600 + step)
        q = inputs.normal_bf16((batch, 8, 128), 700 + step).cuda()
        case.append(kn, vn)
        flux.flux_kv_append_ring(cfg, k_ring, v_ring, ring_len, kn.cuda(), vn.cuda())
        o_full = torch.empty(batch, 8, 128, dtype=torch.bfloat16, device="cuda")
        o_ring = torch.empty_like(o_full)
        flux.flux_decode(cfg, 0, mask, q, case.k, case.v, case.seq_len, o_full, ws)
        flux.flux_decode_ring(cfg, 0, mask, q, k_ring, v_ring, ring_len, o_ring, ws)
        torch.cuda.synchronize()
        assert torch.equal(o_ring, o_full), f"step {step}"
        if step % 16 == 0:
            want = oracle_layer(case, q.cpu()[:, None], [False] * batch)[:, 0]
            assert_close(f64(o_ring), want, f"ring decode step {step}")
    assert flux.flux_get_device_status() == 0


def test_ring_decode_refuses_fa_route():
    cfg = AttnCfg(1, 4, 1, 64, 64, 64, 64)
    k = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([100], dtype=torch.int32, device="cuda")
    mask = torch.ones(1, 1, dtype=torch.int32, device="cuda")  # layer 0 routed to FA
    ws = flux.new_decode_workspace(cfg, 1)
    o = torch.full((1, 4, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    flux.flux_decode_ring(cfg, 0, mask, torch.ones_like(o), k, k, seq, o, ws)
    assert flux.flux_get_device_status() & flux.FLUX_DEVICE_RING_ROUTE
    assert (o == 0).all()


def test_ring_decode_llama_full_size():
    """Llama-3.1-8B decode shape: 16 sequences at 32K context, an SA layer evicted to a
    2048-row ring (2176 rows per head instead of 33024): identical to the full cache."""
    w = configs.LLAMA_DECODE
    cfg = cfg_of(w)
    ctx = [w.seq] * w.batch
    case, k_ring, v_ring, ring_len = _ring_setup(cfg, ctx, w.window, seed=1002)
    mask = mask_words(w.batch, cfg.n_layers, [[] for _ in ctx]).cuda()
    ws = flux.new_decode_workspace(cfg, w.batch)
    for step in range(2):
        kn = inputs.normal_bf16((w.batch, 1, 8, 128), 800 + step)
        vn = inputs.normal_bf16((w.batch, 1, 8, 128), 900 + step)
        q = inputs.normal_bf16((w.batch, 32, 128), 1000 + step).cuda()
        case.append(kn, vn)
        flux.flux_kv_append_ring(cfg, k_ring, v_ring, ring_len, kn.cuda(), vn.cuda())
        o_full = torch.empty(w.batch, 32, 128, dtype=torch.bfloat16, device="cuda")
        o_ring = torch.empty_like(o_full)
        flux.flux_decode(cfg, 7, mask, q, case.k, case.v, case.seq_len, o_full, ws)
        flux.flux_decode_ring(cfg, 7, mask, q, k_ring, v_ring, ring_len, o_ring, ws)
        torch.cuda.synchronize()
        assert torch.equal(o_ring, o_full)
    want = oracle_layer(case, q.cpu()[:, None], [False] * w.batch)[:, 0]
    assert_close(f64(o_ring), want, "ring decode at 32K")


# --------------------------------------------------------- failure detection, chunks


def test_wait_timeout_selftest_reports_and_recovers():
    """A pipeline wait that nothing releases gives up after its limit, reports
    FLUX_DEVICE_TIMEOUT through the status word, and the context keeps working."""
    flux.flux_selftest_wait_timeout(2000)
    assert flux.flux_get_device_status() & flux.FLUX_DEVICE_TIMEOUT
    assert flux.flux_get_device_status() == 0  # read-and-clear
    cfg = AttnCfg(1, 4, 1, 64, 64, 64, 128)
    _decode_case(cfg, [300], [False], 1, seed=77)


@pytest.mark.parametrize("fa", [True, False])
def test_chunked_prefill_identical_to_one_shot(fa):
    """Qwen3-4B shape, 40000-token prompt in 16384-token chunks (Table 6's chunk size):
    bit-identical to the one-shot prefill, and within tolerance of the oracle."""
    from sparse_attention_layer_b200.runtime import HybridAttention
    w = configs.QWEN_PREFILL
    cfg = AttnCfg(1, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.sink, w.window)
    S = 40000
    q = inputs.normal_bf16((1, S, 32, 128), 1).cuda()
    k = inputs.normal_bf16((1, S, 8, 128), 2).cuda()
    v = inputs.normal_bf16((1, S, 8, 128), 3).cuda()
    mask = mask_words(1, 1, [[0] if fa else []]).cuda()
    outs = []
    for chunk in (None, 16384):
        m = HybridAttention(cfg, 1, S, "cuda")
        m.set_mask(mask)
        o = torch.empty_like(q)
        if chunk is None:
            m.prefill_layer(0, q, k, v, o)
        else:
            m.prefill_layer_chunked(0, q, k, v, o, chunk=chunk)
        outs.append(o)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    rows = np.array([0, 16383, 16384, 16385, 32767, 32768, S - 1, 20000])
    kc = k.cpu()[0].transpose(0, 1).float().numpy().astype(np.float64)[None]
    vc = v.cpu()[0].transpose(0, 1).float().numpy().astype(np.float64)[None]
    want = orc.attention_layer(q.cpu().float().numpy().astype(np.float64), kc, vc,
                               np.array([S]), np.array([fa]), cfg.block, cfg.sink, cfg.window,
                               rows=rows, heads=[0, 13])
    got = outs[1].cpu()[:, torch.as_tensor(rows)][:, :, torch.as_tensor([0, 13])]
    assert_close(f64(got), want, "chunked prefill")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("fa", [True, False])
def test_prefill_pages_sa_geometry(d, fa):
    """The pages' SA kernel geometry (Table 6): block 64, sink 128, with a 2048-token
    window, Llama heads, head_dim 64 and 128; sampled rows of a 6000-token prompt."""
    cfg = AttnCfg(1, 32, 8, d, 64, 128, 2048)
    rows = sample_rows(6000, 0, cfg, 24, seed=3)
    _prefill_case(cfg, [0], 6000, [fa], seed=1100 + d + fa, rows=rows, heads=[0, 9, 31])

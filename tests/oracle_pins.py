"""Pin checks for the oracle, written against an oracle-like namespace so that the
mutation test can run the same checks on deliberately broken copies.

Each check pins one oracle function to something other than itself: a library
attention routine (torch's scaled_dot_product_attention in float64), closed forms,
hand-derived golden values under tests/golden/, or invariants that follow from the
definitions.  Each returns None on success and raises AssertionError otherwise.
"""

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- attention core


def check_attention_vs_library(orc, seed=0):
    """masked_attention == torch SDPA (float64, boolean mask) on FA and SA masks,
    including GQA head sharing through attention_layer."""
    rng = _rng(seed)
    batch, n_q, hq, hkv, d, cap = 2, 96, 4, 2, 16, 128
    block, sink, window = 16, 16, 32
    seq = np.array([96, 120])
    q = rng.standard_normal((batch, n_q, hq, d))
    kc = rng.standard_normal((batch, hkv, cap, d))
    vc = rng.standard_normal((batch, hkv, cap, d))
    for is_fa in (True, False):
        got = orc.attention_layer(q, kc, vc, seq, np.array([is_fa, is_fa]), block, sink,
                                  window)
        for b in range(batch):
            n_keys = int(seq[b])
            t = np.arange(n_keys - n_q, n_keys)[:, None]
            j = np.arange(n_keys)[None, :]
            causal = j <= t
            if is_fa:
                m = causal
            else:
                # sink / window written with explicit block ranges, not the predicate
                m = np.zeros_like(causal)
                for r in range(n_q):
                    tt = n_keys - n_q + r
                    qb = tt // block
                    lo = max(0, (qb - window // block + 1) * block)
                    m[r, :min(sink, tt + 1)] = True
                    m[r, lo:tt + 1] = True
            qt = torch.from_numpy(q[b]).permute(1, 0, 2)          # [hq][n_q][d]
            kt = torch.from_numpy(kc[b, :, :n_keys]).repeat_interleave(hq // hkv, 0)
            vt = torch.from_numpy(vc[b, :, :n_keys]).repeat_interleave(hq // hkv, 0)
            ref = torch.nn.functional.scaled_dot_product_attention(
                qt, kt, vt, attn_mask=torch.from_numpy(m))
            ref = ref.permute(1, 0, 2).numpy()
            assert np.allclose(got[b], ref, atol=1e-12, rtol=1e-12), \
                f"attention differs from SDPA (fa={is_fa}, b={b})"


def check_attention_closed_forms(orc):
    rng = _rng(1)
    n, d = 40, 8
    k = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    mask = np.tril(np.ones((n, n), dtype=bool))
    # q = 0: every visible key weighs the same -> mean of the visible value rows
    o = orc.masked_attention(np.zeros((n, d)), k, v, mask)
    for t in range(n):
        assert np.allclose(o[t], v[:t + 1].mean(axis=0), atol=1e-13)
    # constant value rows -> that constant
    c = rng.standard_normal(d)
    o = orc.masked_attention(rng.standard_normal((n, d)), k, np.tile(c, (n, 1)), mask)
    assert np.allclose(o, np.tile(c, (n, 1)), atol=1e-13)
    # a single visible key -> its value row (row 0 of a causal mask)
    o = orc.masked_attention(rng.standard_normal((n, d)), k, v, mask)
    assert np.allclose(o[0], v[0], atol=1e-14)
    # two keys with a score gap of ln 3 -> weights 1/4, 3/4 (hand-derived)
    d2 = 4
    q2 = np.array([[math.log(3.0) * math.sqrt(d2), 0.0, 0.0, 0.0]])
    k2 = np.array([[0.0, 1.0, 0.0, 0.0], [1.0, 0.0, 0.0, 0.0]])
    v2 = np.array([[4.0, 0.0, 8.0, -4.0], [0.0, 4.0, -8.0, 4.0]])
    o = orc.masked_attention(q2, k2, v2, np.ones((1, 2), dtype=bool))
    assert np.allclose(o[0], [1.0, 3.0, -4.0, 2.0], atol=1e-13)
    # scale is 1/sqrt(d): scores q.k = sqrt(d) * ln 3 must give the same 1/4, 3/4
    d3 = 16
    q3 = np.zeros((1, d3)); q3[0, 0] = math.log(3.0) * math.sqrt(d3)
    k3 = np.zeros((2, d3)); k3[1, 0] = 1.0
    v3 = np.zeros((2, d3)); v3[0, 1] = 4.0; v3[1, 1] = 8.0
    o = orc.masked_attention(q3, k3, v3, np.ones((1, 2), dtype=bool))
    assert abs(o[0, 1] - (0.25 * 4.0 + 0.75 * 8.0)) < 1e-13


def check_softmax_rows(orc):
    rng = _rng(2)
    n, d = 64, 16
    q = rng.standard_normal((n, d)) * 3
    k = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    t = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    mask = orc.sa_key_visible(t, j, 8, 8, 16)
    _, p = orc.masked_attention(q, k, v, mask, return_probs=True)
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-12)
    assert (p[~mask] == 0).all() and (p[mask] > 0).all()


# ---------------------------------------------------------------- SA visibility


def check_sa_counts_golden(orc):
    data = _load("sa_visible_counts.json")
    for cfg in data["configs"]:
        for row in cfg["rows"]:
            t = row["t"]
            j = np.arange(t + 1)
            got = int(orc.sa_key_visible(t, j, cfg["block"], cfg["sink"],
                                         cfg["window"]).sum())
            assert got == row["count"], (cfg["name"], t, got, row["count"])


def check_sa_count_closed_form(orc):
    """|V(t)| = sink + (n_w - 1) * block + (t mod block) + 1 once the window has left
    the sink (qb >= n_sink + n_win); t + 1 before the first skipped block."""
    for block, sink, window in ((64, 64, 256), (128, 128, 2048), (64, 128, 256),
                                (16, 32, 48)):
        n_s, n_w = sink // block, window // block
        for t in range(0, (n_s + n_w + 6) * block, 7):
            got = int(orc.sa_key_visible(t, np.arange(t + 1), block, sink, window).sum())
            qb = t // block
            if qb >= n_s + n_w:
                want = sink + (n_w - 1) * block + (t % block) + 1
            else:
                want = t + 1
            assert got == want, (block, sink, window, t, got, want)


def check_sa_covers_fa(orc):
    """SA equals causal FA when sink + window reach back to key 0 for every row."""
    block, sink, window = 32, 32, 96
    n = (sink + window)  # n_s + n_w >= ceil(n / block)
    q_pos = np.arange(n)
    fa = orc.visible_mask(True, q_pos, n, block, sink, window)
    sa = orc.visible_mask(False, q_pos, n, block, sink, window)
    assert (fa == sa).all()
    # one block longer and SA must drop something
    n2 = n + block + 1
    q_pos = np.arange(n2)
    fa = orc.visible_mask(True, q_pos, n2, block, sink, window)
    sa = orc.visible_mask(False, q_pos, n2, block, sink, window)
    assert (sa <= fa).all() and (sa != fa).any()


def check_sa_token_reading_close(orc):
    """The alternative token-granular reading differs by fewer than block keys/row."""
    block, sink, window = 64, 64, 256
    for t in range(0, 2048, 13):
        j = np.arange(t + 1)
        a = orc.sa_key_visible(t, j, block, sink, window)
        b = orc.sa_key_visible_token_granular(t, j, sink, window)
        assert abs(int(a.sum()) - int(b.sum())) < block
        assert a[: min(sink, t + 1)].all() and a[t]


def check_sa_key_blocks(orc):
    """Visible key-block sets of whole query blocks: sink blocks plus the n_w blocks
    ending at the query block (hand-stated for the tiny and Llama geometries)."""
    for block, sink, window in ((64, 64, 256), (128, 128, 2048)):
        n_s, n_w = sink // block, window // block
        n_kb = 40
        for qb in range(n_kb):
            got = orc.sa_visible_key_blocks(qb, n_kb, block, sink, window)
            want = set(range(min(n_s, qb + 1))) | set(range(max(0, qb - n_w + 1), qb + 1))
            assert got == want, (block, qb, sorted(got), sorted(want))


def check_key_tiles_of_rows(orc):
    """Key tiles visited / masked for a run of query rows: the FA closed form (tiles up to
    the last row's, masked where a key passes the first row), agreement with the key-block
    sets of whole query blocks when tile == block, and two hand-worked SA examples."""
    for t_min, t_max, tile in ((0, 127, 128), (1000, 1127, 128), (5, 5, 64), (300, 427, 64)):
        vis, msk = orc.key_tiles_of_rows(True, np.arange(t_min, t_max + 1), tile, 64, 64, 256)
        assert vis == list(range(t_max // tile + 1))
        assert msk == [kt for kt in vis if kt * tile + tile - 1 > t_min]
    for block, sink, window in ((64, 64, 256), (128, 128, 2048), (64, 0, 64)):
        for qb in (0, 1, 3, 7, 20, 33):
            rows = np.arange(qb * block, (qb + 1) * block)
            vis, _ = orc.key_tiles_of_rows(False, rows, block, block, sink, window)
            assert set(vis) == orc.sa_visible_key_blocks(qb, qb + 1, block, sink, window)
    # block 64, sink 128, window 256, rows 1000..1127, 128-key tiles: sink keys [0, 128),
    # row 1000 sees from key 768 (block 12), row 1127 from key 896 (block 14)
    assert orc.key_tiles_of_rows(False, np.arange(1000, 1128), 128, 64, 128, 256) == \
        ([0, 6, 7, 8], [6, 7, 8])
    # block 64, sink 64, window 128: sink keys [0, 64) (keys 64..127 of tile 0 hidden),
    # row 1000 sees from key 896, row 1127 from key 1024
    assert orc.key_tiles_of_rows(False, np.arange(1000, 1128), 128, 64, 64, 128) == \
        ([0, 7, 8], [0, 7, 8])


# ---------------------------------------------------------------- decode, append


def check_decode_is_prefill_row(orc):
    rng = _rng(3)
    batch, hq, hkv, d, cap = 2, 4, 2, 8, 80
    block, sink, window = 8, 8, 16
    kc = rng.standard_normal((batch, hkv, cap, d))
    vc = rng.standard_normal((batch, hkv, cap, d))
    seq = np.array([70, 33])
    n_q = 33
    q = rng.standard_normal((batch, n_q, hq, d))
    for is_fa in (True, False):
        bits = np.array([is_fa, is_fa])
        full = orc.attention_layer(q, kc, vc, seq, bits, block, sink, window)
        dec = orc.decode_attention(q[:, -1], kc, vc, seq, bits, block, sink, window)
        assert np.allclose(dec, full[:, -1], atol=1e-13, rtol=0)
        # and the decode row sees exactly key positions <= seq_len - 1
        kc2 = kc.copy(); kc2[:, :, int(seq.max()):] = 1e6
        dec2 = orc.decode_attention(q[:, -1], kc2, vc, seq, bits, block, sink, window)
        assert np.allclose(dec, dec2, atol=1e-13, rtol=0)


def check_kv_append(orc):
    rng = _rng(4)
    batch, hkv, cap, d, n = 3, 2, 10, 4, 3
    kc = rng.standard_normal((batch, hkv, cap, d))
    vc = rng.standard_normal((batch, hkv, cap, d))
    seq = np.array([0, 5, 8])
    kn = rng.standard_normal((batch, n, hkv, d))
    vn = rng.standard_normal((batch, n, hkv, d))
    k2, v2, s2, over = orc.kv_append(kc, vc, seq, kn, vn)
    assert list(s2) == [3, 8, 8] and list(over) == [False, False, True]
    assert np.array_equal(k2[0, 1, 0:3], kn[0, :, 1]) and np.array_equal(v2[1, 0, 5:8], vn[1, :, 0])
    assert np.array_equal(k2[2], kc[2]) and np.array_equal(k2[0, :, 3:], kc[0, :, 3:])


# ---------------------------------------------------------------- router


def check_router_golden(orc):
    g = _load("router_toy.json")
    xq = np.array(g["xq"], dtype=np.float64)
    w1, b1 = np.array(g["w1"], float), np.array(g["b1"], float)
    w2, b2 = np.array(g["w2"], float), np.array(g["b2"], float)
    for case in g["cases"]:
        idx = orc.pool_token_indices(xq.shape[1], case["pool_len"])
        assert list(idx) == case["pooled_tokens"]
        res = orc.router(xq, w1, b1, w2, b2, case["pool_len"], g["tau"])
        assert np.allclose(res["logits"], case["logits"], atol=1e-9)
        assert (res["fa_bits"].astype(int) == np.array(case["fa_bits"])).all()
        assert res["fa_mask"].tolist() == case["mask_words"]
        if "omega_msr" in case:
            assert np.allclose(orc.omega_msr(res["fa_bits"]), case["omega_msr"])
    pk = g["packing"]
    bits = np.zeros((1, pk["n_layers"]), dtype=bool)
    bits[0, pk["fa_layers"]] = True
    assert orc.pack_fa_mask(bits)[0].tolist() == pk["mask_words"]


def check_pool_indices(orc):
    assert list(orc.pool_token_indices(8192, 100)) == list(range(50)) + list(range(8142, 8192))
    assert list(orc.pool_token_indices(10, 5)) == [0, 1, 2, 8, 9]
    assert list(orc.pool_token_indices(7, 100)) == list(range(7))
    assert list(orc.pool_token_indices(7, 0)) == list(range(7))
    # the pooled mean of a ramp x_t = t is the mean of the chosen positions
    xq = np.arange(1000, dtype=float).reshape(1, 1000, 1)
    want = (sum(range(50)) + sum(range(950, 1000))) / 100.0
    assert orc.router_pool(xq, 100)[0, 0] == want


def check_omega_pages(orc):
    g = _load("omega_msr_pages.json")
    for row in g["rows"]:
        bits = np.ones((1, g["n_layers"]), dtype=bool)
        bits[0, : row["n_sa_layers"]] = False
        assert round(float(orc.omega_msr(bits)[0]), 3) == row["printed"]


def check_router_error_bound(orc):
    """The fp64 bound really bounds an fp32 evaluation (which it must exceed by the
    ratio of unit roundoffs) and the fp32 bound covers a float32 numpy evaluation."""
    rng = _rng(5)
    xq = rng.standard_normal((2, 300, 64)).astype(np.float32).astype(np.float64)
    w1 = (rng.standard_normal((16, 64)) * 0.02).astype(np.float32).astype(np.float64)
    w2 = (rng.standard_normal((5, 16)) * 0.02).astype(np.float32).astype(np.float64)
    b1 = np.zeros(16); b2 = np.zeros(5)
    exact = orc.router(xq, w1, b1, w2, b2, 100, 0.0)["logits"]
    idx = orc.pool_token_indices(300, 100)
    p32 = xq[:, idx, :].astype(np.float32).mean(axis=1, dtype=np.float32)
    h32 = np.maximum(p32 @ w1.T.astype(np.float32), np.float32(0))
    z32 = (h32 @ w2.T.astype(np.float32)).astype(np.float64)
    bound32 = orc.router_error_bound(xq, w1, b1, w2, b2, 100, 2.0 ** -24)
    bound64 = orc.router_error_bound(xq, w1, b1, w2, b2, 100)
    assert (np.abs(z32 - exact) <= bound32).all()
    assert (bound64 < bound32 * 2.0 ** -28).all()


def check_ring_keeps_every_visible_key(orc):
    """For every length T, the keys an SA decode query at T - 1 can see are all retained
    by a ring of `window` rows, each in a slot of its own (no retained key is evicted
    while still visible); a ring one row shorter loses one for some T."""
    for block, sink, window in ((64, 64, 256), (128, 128, 2048), (64, 0, 128), (64, 128, 64)):
        for T in range(1, sink + 3 * window + 2 * block, 5 if window > 512 else 1):
            vis = np.nonzero(orc.sa_key_visible(T - 1, np.arange(T), block, sink, window))[0]
            kept = set(orc.ring_retained_positions(T, sink, window).tolist())
            assert set(vis.tolist()) <= kept, (block, sink, window, T)
            slots = orc.ring_slot(vis, sink, window)
            assert len(set(slots.tolist())) == len(vis)
        lost = False
        for T in range(1, sink + 3 * window + 2 * block):
            vis = np.nonzero(orc.sa_key_visible(T - 1, np.arange(T), block, sink, window))[0]
            if not set(vis.tolist()) <= set(orc.ring_retained_positions(T, sink, window - 1).tolist()):
                lost = True
                break
        assert lost, (block, sink, window)


def check_ring_placement_hand_example(orc):
    """sink 2, ring 3, 9 positions written: slots 0, 1 hold positions 0, 1; the ring
    holds positions 6, 7, 8 at slots 2 + (6-2)%3 = 3, 2 + 5%3 = 4, 2 + 6%3 = 2."""
    assert orc.ring_slot([0, 1, 2, 3, 4, 5, 6, 7, 8], 2, 3).tolist() == [0, 1, 2, 3, 4, 2, 3, 4, 2]
    assert orc.ring_retained_positions(9, 2, 3).tolist() == [0, 1, 6, 7, 8]
    k = np.arange(9, dtype=float).reshape(1, 1, 9, 1) + 1
    kr, vr = orc.kv_compact_ring(k, k, np.array([9]), 2, 3)
    assert kr[0, 0, :, 0].tolist() == [1, 2, 9, 7, 8]
    # appending position 9 overwrites slot 2 + 7 % 3 = 3 (position 6, no longer needed)
    k2, v2, s2 = orc.kv_append_ring(kr, vr, np.array([9]), np.full((1, 1, 1, 1), 10.0),
                                    np.full((1, 1, 1, 1), 10.0), 2, 3)
    assert k2[0, 0, :, 0].tolist() == [1, 2, 9, 10, 8] and s2.tolist() == [10]


ALL_CHECKS = [
    check_attention_vs_library, check_attention_closed_forms, check_softmax_rows,
    check_sa_counts_golden, check_sa_count_closed_form, check_sa_covers_fa,
    check_sa_token_reading_close, check_sa_key_blocks, check_key_tiles_of_rows,
    check_decode_is_prefill_row,
    check_kv_append, check_router_golden, check_pool_indices, check_omega_pages,
    check_router_error_bound, check_ring_keeps_every_visible_key,
    check_ring_placement_hand_example,
]

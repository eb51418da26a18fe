"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the pin
suite catches every one of them: a dropped term, a wrong sign or index, a swapped
operand.  The real oracle module is never modified."""

import inspect
import types

import pytest

from oracle import flux_oracle as orc
from tests import oracle_pins as pins

MUTATIONS = {
    "drop_softmax_scale": ("(q @ k.T) / math.sqrt(d)", "(q @ k.T)"),
    "causal_strict": ('"""Causal full attention: key j is visible from query position t iff j <= t."""\n    return j <= t',
                      '"""Causal full attention: key j is visible from query position t iff j <= t."""\n    return j < t'),
    "window_off_by_one": ("(jb >= qb - n_win + 1)", "(jb >= qb - n_win)"),
    "sink_off_by_one": ("(jb < n_sink)", "(jb <= n_sink)"),
    "no_causality_in_sa": ("return (j <= t) & ((jb < n_sink) | (jb >= qb - n_win + 1))",
                           "return ((jb < n_sink) | (jb >= qb - n_win + 1))"),
    "gqa_modulo_mapping": ("kvh = h // group", "kvh = h % n_kvh"),
    "value_operand_swapped": ("out = probs @ v", "out = probs @ k"),
    "query_positions_from_zero": ("q_pos = n_keys - n_q + rows", "q_pos = rows"),
    "pool_prefix_short": ("n_prefix = (pool_len + 1) // 2", "n_prefix = pool_len // 2"),
    "pool_first_tokens_only": ("np.arange(seq_len - n_suffix, seq_len, dtype=np.int64)",
                               "np.arange(n_prefix, n_prefix + n_suffix, dtype=np.int64)"),
    "router_no_relu": ("hidden = np.maximum(pooled @ w1.T + b1, 0.0)\n    return hidden",
                       "hidden = pooled @ w1.T + b1\n    return hidden"),
    "router_drop_bias2": ("return hidden @ w2.T + b2", "return hidden @ w2.T"),
    "tie_goes_to_fa": ("return logits > tau", "return logits >= tau"),
    "pack_wrong_word": ("out[b, layer // 32] |=", "out[b, 0] |="),
    "omega_counts_fa": ("return 1.0 - fa_bits.sum(axis=-1) / n_layers",
                        "return fa_bits.sum(axis=-1) / n_layers"),
    "append_off_by_one": ("k_out[b, :, start + i, :] = k_new[b, i]",
                          "k_out[b, :, start + i + 1, :] = k_new[b, i]"),
    "append_no_advance": ("len_out[b] = start + n_new", "len_out[b] = start"),
    "ring_slot_offset": ("sink + (p - sink) % ring_rows)", "(p - sink) % ring_rows)"),
    "tile_mask_never": ("if not per_tile[:, kt, :].all()]", "if not per_tile[:, kt, :].any()]"),
    "tile_visit_misses_last": ("n_tiles = int(q_pos.max()) // tile + 1",
                               "n_tiles = int(q_pos.max()) // tile"),
    "ring_keeps_too_few": ("np.arange(max(sink, seq_len - ring_rows), seq_len",
                           "np.arange(max(sink, seq_len - ring_rows + 1), seq_len"),
}


def _mutant(old, new):
    src = inspect.getsource(orc)
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mod = types.ModuleType("flux_oracle_mutant")
    exec(compile(src.replace(old, new), "flux_oracle_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name):
    mod = _mutant(*MUTATIONS[name])
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(mod)
        except Exception:  # noqa: BLE001 - any failure counts as caught
            caught.append(check.__name__)
    assert caught, f"no pin catches mutation {name}"

"""tests/golden/router_seeds.json is reproducible from the oracle alone: rerunning the
seed search of tests/golden/make_router_seeds.py for the Llama prefill workload gives
the stored seed, layer count, Omega_MSR and bits.  CPU only (the Qwen entry, whose x_Q
is 131072 x 2560, is checked at full size against the GPU router in the parity tests)."""

import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_llama_router_seed_reproduces():
    spec = importlib.util.spec_from_file_location(
        "make_router_seeds", os.path.join(ROOT, "tests", "golden", "make_router_seeds.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    from sparse_attention_layer_b200.configs import LLAMA_PREFILL
    got = mod.search(LLAMA_PREFILL)
    with open(os.path.join(ROOT, "tests", "golden", "router_seeds.json")) as f:
        want = json.load(f)[LLAMA_PREFILL.name]
    for key in ("router_seed", "n_sa_layers", "omega_msr", "pooled_tokens", "fa_bits"):
        assert got[key] == want[key], key
    assert got["min_margin_over_fp64_bound"] > 1000.0


def test_workload_seed_constants_match_the_record():
    """The workload definitions carry the recorded seeds as constants (the product
    package never reads the test tree)."""
    from sparse_attention_layer_b200 import configs
    with open(os.path.join(ROOT, "tests", "golden", "router_seeds.json")) as f:
        rec = json.load(f)
    for w in (configs.LLAMA_PREFILL, configs.QWEN_PREFILL):
        assert w.router_seed == rec[w.name]["router_seed"], w.name
        assert w.target_sa_layers == rec[w.name]["n_sa_layers"], w.name

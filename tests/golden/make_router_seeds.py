"""Write tests/golden/router_seeds.json: for each routed prefill workload, the first
router seed (0, 1, 2, ...) whose hard decisions put exactly the target number of
layers on SA, with every logit farther from tau than the fp64 error bound (the library
accumulates the router in fp64, so both sides decide in the same precision).

Calls only the oracle (and the seeded input generators); no GPU, no CUDA library.
Run from the repository root:  python tests/golden/make_router_seeds.py
"""

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import flux_oracle as orc  # noqa: E402
from sparse_attention_layer_b200 import inputs  # noqa: E402
from sparse_attention_layer_b200.configs import LLAMA_PREFILL, QWEN_PREFILL  # noqa: E402


def boundary_xq(w):
    xq = inputs.normal_bf16((w.batch, w.seq, w.router_hidden),
                            inputs.layer_seed(w.data_seed, 0, inputs.XQ))
    idx = orc.pool_token_indices(w.seq, w.pool_len)
    # only the pooled rows enter the router; keep them (exact bf16 values) as float64
    return xq[:, idx, :].float().numpy().astype(np.float64), len(idx)


def search(w, max_seed=500):
    xb, n_idx = boundary_xq(w)
    for seed in range(max_seed):
        w1, b1, w2, b2 = (t.float().numpy().astype(np.float64)
                          for t in inputs.router_weights(w.router_hidden, w.router_rank,
                                                         w.n_layers, seed))
        # xb already holds only the pooled rows, so pool it whole (pool_len = 0)
        res = orc.router(xb, w1, b1, w2, b2, 0, w.tau)
        bound = orc.router_error_bound(xb, w1, b1, w2, b2, 0)
        n_sa = int((~res["fa_bits"]).sum())
        margin = float((np.abs(res["logits"] - w.tau) / bound).min())
        if n_sa == w.target_sa_layers and margin > 1000.0:
            return {"router_seed": seed, "n_sa_layers": n_sa,
                    "omega_msr": float(orc.omega_msr(res["fa_bits"])[0]),
                    "min_margin_over_fp64_bound": margin,
                    "pooled_tokens": n_idx,
                    "fa_bits": [int(x) for x in res["fa_bits"][0]]}
    raise RuntimeError(f"no seed below {max_seed} for {w.name}")


def main():
    out = {}
    for w in (LLAMA_PREFILL, QWEN_PREFILL):
        out[w.name] = search(w)
        print(w.name, out[w.name]["router_seed"], out[w.name]["n_sa_layers"])
    path = os.path.join(ROOT, "tests", "golden", "router_seeds.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()

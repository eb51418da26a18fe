"""Small, self-contained launches of one kernel for profiling (ncu) and quick timing.

    python -m sparse_attention_layer_b200.profile_case prefill [--sa] [--launches N]
    python -m sparse_attention_layer_b200.profile_case decode [--sa] [--batch B]

prefill: one Llama-3.1-8B-shaped layer, 8192-token prompt (Q 64 MB, K/V 16 MB each,
         O 64 MB: more than the 126 MB L2 together), FA route unless --sa.
decode:  one Llama-shaped layer, `batch` sequences at 32768 context (K+V 134 MB per
         sequence), FA route unless --sa; each launch is the decode step's
         flux_decode_append (the new row is appended, so launch i attends 32769 + i keys,
         as the bench's decode steps do).
Each launch is timed with CUDA events; the script prints one JSON line.
"""

from __future__ import annotations

import argparse
import json

import torch

from . import flux, inputs
from .flux import AttnCfg
from .runtime import HybridAttention


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["prefill", "decode"])
    ap.add_argument("--sa", action="store_true")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--seq", type=int, default=0)
    args = ap.parse_args()
    torch.cuda.set_device(0)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    cfg = AttnCfg(1, 32, 8, 128, 128, 128, 2048)
    bits = inputs.fa_bits_from_sa_layers(1 if args.kernel == "prefill" else args.batch, 1,
                                         [0] if args.sa else [])
    times = []
    if args.kernel == "prefill":
        S = args.seq or 8192
        m = HybridAttention(cfg, 1, S, "cuda")
        m.set_mask(inputs.pack_bits_u32(bits).cuda())
        q = torch.randn(1, S, 32, 128, device="cuda", generator=gen).to(torch.bfloat16)
        k = torch.randn(1, S, 8, 128, device="cuda", generator=gen).to(torch.bfloat16)
        v = torch.randn(1, S, 8, 128, device="cuda", generator=gen).to(torch.bfloat16)
        o = torch.empty_like(q)
        c = m.caches[0]
        flux.flux_kv_append(cfg, c.k, c.v, c.seq_len, k, v)
        for _ in range(args.launches):
            a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
            a.record()
            flux.flux_prefill(cfg, 0, m.fa_mask, q, c.k, c.v, c.seq_len, o)
            b.record()
            times.append((a, b))
        n_units = S
    else:
        T = args.seq or 32768
        B = args.batch
        m = HybridAttention(cfg, B, T + args.launches, "cuda")
        m.set_mask(inputs.pack_bits_u32(bits).cuda())
        c = m.caches[0]
        c.k.normal_(generator=gen)
        c.v.normal_(generator=gen)
        c.seq_len.fill_(T)
        q = torch.randn(B, 32, 128, device="cuda", generator=gen).to(torch.bfloat16)
        kn = torch.randn(B, 1, 8, 128, device="cuda", generator=gen).to(torch.bfloat16)
        o = torch.empty_like(q)
        for _ in range(args.launches):
            a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
            a.record()
            flux.flux_decode_append(cfg, 0, m.fa_mask, q, kn, kn, c.k, c.v, c.seq_len, o,
                                    m.workspace)
            b.record()
            times.append((a, b))
        n_units = B
    torch.cuda.synchronize()
    status = flux.flux_get_device_status()
    ms = [a.elapsed_time(b) for a, b in times]
    print(json.dumps({"kernel": args.kernel, "route": "SA" if args.sa else "FA", "ms": ms,
                      "units": n_units, "status": status}))
    if status:
        raise SystemExit(f"device status {status:#x}")


if __name__ == "__main__":
    main()

"""Benchmark of the hybrid-attention hot path (Flux Attention: layer router + FA/SA
prefill + FA/SA decode) on B200.

Main line (`value`): decode tokens/s of the Llama-3.1-8B attention shape serving 16
sequences at a 32768-token context, 32 layers of which a fixed seeded 16 run SA
(sink 128 + window 2048, block 128).  One step = one decode token for every sequence:
per layer one launch that appends the token's K/V row and runs the FA- or SA-routed
split-KV decode (flux_decode_append), the 32 layers captured once as a CUDA graph and
replayed per step.  The per-route rooflines time the same launches replayed as a graph
of one route's layers.  The same run times:
  * prefill: router + 32 x (KV append + FA/SA prefill) of an 8192-token Llama-shaped
    prompt with router-chosen routes, its FA and SA prefill rooflines, and the prefill
    step at every SA-layer fraction of the routing mix;
  * the Qwen3-4B-shaped 131072-token prefill (36 layers, router-chosen 22 SA, window
    4096);
  * the decode step at every SA-layer fraction, decode after SA-layer KV eviction, the
    pages' SA geometry (block 64, sink 128) at head_dim 64 and 128, and a compact
    context x batch x routing-mix sweep.
Protocol: W warm-up then K timed steps (default 10 and 50), CUDA events on the
launching stream, barrier + synchronize around the timed region, max over ranks.

`--impl reference` times the fp64 CPU oracle on the host cores instead, on a bounded
sample of the same decode workload, and prints the same metric.  `--sweep` runs the
full context x batch x routing-mix sweep.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl flux|reference]
Multi-GPU (replicas, no data-path collective):
  python -m torch.distributed.run --nproc-per-node N --master-addr 127.0.0.1 bench.py --gpus N
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "hybrid-attn prefill & decode tokens/s at 32K ctx; % of tensor/HBM roofline"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (DGX figure)


# ------------------------------------------------------------------------ helpers


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"flux_clocks_{os.getpid()}_{id(self)}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.remove(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def measured_traffic(kernel: str, units: float):
    """DRAM bytes per launch of `kernel` scaled from the committed ncu capture in
    profiles/traffic.txt to `units` (sequences for decode, prompts for prefill); None
    when the capture is missing or the kernel's sources changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            kv = dict(line.split(" = ", 1) for line in f.read().splitlines()
                      if " = " in line and not line.startswith("#"))
        for item in kv[f"{kernel}.sources"].split():
            rel, digest = item.split(":")
            with open(os.path.join(ROOT, "sparse_attention_layer_b200", rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest()[:16] != digest:
                    return None
        return float(kv[f"{kernel}.bytes"]) / float(kv[f"{kernel}.units"]) * units
    except (OSError, KeyError, ValueError):
        return None


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if world != n_gpus:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE {world}", file=sys.stderr)
    return world, rank, local


def barrier(world, device="cuda"):
    if world > 1:
        torch.distributed.barrier()
    if device == "cuda":
        torch.cuda.synchronize()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """Largest value over the ranks (the slowest rank's time decides a replica run)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_tokens_per_s(world: int, tokens_per_rank: int, steps: int, t_ms: float) -> float:
    """Whole-job throughput of N independent replicas: every rank processes its own
    tokens_per_rank per step; the job takes as long as its slowest rank (t_ms)."""
    return world * tokens_per_rank * steps / (t_ms / 1e3)


def host_cores() -> int:
    """Cores this process may run on (what nproc reports)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_threads() -> int:
    try:
        import threadpoolctl
        import numpy  # noqa: F401
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return os.cpu_count() or 1


def graph_ms(graph, warm: int, reps: int, reset=None) -> float:
    """Median time of one replay of `graph` (CUDA events on the current stream); `reset`
    runs before every replay (outside the timed interval)."""
    for _ in range(warm):
        if reset:
            reset()
        graph.replay()
    times = []
    for _ in range(reps):
        if reset:
            reset()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        graph.replay()
        b.record()
        times.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in times)


# ------------------------------------------------------------------- workloads


def decode_geometry():
    from sparse_attention_layer_b200 import configs
    from sparse_attention_layer_b200.flux import AttnCfg
    w = configs.LLAMA_DECODE
    cfg = AttnCfg(w.n_layers, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.sink, w.window)
    return w, cfg


def visible_keys(cfg, T: int, fa: bool) -> int:
    """Keys a decode query at position T - 1 sees (T keys in the sequence)."""
    if fa:
        return T
    t = T - 1
    qb = t // cfg.block
    win_lo = max(0, (qb - cfg.window // cfg.block + 1) * cfg.block)
    return (T - win_lo) + min(cfg.sink, win_lo)


def decode_bytes_per_layer(w, cfg, T: int, fa: bool, append: bool = False) -> int:
    """Algorithmic bytes of one decode launch: K and V rows of every visible key plus q
    in and o out, for all sequences (T = keys after the append); with append, also the
    new K/V row written into the cache."""
    kv = 2 * 2 * w.batch * cfg.n_kv_heads * cfg.head_dim * visible_keys(cfg, T, fa)
    qo = 2 * 2 * w.batch * cfg.n_q_heads * cfg.head_dim
    new_rows = 2 * 2 * w.batch * cfg.n_kv_heads * cfg.head_dim if append else 0
    return kv + qo + new_rows


def prefill_flops_per_layer(cfg, S: int, fa: bool) -> float:
    """Algorithmic flops of one prefill launch (batch 1): 4 d Hq per visible pair."""
    total = 0
    for t in range(S):
        if fa:
            total += t + 1
        else:
            qb = t // cfg.block
            win_lo = max(0, (qb - cfg.window // cfg.block + 1) * cfg.block)
            total += (t + 1 - win_lo) + min(cfg.sink, win_lo)
    return 4.0 * cfg.head_dim * cfg.n_q_heads * total


def tensor_roofline(kernel: str, flops: float, launch_ms: float, peaks, peak_kind: str,
                    clocks: dict, traffic=None) -> dict:
    """Tensor-bound roofline line: fraction of the burst bf16 peak (the launches are timed
    inside a phase of well under a second), the sustained peak beside it."""
    tflops = flops / (launch_ms / 1e3) / 1e12
    return {"bound": "tensor", "kernel": kernel, "achieved": tflops,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
            "peak_kind": f"{peak_kind} bf16_tflops (burst)",
            "frac_of_sustained_peak": tflops / peaks["bf16_tflops_sustained"],
            "traffic": traffic, "launch_ms": launch_ms, "algorithmic_flops_per_launch": flops,
            "phase_clocks_sm_mhz": clocks.get("sm_mhz"), "phase_clock_reasons": clocks.get("reasons")}


def hbm_roofline(kernel: str, nbytes: float, launch_ms: float, peaks, peak_kind: str,
                 traffic=None, timing: str = "") -> dict:
    gbs = nbytes / (launch_ms / 1e3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": gbs, "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "peak_kind": f"{peak_kind} hbm_gbs",
            "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
            "peak_note": "the measured peak is a copy (read + write); read-only streaming "
                         "can exceed it",
            "traffic": traffic, "launch_us": launch_ms * 1e3,
            "algorithmic_bytes_per_launch": nbytes, "timing": timing}


class DecodeBench:
    """Llama-shape decode at 32K context: 32 layers of KV cache resident in HBM."""

    def __init__(self, seed: int):
        from sparse_attention_layer_b200 import configs, inputs
        from sparse_attention_layer_b200.runtime import HybridAttention
        self.w, self.cfg = decode_geometry()
        w, cfg = self.w, self.cfg
        self.model = HybridAttention(cfg, w.batch, w.capacity(), "cuda")
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        for c in self.model.caches:
            c.k[:, :, :w.seq].normal_(generator=gen)
            c.v[:, :, :w.seq].normal_(generator=gen)
        self.ctx = w.seq
        self.sa_layers = inputs.fixed_sa_layers(w.n_layers, w.target_sa_layers,
                                                configs.LLAMA_DECODE_MASK_SEED)
        self.set_sa_layers(self.sa_layers)
        L, B = w.n_layers, w.batch
        self.q = torch.randn(L, B, cfg.n_q_heads, cfg.head_dim, device="cuda",
                             generator=gen).to(torch.bfloat16)
        self.k_new = torch.randn(L, B, 1, cfg.n_kv_heads, cfg.head_dim, device="cuda",
                                 generator=gen).to(torch.bfloat16)
        self.v_new = torch.randn(L, B, 1, cfg.n_kv_heads, cfg.head_dim, device="cuda",
                                 generator=gen).to(torch.bfloat16)
        self.o = torch.empty(L, B, cfg.n_q_heads, cfg.head_dim, dtype=torch.bfloat16,
                             device="cuda")

    def set_sa_layers(self, sa_layers):
        from sparse_attention_layer_b200 import inputs
        bits = inputs.fa_bits_from_sa_layers(self.w.batch, self.w.n_layers, sa_layers)
        self.fa = [bool(bits[0, i]) for i in range(self.w.n_layers)]
        self.model.set_mask(inputs.pack_bits_u32(bits).cuda())

    def reset(self):
        for c in self.model.caches:
            c.seq_len.fill_(self.ctx)

    def layers_graph(self, layers):
        """The decode launches of `layers` (in order) captured as one CUDA graph."""
        m = self.model
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for layer in layers:
                m.decode_layer(layer, self.q[layer], self.k_new[layer], self.v_new[layer],
                               self.o[layer])
        return g

    # kernels of this library per step: one append + decode launch per layer
    launches_per_step = property(lambda self: self.w.n_layers)


class PrefillBench:
    """Prefill of one prompt: router on x_Q, then per layer KV append + FA/SA prefill.
    Layers have separate caches; q/k/v inputs are shared by the layers (the work does
    not depend on their values)."""

    def __init__(self, w, seed: int):
        from sparse_attention_layer_b200 import inputs
        from sparse_attention_layer_b200.flux import AttnCfg
        from sparse_attention_layer_b200.runtime import HybridAttention
        self.w = w
        self.cfg = AttnCfg(w.n_layers, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.sink,
                           w.window)
        self.model = HybridAttention(self.cfg, w.batch, w.seq, "cuda")
        w1, b1, w2, b2 = inputs.router_weights(w.router_hidden, w.router_rank, w.n_layers,
                                               w.router_seed)
        self.router = [t.cuda() for t in (w1, b1, w2, b2)]
        self.xq = inputs.normal_bf16((w.batch, w.seq, w.router_hidden),
                                     inputs.layer_seed(w.data_seed, 0, inputs.XQ)).cuda()
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        B, S = w.batch, w.seq
        self.q = torch.randn(B, S, w.n_q_heads, w.head_dim, device="cuda",
                             generator=gen).to(torch.bfloat16)
        self.k = torch.randn(B, S, w.n_kv_heads, w.head_dim, device="cuda",
                             generator=gen).to(torch.bfloat16)
        self.v = torch.randn(B, S, w.n_kv_heads, w.head_dim, device="cuda",
                             generator=gen).to(torch.bfloat16)
        self.o = torch.empty(B, S, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
        # route once to learn the mask (the timed steps route again)
        self.model.route(*self.router, self.xq, w.pool_len, w.tau)
        self.router_mask = self.model.fa_mask.clone()
        self.fa = self.mask_bits(self.router_mask)

    def mask_bits(self, mask):
        words = mask.cpu()[0]
        return [bool((int(words[i // 32]) >> (i % 32)) & 1) for i in range(self.w.n_layers)]

    def reset(self):
        for c in self.model.caches:
            c.seq_len.zero_()

    def step(self, route=True, fa_events=None, sa_events=None, router_events=None,
             append_events=None):
        """router (optional) + every layer's KV append and prefill; with *_events, the
        FA / SA prefill launches, the appends and the router are bracketed by CUDA
        events."""
        from sparse_attention_layer_b200 import flux
        m, w = self.model, self.w

        def ev():
            return torch.cuda.Event(enable_timing=True)
        if route:
            if router_events is not None:
                e0, e1 = ev(), ev()
                e0.record()
            m.route(*self.router, self.xq, w.pool_len, w.tau)
            if router_events is not None:
                e1.record()
                router_events.append((e0, e1))
        for layer in range(w.n_layers):
            c = m.caches[layer]
            if append_events is not None:
                a0, a1 = ev(), ev()
                a0.record()
            flux.flux_kv_append(self.cfg, c.k, c.v, c.seq_len, self.k, self.v)
            if append_events is not None:
                a1.record()
                append_events.append((a0, a1))
            events = fa_events if self.fa[layer] else sa_events
            if events is not None:
                e0, e1 = ev(), ev()
                e0.record()
            flux.flux_prefill(self.cfg, layer, m.fa_mask, self.q, c.k, c.v, c.seq_len, self.o)
            if events is not None:
                e1.record()
                events.append((e0, e1))

    # route 1, per layer: append copy + length update, prefill
    launches_per_step = property(lambda self: 1 + self.w.n_layers * 3)


def elapsed_ms(pairs):
    return [a.elapsed_time(b) for a, b in pairs]


# ---------------------------------------------------------------- CPU baseline


def cpu_oracle_decode_sample(n_seq: int = 1, seed: int = 5):
    """Time the fp64 oracle on one decode step of n_seq sequences of the 32K decode
    workload, for one FA and one SA layer; returns seconds per layer-step per sequence."""
    import numpy as np

    from oracle import flux_oracle as orc
    from sparse_attention_layer_b200 import inputs
    w, cfg = decode_geometry()
    T = w.seq + 1
    shape = (n_seq, cfg.n_kv_heads, T, cfg.head_dim)
    kc = inputs.normal_bf16(shape, seed).float().numpy().astype(np.float64)
    vc = inputs.normal_bf16(shape, seed + 1).float().numpy().astype(np.float64)
    q = inputs.normal_bf16((n_seq, cfg.n_q_heads, cfg.head_dim), seed + 2).float().numpy().astype(np.float64)
    lens = np.full(n_seq, T)
    out = {}
    for fa in (True, False):
        t0 = time.perf_counter()
        orc.decode_attention(q, kc, vc, lens, np.full(n_seq, fa), cfg.block, cfg.sink, cfg.window)
        out[fa] = (time.perf_counter() - t0) / n_seq
    return out


def cpu_oracle_prefill_sample(w, n_rows: int = 16, seed: int = 9):
    """Time the fp64 oracle on n_rows query rows, evenly spaced over the prompt of
    workload w, of one FA and one SA layer (all query heads); returns seconds per query
    row per layer for each route."""
    import numpy as np

    from oracle import flux_oracle as orc
    from sparse_attention_layer_b200 import inputs
    S = w.seq
    rows = np.linspace(0, S - 1, n_rows).astype(np.int64)
    # only the sampled query rows are drawn (np.zeros leaves the rest unallocated)
    q = np.zeros((1, S, w.n_q_heads, w.head_dim))
    q[0, rows] = inputs.normal_bf16((n_rows, w.n_q_heads, w.head_dim), seed).float().numpy()
    shape = (1, w.n_kv_heads, S, w.head_dim)
    kc = inputs.normal_bf16(shape, seed + 1).float().numpy().astype(np.float64)
    vc = inputs.normal_bf16(shape, seed + 2).float().numpy().astype(np.float64)
    out = {}
    for fa in (True, False):
        t0 = time.perf_counter()
        orc.attention_layer(q, kc, vc, np.array([S]), np.array([fa]), w.block, w.sink, w.window,
                            rows=rows)
        out[fa] = (time.perf_counter() - t0) / n_rows
    return out


def cpu_prefill_baseline(w, n_fa: int, n_rows: int = 16):
    t0 = time.perf_counter()
    per_row = cpu_oracle_prefill_sample(w, n_rows)
    n_sa = w.n_layers - n_fa
    sec = w.seq * (n_fa * per_row[True] + n_sa * per_row[False])
    return {"value": w.batch * w.seq / sec, "unit": "tokens/s", "cores": host_cores(),
            "blas_threads": blas_threads(), "kind": "oracle", "extrapolated": True,
            "sample": f"{n_rows} evenly spaced query rows x {w.n_q_heads} heads of one FA and one "
                      f"SA layer of the {w.seq}-token prompt (fp64 oracle), extrapolated to all "
                      f"rows of {n_fa} FA + {n_sa} SA layers; "
                      f"{time.perf_counter() - t0:.1f} s wall, data generation included"}


def cpu_baseline_decode_tok_s(w, n_sa, n_seq=2, chunks=1):
    """Oracle decode throughput from `chunks` samples of n_seq sequences each (distinct
    seeded caches), averaged."""
    fa = sa = 0.0
    for i in range(chunks):
        per = cpu_oracle_decode_sample(n_seq, seed=5 + 3 * i)
        fa += per[True] / chunks
        sa += per[False] / chunks
    per_seq_step = (w.n_layers - n_sa) * fa + n_sa * sa
    return 1.0 / per_seq_step, {True: fa, False: sa}


# ---------------------------------------------------------------------- runs


def run_reference(args, world, rank):
    """The oracle timed on the host cores, on bounded samples of the decode workload."""
    if rank != 0:
        return
    from sparse_attention_layer_b200 import configs, inputs
    w, cfg = decode_geometry()
    sa = inputs.fixed_sa_layers(w.n_layers, w.target_sa_layers, configs.LLAMA_DECODE_MASK_SEED)
    for _ in range(args.warmup):
        cpu_oracle_decode_sample(1)
    times = []
    for _ in range(args.steps):
        per = cpu_oracle_decode_sample(1)
        times.append((w.n_layers - len(sa)) * per[True] + len(sa) * per[False])
    per_seq_step = statistics.mean(times)
    value = 1.0 / per_seq_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_seq_step * 1e3 * w.batch, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "extrapolated": True,
        "config": decode_config(w, cfg, sa),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(),
                         "blas_threads": blas_threads(), "kind": "oracle", "extrapolated": True,
                         "sample": "per step: one decode token of 1 of the 16 sequences at "
                                   "32768 context, one FA and one SA layer, scaled to 16 FA + "
                                   "16 SA layers; a batch of 16 costs 16x (sequences are "
                                   "independent), so ms_per_step is scaled, not measured"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def decode_config(w, cfg, sa_layers):
    return {"workload": "llama3.1-8b-shape hybrid attention decode, 16 sequences at 32768 "
                        "context, 32 layers (16 FA + 16 SA, fixed seeded mask)",
            "batch": w.batch, "context": w.seq, "n_layers": w.n_layers,
            "q_heads": cfg.n_q_heads, "kv_heads": cfg.n_kv_heads, "head_dim": cfg.head_dim,
            "sa_layers": len(sa_layers), "sink": cfg.sink, "window": cfg.window,
            "block": cfg.block, "parallelism": "replicas (one independent model per GPU)",
            "l2": "no flush needed: each step streams ~37 GB of KV, far above the 126 MB L2"}


def run_decode(args, world, local, peaks, peak_kind):
    """Headline decode step, its per-route rooflines, e2e, routing mix, eviction."""
    from sparse_attention_layer_b200 import flux
    from sparse_attention_layer_b200.runtime import DecodeStepGraph
    db = DecodeBench(seed=1234 + world)
    w, cfg = db.w, db.cfg
    sa_layers = list(db.sa_layers)

    # ---------------- the decode step as one CUDA graph (the headline number)
    db.reset()
    for layer in range(w.n_layers):  # one eager step: per-device one-time set-up
        db.model.decode_layer(layer, db.q[layer], db.k_new[layer], db.v_new[layer], db.o[layer])
    db.reset()
    graph = DecodeStepGraph(db.model, db.q, db.k_new, db.v_new, db.o)
    db.reset()
    for _ in range(args.warmup):  # warm-up replays outside the timed region
        graph.replay()
    db.reset()
    sampler = ClockSampler(local)
    barrier(world)
    sampler.start()
    gs = torch.cuda.Event(enable_timing=True)
    ge = torch.cuda.Event(enable_timing=True)
    barrier(world)
    gs.record()
    for _ in range(args.steps):
        graph.replay()
    ge.record()
    barrier(world)
    tg_ms = max_over_ranks(gs.elapsed_time(ge), world)
    value = replica_tokens_per_s(world, w.batch, args.steps, tg_ms)
    ms_step = tg_ms / args.steps
    st = flux.flux_get_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the graph decode steps")

    # ---------------- per-route rooflines: the same launches, one route's layers per graph
    fa_layers = [i for i in range(w.n_layers) if db.fa[i]]
    route_ms = {}
    for name, layers in (("fa", fa_layers), ("sa", sa_layers)):
        db.reset()
        g = db.layers_graph(layers)
        reps = max(5, min(args.steps, 20))
        route_ms[name] = graph_ms(g, 2, reps, reset=db.reset) / len(layers)
        del g
    clocks = sampler.stop()  # sampled over the graph step and the per-route graphs
    T_mean = w.seq + 1 + (args.steps - 1) / 2.0  # keys after the append, mean over the steps
    T_route = w.seq + 1
    fa_bytes = decode_bytes_per_layer(w, cfg, T_route, True, append=True)
    sa_bytes = decode_bytes_per_layer(w, cfg, T_route, False, append=True)
    timing = ("graph of the route's layers (one flux_decode_append launch each, as in the "
              "step), replayed; launch time = replay time / layers")
    roofline = hbm_roofline("decode_kernel (flux_decode_append), FA layers", fa_bytes,
                            route_ms["fa"], peaks, peak_kind,
                            traffic=measured_traffic("decode", w.batch), timing=timing)
    roofline["traffic_note"] = "ncu dram bytes of a 4-sequence capture scaled to 16"
    roofline_sa = hbm_roofline("decode_kernel (flux_decode_append), SA layers", sa_bytes,
                               route_ms["sa"], peaks, peak_kind,
                               traffic=measured_traffic("decode_sa", w.batch), timing=timing)
    step_bytes = sum(decode_bytes_per_layer(w, cfg, int(round(T_mean)), fa, append=True)
                     for fa in db.fa)

    # ---------------- decode: end to end from pinned host buffers
    q_h = db.q.cpu().pin_memory()
    k_h = db.k_new.cpu().pin_memory()
    v_h = db.v_new.cpu().pin_memory()
    o_h = torch.empty(db.o.shape, dtype=db.o.dtype).pin_memory()
    db.reset()
    barrier(world)
    s2 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(args.steps):
        db.q.copy_(q_h, non_blocking=True)
        db.k_new.copy_(k_h, non_blocking=True)
        db.v_new.copy_(v_h, non_blocking=True)
        graph.replay()
        o_h.copy_(db.o, non_blocking=True)
    e2.record()
    barrier(world)
    t2 = max_over_ranks(s2.elapsed_time(e2), world)
    e2e = {"value": replica_tokens_per_s(world, w.batch, args.steps, t2), "unit": "tokens/s",
           "h2d_bytes_per_step": (q_h.numel() + k_h.numel() + v_h.numel()) * 2,
           "d2h_bytes_per_step": o_h.numel() * 2,
           "what": "per step: pinned-host q, k_new, v_new for all 32 layers copied in, the "
                   "captured 32-layer decode step replayed, outputs of all layers copied out"}

    # ---------------- routing mix: decode step time vs SA-layer fraction
    mix = {}
    n_mix_steps = max(5, min(20, args.steps))
    perm_sa = db.sa_layers + [i for i in range(w.n_layers) if i not in db.sa_layers]
    for frac in (0.0, 0.25, 0.5, 0.75, 1.0):
        n_sa = int(round(frac * w.n_layers))
        db.set_sa_layers(perm_sa[:n_sa])
        db.reset()
        graph.replay()
        barrier(world)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n_mix_steps):
            graph.replay()
        b.record()
        barrier(world)
        ms = max_over_ranks(a.elapsed_time(b), world) / n_mix_steps
        mix[f"{int(frac * 100)}%"] = {"sa_layers": n_sa, "ms_per_step": ms,
                                      "tokens_per_s": world * w.batch / (ms / 1e3)}
    base = mix["0%"]["ms_per_step"]
    for v in mix.values():
        v["speedup_vs_all_fa"] = base / v["ms_per_step"]
    db.set_sa_layers(db.sa_layers)
    del graph

    # ---------------- SA-layer KV eviction: rings of sink + window rows per SA layer
    db.reset()
    kv_full = db.model.kv_bytes()
    db.model.evict_sa_layers()
    torch.cuda.synchronize()
    kv_evicted = db.model.kv_bytes()
    db.reset()
    ring_graph = DecodeStepGraph(db.model, db.q, db.k_new, db.v_new, db.o)
    db.reset()
    for _ in range(args.warmup):
        ring_graph.replay()
    db.reset()
    barrier(world)
    rs = torch.cuda.Event(enable_timing=True)
    re_ = torch.cuda.Event(enable_timing=True)
    rs.record()
    for _ in range(args.steps):
        ring_graph.replay()
    re_.record()
    barrier(world)
    tr_ms = max_over_ranks(rs.elapsed_time(re_), world)
    st = flux.flux_get_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the ring decode steps")
    gib = float(1 << 30)
    hbm_budget = 160 * gib  # leaves room for weights and activations on a 180 GB part
    eviction = {
        "kv_gib_full": kv_full / gib, "kv_gib_evicted": kv_evicted / gib,
        "saving": 1.0 - kv_evicted / kv_full,
        "decode_tokens_per_s": replica_tokens_per_s(world, w.batch, args.steps, tr_ms),
        "ms_per_step": tr_ms / args.steps,
        "max_batch_in_160_gib": {"full": int(hbm_budget // (kv_full / w.batch)),
                                 "evicted": int(hbm_budget // (kv_evicted / w.batch))},
        "what": "the 16 SA layers' caches moved to rings of sink 128 + 2048 rows per "
                "(sequence, KV head) after prefill; the same graph-replayed decode step",
    }
    out = {
        "value": value, "ms_per_step": ms_step, "config": decode_config(w, cfg, sa_layers),
        "roofline": roofline, "roofline_sa": roofline_sa,
        "decode_step": {"algorithmic_gb_per_step": step_bytes / 1e9,
                        "step_gb_per_s": step_bytes / (ms_step / 1e3) / 1e9,
                        "fa_layer_bytes": fa_bytes, "sa_layer_bytes": sa_bytes,
                        "fa_layer_us": route_ms["fa"] * 1e3, "sa_layer_us": route_ms["sa"] * 1e3},
        "e2e": e2e, "gpu_launches": db.launches_per_step * args.steps, "clocks": clocks,
        "routing_mix": mix, "sa_kv_eviction": eviction, "sa_layers": sa_layers,
    }
    del ring_graph, db
    torch.cuda.empty_cache()
    return out


def run_prefill_llama(args, world, local, peaks, peak_kind):
    """Llama 8K prompt: router-chosen step, per-route prefill rooflines, routing mix."""
    from sparse_attention_layer_b200 import configs, inputs
    w = configs.LLAMA_PREFILL
    pb = PrefillBench(w, seed=99 + world)
    for _ in range(3):
        pb.reset()
        pb.step()
    n_pf = max(3, min(10, args.steps))
    pf_ms, fa_ev, sa_ev, rt_ev, ap_ev = [], [], [], [], []
    sampler = ClockSampler(local).start()
    barrier(world)
    for _ in range(n_pf):
        pb.reset()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        pb.step(fa_events=fa_ev, sa_events=sa_ev, router_events=rt_ev, append_events=ap_ev)
        b.record()
        pf_ms.append((a, b))
    barrier(world)
    pf_step = max_over_ranks(statistics.mean(elapsed_ms(pf_ms)), world)
    n_fa = sum(pb.fa)
    flops_fa = prefill_flops_per_layer(pb.cfg, w.seq, True)
    flops_sa = prefill_flops_per_layer(pb.cfg, w.seq, False)

    # routing mix: the same 32 layers with the first n of a seeded layer permutation on SA
    mix = {}
    for frac in (0.0, 0.25, 0.5, 0.75, 1.0):
        n_sa = int(round(frac * w.n_layers))
        sa = inputs.fixed_sa_layers(w.n_layers, n_sa, seed=11)
        bits = inputs.fa_bits_from_sa_layers(w.batch, w.n_layers, sa)
        pb.model.set_mask(inputs.pack_bits_u32(bits).cuda())
        pb.fa = [bool(bits[0, i]) for i in range(w.n_layers)]
        pb.reset()
        pb.step(route=False)
        times = []
        for _ in range(3):
            pb.reset()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            pb.step(route=False)
            b.record()
            times.append((a, b))
        barrier(world)
        ms = max_over_ranks(statistics.median(elapsed_ms(times)), world)
        mix[f"{int(frac * 100)}%"] = {"sa_layers": n_sa, "ms_per_step": ms,
                                      "tokens_per_s": world * w.batch * w.seq / (ms / 1e3)}
    base = mix["0%"]["ms_per_step"]
    for v in mix.values():
        v["speedup_vs_all_fa"] = base / v["ms_per_step"]
    clocks = sampler.stop()
    pb.fa = pb.mask_bits(pb.router_mask)
    pb.model.set_mask(pb.router_mask)

    # end to end from pinned host buffers: per step x_Q in for the router, then per layer
    # q, k, v in and o out (layer inputs arrive and outputs leave as the layers run)
    from sparse_attention_layer_b200 import flux
    xq_h = pb.xq.cpu().pin_memory()
    q_h, k_h, v_h = (t.cpu().pin_memory() for t in (pb.q, pb.k, pb.v))
    o_h = torch.empty(pb.o.shape, dtype=pb.o.dtype).pin_memory()
    m = pb.model
    e2e_steps = 3
    barrier(world)
    s2 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    s2.record()
    for _ in range(e2e_steps):
        pb.reset()
        pb.xq.copy_(xq_h, non_blocking=True)
        m.route(*pb.router, pb.xq, w.pool_len, w.tau)
        for layer in range(w.n_layers):
            pb.q.copy_(q_h, non_blocking=True)
            pb.k.copy_(k_h, non_blocking=True)
            pb.v.copy_(v_h, non_blocking=True)
            c = m.caches[layer]
            flux.flux_kv_append(pb.cfg, c.k, c.v, c.seq_len, pb.k, pb.v)
            flux.flux_prefill(pb.cfg, layer, m.fa_mask, pb.q, c.k, c.v, c.seq_len, pb.o)
            o_h.copy_(pb.o, non_blocking=True)
    e2.record()
    barrier(world)
    t_e2e = max_over_ranks(s2.elapsed_time(e2), world) / e2e_steps
    e2e = {"value": world * w.batch * w.seq / (t_e2e / 1e3), "unit": "tokens/s",
           "ms_per_step": t_e2e,
           "h2d_bytes_per_step": xq_h.numel() * 2 + w.n_layers * (q_h.numel() + k_h.numel() +
                                                                 v_h.numel()) * 2,
           "d2h_bytes_per_step": w.n_layers * o_h.numel() * 2,
           "what": "per step: pinned-host x_Q copied in and routed, then per layer pinned-host "
                   "q, k, v copied in, KV append + prefill, the layer's output copied out"}
    out = {
        "workload": "llama3.1-8b-shape prefill, 1 x 8192 tokens, router 4096->256->32 "
                    f"(seeded; {w.n_layers - n_fa} SA layers), SA sink 128 + window 2048",
        "tokens_per_s": world * w.batch * w.seq / (pf_step / 1e3),
        "ms_per_step": pf_step, "steps": n_pf, "sa_layers": w.n_layers - n_fa,
        # the router's sparsity ratio: the share of layers it sends to SA
        "omega_msr": (w.n_layers - n_fa) / w.n_layers,
        "router_ms": statistics.mean(elapsed_ms(rt_ev)),
        "algorithmic_tflops_per_step": (n_fa * flops_fa + (w.n_layers - n_fa) * flops_sa) / 1e12,
        "roofline": tensor_roofline("prefill_kernel<128> (tcgen05), FA layers", flops_fa,
                                    statistics.mean(elapsed_ms(fa_ev)), peaks, peak_kind, clocks,
                                    traffic=measured_traffic("prefill", w.batch)),
        "roofline_sa": tensor_roofline("prefill_kernel<128> (tcgen05), SA layers", flops_sa,
                                       statistics.mean(elapsed_ms(sa_ev)), peaks, peak_kind,
                                       clocks, traffic=measured_traffic("prefill_sa", w.batch)),
        # the layer's KV append: the prompt's K and V rows read from the projection layout
        # and written head-major into the cache (a copy: the measured peak's own kind)
        "append_roofline": hbm_roofline(
            "kv_append_copy_kernel + kv_append_advance_kernel (flux_kv_append, one layer)",
            2.0 * 2 * w.batch * w.seq * w.n_kv_heads * w.head_dim * 2,
            statistics.mean(elapsed_ms(ap_ev)), peaks, peak_kind,
            traffic=measured_traffic("append", w.batch),
            timing="CUDA events around each layer's flux_kv_append inside the timed steps"),
        "routing_mix": mix,
        "e2e": e2e,
        "gpu_launches_per_step": pb.launches_per_step,
        "clocks": clocks,
        "cpu_baseline": None,
    }
    del pb, xq_h, q_h, k_h, v_h, o_h
    torch.cuda.empty_cache()
    if world == 1 and not args.no_cpu:
        out["cpu_baseline"] = cpu_prefill_baseline(w, n_fa, n_rows=2048)
    return out


def run_prefill_qwen(args, world, local, peaks, peak_kind):
    """Qwen3-4B 131072-token prompt: router + 36 x (append + prefill), measured whole."""
    from sparse_attention_layer_b200 import configs
    w = configs.QWEN_PREFILL
    pb = PrefillBench(w, seed=199 + world)
    pb.reset()
    pb.step()
    sampler = ClockSampler(local).start()
    barrier(world)
    fa_ev, sa_ev, rt_ev, steps = [], [], [], []
    for _ in range(2):
        pb.reset()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        pb.step(fa_events=fa_ev, sa_events=sa_ev, router_events=rt_ev)
        b.record()
        steps.append((a, b))
    barrier(world)
    clocks = sampler.stop()
    ms = max_over_ranks(statistics.mean(elapsed_ms(steps)), world)
    n_fa = sum(pb.fa)
    flops_fa = prefill_flops_per_layer(pb.cfg, w.seq, True)
    flops_sa = prefill_flops_per_layer(pb.cfg, w.seq, False)
    fa_roof = tensor_roofline("prefill_kernel<128> (tcgen05), FA layers", flops_fa,
                              statistics.mean(elapsed_ms(fa_ev)), peaks, peak_kind, clocks)
    fa_roof["peak_note"] = ("a multi-second phase: compare with the sustained peak when the "
                            "phase clocks show sw_power_cap")
    out = {
        "workload": "qwen3-4b-shape prefill, 1 x 131072 tokens, 36 layers, router 2560->256->36 "
                    f"(seeded; {w.n_layers - n_fa} SA layers), SA sink 128 + window 4096",
        "tokens_per_s": world * w.batch * w.seq / (ms / 1e3), "ms_per_step": ms, "steps": 2,
        "sa_layers": w.n_layers - n_fa, "omega_msr": (w.n_layers - n_fa) / w.n_layers,
        "router_ms": statistics.mean(elapsed_ms(rt_ev)),
        "fa_layer_ms": statistics.mean(elapsed_ms(fa_ev)),
        "sa_layer_ms": statistics.mean(elapsed_ms(sa_ev)),
        "algorithmic_tflops_per_step": (n_fa * flops_fa + (w.n_layers - n_fa) * flops_sa) / 1e12,
        "roofline": fa_roof,
        "roofline_sa": tensor_roofline("prefill_kernel<128> (tcgen05), SA layers", flops_sa,
                                       statistics.mean(elapsed_ms(sa_ev)), peaks, peak_kind,
                                       clocks, traffic=measured_traffic("prefill_sa", w.batch)),
        "clocks": clocks, "cpu_baseline": None,
    }
    del pb
    torch.cuda.empty_cache()
    if world == 1 and not args.no_cpu:
        out["cpu_baseline"] = cpu_prefill_baseline(w, n_fa, n_rows=64)
    return out


# ------------------------------------------------------------------ sweeps


def decode_sweep_point(cfg, T: int, B: int, fracs, warm=3, reps=10, seed=5):
    """Graph-replayed 32-layer decode steps (one append + decode launch per layer) at
    context T and batch B, for each SA-layer fraction.  Layers cycle over n distinct KV
    caches: n = the layer count where they fit in 120 GB and at least 512 MB of cache is
    read between two visits of one cache (so repeated layers are not served from L2)."""
    from sparse_attention_layer_b200 import inputs
    from sparse_attention_layer_b200.runtime import HybridAttention
    n_layers = cfg.n_layers
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    cap = T + n_layers * (warm + reps + 2) + 64
    cache_bytes = 2 * B * cfg.n_kv_heads * cap * cfg.head_dim * 2
    n_cache = max(1, min(n_layers, -(-512 * 2**20 // cache_bytes), (120 << 30) // cache_bytes))
    m = HybridAttention(cfg, B, cap, "cuda", layers=n_cache)
    for c in m.caches:
        c.k.normal_(generator=gen)
        c.v.normal_(generator=gen)
    q = torch.randn(B, cfg.n_q_heads, cfg.head_dim, device="cuda", generator=gen).to(torch.bfloat16)
    kn = torch.randn(B, 1, cfg.n_kv_heads, cfg.head_dim, device="cuda", generator=gen).to(torch.bfloat16)
    o = torch.empty_like(q)

    def step():
        for layer in range(n_layers):
            m.decode_layer(layer, q, kn, kn, o, cache_index=layer % n_cache)

    def reset():
        for c in m.caches:
            c.seq_len.fill_(T)
    reset()
    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    row = {"context": T, "batch": B, "distinct_caches": n_cache,
           "composed": n_cache < n_layers}
    for f in fracs:
        sa = inputs.fixed_sa_layers(n_layers, int(round(f * n_layers)), seed=11)
        m.set_mask(inputs.pack_bits_u32(inputs.fa_bits_from_sa_layers(B, n_layers, sa)).cuda())
        reset()
        for _ in range(warm):
            graph.replay()
        reset()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for a, b in ev:
            a.record()
            graph.replay()
            b.record()
        torch.cuda.synchronize()
        ms = statistics.median(a.elapsed_time(b) for a, b in ev)
        row[f"{int(f * 100)}%"] = {"ms_per_step": ms, "tokens_per_s": B / (ms / 1e3)}
    if "0%" in row:
        base = row["0%"]["ms_per_step"]
        for f in fracs:
            row[f"{int(f * 100)}%"]["speedup_vs_all_fa"] = base / row[f"{int(f * 100)}%"]["ms_per_step"]
        row["fa_layer_us"] = base / n_layers * 1e3
    if "100%" in row:
        row["sa_layer_us"] = row["100%"]["ms_per_step"] / n_layers * 1e3
    del graph, m, q, kn, o
    torch.cuda.empty_cache()
    return row


def prefill_sweep_point(cfg, T: int, fracs, seed=6):
    """Graph-replayed 32-layer prefill steps (batch 1, KV append + FA/SA prefill per
    layer on separate caches) of a T-token prompt for each SA-layer fraction."""
    from sparse_attention_layer_b200 import inputs
    from sparse_attention_layer_b200.runtime import HybridAttention
    n_layers = cfg.n_layers
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    m = HybridAttention(cfg, 1, T, "cuda")
    lens = torch.zeros(n_layers, 1, dtype=torch.int32, device="cuda")
    for i, c in enumerate(m.caches):
        c.seq_len = lens[i]
    qp = torch.randn(1, T, cfg.n_q_heads, cfg.head_dim, device="cuda", generator=gen).to(torch.bfloat16)
    kp = torch.randn(1, T, cfg.n_kv_heads, cfg.head_dim, device="cuda", generator=gen).to(torch.bfloat16)
    op = torch.empty_like(qp)

    def pstep():
        lens.zero_()
        for layer in range(n_layers):
            m.prefill_layer(layer, qp, kp, kp, op)
    pstep()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        pstep()
    row = {"context": T}
    pw, pr = (1, 2) if T >= 65536 else (2, 5)
    for f in fracs:
        sa = inputs.fixed_sa_layers(n_layers, int(round(f * n_layers)), seed=11)
        m.set_mask(inputs.pack_bits_u32(inputs.fa_bits_from_sa_layers(1, n_layers, sa)).cuda())
        ms = graph_ms(graph, pw, pr)
        row[f"{int(f * 100)}%"] = {"ms": ms, "tokens_per_s": T / (ms / 1e3)}
    if "0%" in row:
        base = row["0%"]["ms"]
        for f in fracs:
            row[f"{int(f * 100)}%"]["speedup_vs_all_fa"] = base / row[f"{int(f * 100)}%"]["ms"]
        row["fa_layer_ms"] = base / n_layers
        row["fa_tflops"] = prefill_flops_per_layer(cfg, T, True) / (row["fa_layer_ms"] / 1e3) / 1e12
    if "100%" in row:
        row["sa_layer_ms"] = row["100%"]["ms"] / n_layers
        row["sa_tflops"] = prefill_flops_per_layer(cfg, T, False) / (row["sa_layer_ms"] / 1e3) / 1e12
    del graph, m, lens, qp, kp, op
    torch.cuda.empty_cache()
    return row


def llama_sweep_cfg(block=128, sink=128, window=2048, head_dim=128):
    from sparse_attention_layer_b200.flux import AttnCfg
    return AttnCfg(32, 32, 8, head_dim, block, sink, window)


def run_pages_geometry(peaks, peak_kind):
    """The pages' SA kernel geometry (block 64, sink 128; window 2048), head_dim 64 and
    128: decode at 16 x 32K (32 layers, 0/50/100 % SA) and the 8K prefill."""
    out = {}
    for d in (64, 128):
        cfg = llama_sweep_cfg(block=64, sink=128, window=2048, head_dim=d)
        dec = decode_sweep_point(cfg, 32768, 16, (0.0, 0.5, 1.0), seed=7 + d)
        pre = prefill_sweep_point(cfg, 8192, (0.0, 0.5, 1.0), seed=8 + d)
        w16 = type("W", (), {"batch": 16})
        sa_bytes = decode_bytes_per_layer(w16, cfg, 32769, False, append=True)
        fa_bytes = decode_bytes_per_layer(w16, cfg, 32769, True, append=True)
        dec["sa_layer_gb_per_s"] = sa_bytes / (dec["sa_layer_us"] / 1e6) / 1e9
        dec["fa_layer_gb_per_s"] = fa_bytes / (dec["fa_layer_us"] / 1e6) / 1e9
        dec["sa_frac_of_hbm_peak"] = dec["sa_layer_gb_per_s"] / peaks["hbm_gbs"]
        dec["fa_frac_of_hbm_peak"] = dec["fa_layer_gb_per_s"] / peaks["hbm_gbs"]
        pre["fa_frac_of_burst_peak"] = pre["fa_tflops"] / peaks["bf16_tflops"]
        pre["sa_frac_of_burst_peak"] = pre["sa_tflops"] / peaks["bf16_tflops"]
        out[f"head_dim_{d}"] = {"decode_16x32k": dec, "prefill_8k": pre}
    out["what"] = ("Llama heads (32 q / 8 kv), block 64, sink 128, window 2048; per-layer "
                   "times are the 0 % / 100 % SA steps / 32 (append + attention per layer)")
    return out


def run_sweep_subset():
    """Compact context x batch x routing-mix sweep (Llama shape, block 128)."""
    cfg = llama_sweep_cfg()
    fracs = (0.0, 0.5, 1.0)
    dec = [decode_sweep_point(cfg, T, B, fracs) for T in (32768, 131072) for B in (1, 32)]
    pre = [prefill_sweep_point(cfg, T, fracs) for T in (32768, 131072)]
    return {"decode": dec, "prefill": pre,
            "what": "graph-replayed 32-layer steps; decode batch 1 / 32 at 32K and 128K, "
                    "prefill batch 1; 0 / 50 / 100 % SA layers; 'composed' rows cycle "
                    "fewer distinct caches than layers (the full model does not fit)"}


def run_table16():
    """The pages' latency-memory comparison (Table 16: Omega_MSR, prefill ms, decode
    ms/token, persistent KV GiB and its saving, peak GiB, at 8K and 16K contexts) for
    this attention path: Llama-3.1-8B shape, batch 1, routes from the seeded router on
    synthetic x_Q, against every layer on FA (the dense reference).  Memory counts what
    the attention path holds on the device (KV caches, q/k/v/o, x_Q, workspace), not a
    model's weights or activations."""
    import dataclasses

    from sparse_attention_layer_b200 import configs, inputs
    from sparse_attention_layer_b200.runtime import DecodeStepGraph, HybridAttention
    GiB = float(1 << 30)
    out = {}
    for T in (8192, 16384):
        w = dataclasses.replace(configs.LLAMA_PREFILL, seq=T)
        cfg = llama_sweep_cfg()
        base_alloc = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        steps = 48
        model = HybridAttention(cfg, 1, T + steps + 16, "cuda")
        router = [t.cuda() for t in inputs.router_weights(w.router_hidden, w.router_rank,
                                                            w.n_layers, w.router_seed)]
        xq = inputs.normal_bf16((1, T, w.router_hidden),
                                inputs.layer_seed(w.data_seed, 0, inputs.XQ)).cuda()
        gen = torch.Generator(device="cuda")
        gen.manual_seed(1600 + T)
        q = torch.randn(1, T, cfg.n_q_heads, cfg.head_dim, device="cuda",
                        generator=gen).to(torch.bfloat16)
        k = torch.randn(1, T, cfg.n_kv_heads, cfg.head_dim, device="cuda",
                        generator=gen).to(torch.bfloat16)
        v = torch.randn_like(k)
        o = torch.empty_like(q)
        L = cfg.n_layers
        dq = torch.randn(L, 1, cfg.n_q_heads, cfg.head_dim, device="cuda").to(torch.bfloat16)
        dk = torch.randn(L, 1, 1, cfg.n_kv_heads, cfg.head_dim, device="cuda").to(torch.bfloat16)
        dv = torch.randn_like(dk)
        do = torch.empty_like(dq)
        model.route(*router, xq, w.pool_len, w.tau)
        router_mask = model.fa_mask.clone()
        all_fa = inputs.pack_bits_u32(inputs.fa_bits_from_sa_layers(1, L, [])).cuda()

        def prefill(route):
            for c in model.caches:
                c.seq_len.zero_()
            if route:
                model.route(*router, xq, w.pool_len, w.tau)
            for layer in range(L):
                model.prefill_layer(layer, q, k, v, o)

        def timed(fn, reps=3):
            fn()
            times = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                times.append((a, b))
            torch.cuda.synchronize()
            return statistics.median(x.elapsed_time(y) for x, y in times)

        def decode_ms():
            # one eager step (library set-up), then the captured step, replayed; the
            # appends advance the lengths from T
            for layer in range(L):
                model.decode_layer(layer, dq[layer], dk[layer], dv[layer], do[layer])
            g = DecodeStepGraph(model, dq, dk, dv, do)
            ms = graph_ms(g.graph, warm=3, reps=20)
            del g
            return ms

        model.set_mask(all_fa)
        row_fa_prefill = timed(lambda: prefill(False))
        prefill(False)
        row_fa_decode = decode_ms()
        peak_prefill = (torch.cuda.max_memory_allocated() - base_alloc) / GiB
        kv_fa = model.kv_bytes() / GiB
        model.set_mask(router_mask)
        row_flux_prefill = timed(lambda: prefill(True))
        prefill(False)
        n_sa = len(model.sa_layers())
        row_flux_decode = decode_ms()
        model.evict_sa_layers()
        torch.cuda.synchronize()
        kv_flux = model.kv_bytes() / GiB
        row_flux_decode_rings = decode_ms()
        # the context's own K/V (T rows per layer; the allocation adds room for the steps)
        per_row = 2 * cfg.n_kv_heads * cfg.head_dim * 2
        logical_full = L * T * per_row / GiB
        logical_flux = ((L - n_sa) * T + n_sa * (cfg.sink + cfg.window)) * per_row / GiB
        row = {
            "omega_msr": n_sa / L, "sa_layers": n_sa,
            "prefill_ms": {"flux": row_flux_prefill, "all_fa": row_fa_prefill,
                           "speedup": row_fa_prefill / row_flux_prefill},
            "decode_ms_per_token": {"flux": row_flux_decode, "all_fa": row_fa_decode,
                                    "speedup": row_fa_decode / row_flux_decode,
                                    "flux_sa_layers_evicted": row_flux_decode_rings},
            "persistent_kv_gib": {"all_fa": logical_full, "flux_evicted": logical_flux,
                                  "saving": 1.0 - logical_flux / logical_full,
                                  "allocated_all_fa": kv_fa, "allocated_flux_evicted": kv_flux},
            "peak_gib_prefill": peak_prefill,
        }
        out[f"{T // 1024}K"] = row
        del model, xq, q, k, v, o, dq, dk, dv, do
        torch.cuda.empty_cache()
    out["what"] = ("batch 1, Llama-3.1-8B attention shape, seeded router on synthetic x_Q "
                   "(routes) vs all layers on FA; prefill = router + 32 x (append + prefill); "
                   "decode = the captured 32-layer step (one token); persistent KV = the "
                   "context's K/V rows, SA layers as rings of sink + window rows after "
                   "eviction; peak = device memory the attention path allocated")
    return out


def run_flux(args, world, rank, local):
    from sparse_attention_layer_b200 import flux
    peaks, peak_kind = load_peaks()
    dec = run_decode(args, world, local, peaks, peak_kind)
    prefill = run_prefill_llama(args, world, local, peaks, peak_kind)
    extra = {}
    if not args.quick and world == 1:  # per-GPU figures: the N = 1 run reports them
        extra["prefill_qwen_128k"] = run_prefill_qwen(args, world, local, peaks, peak_kind)
        extra["pages_sa_geometry"] = run_pages_geometry(peaks, peak_kind)
        extra["sweep_subset"] = run_sweep_subset()
        extra["table16_llama"] = run_table16()
    if flux.flux_get_device_status():
        raise RuntimeError("device status set during the benchmark")

    # ---------------- CPU baseline of the headline (rank 0, N = 1 only)
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu:
        w, _ = decode_geometry()
        t0 = time.perf_counter()
        tok_s, _ = cpu_baseline_decode_tok_s(w, len(dec["sa_layers"]), n_seq=2, chunks=8)
        cpu = {"value": tok_s, "unit": "tokens/s", "cores": host_cores(),
               "blas_threads": blas_threads(), "kind": "oracle", "extrapolated": True,
               "sample": "one decode token of all 16 sequences (8 draws of 2) at 32768 context for "
                         "one FA and one SA layer (fp64 oracle), scaled to 16 FA + 16 SA "
                         f"layers; {time.perf_counter() - t0:.1f} s wall, data generation "
                         "included"}

    line = {
        "metric": METRIC, "value": dec["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dec["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dec["config"],
        "roofline": dec["roofline"], "roofline_sa": dec["roofline_sa"],
        "decode_step": dec["decode_step"], "cpu_baseline": cpu, "e2e": dec["e2e"],
        "gpu_launches": dec["gpu_launches"], "clocks": dec["clocks"],
        "prefill": prefill, "routing_mix": dec["routing_mix"],
        "sa_kv_eviction": dec["sa_kv_eviction"],
    }
    line.update(extra)
    if rank == 0:
        print(json.dumps(line))


def run_sweep(args):
    """The full routing-mix x context x batch sweep of the Llama-3.1-8B shape (32 layers,
    32/8 heads, d 128, sink 128 + window 2048, block 128)."""
    from sparse_attention_layer_b200 import configs, flux
    torch.cuda.set_device(0)
    cfg = llama_sweep_cfg()
    fracs = configs.SWEEP_SA_FRACTIONS
    out = {"decode": [], "prefill": []}
    sampler = ClockSampler(0).start()
    for T in configs.SWEEP_CONTEXTS:
        for B in configs.SWEEP_BATCHES:
            out["decode"].append(decode_sweep_point(cfg, T, B, fracs))
        out["prefill"].append(prefill_sweep_point(cfg, T, fracs))
    clocks = sampler.stop()
    if flux.flux_get_device_status():
        raise RuntimeError("device status set during the sweep")
    print(json.dumps({"sweep": out, "measured": "graph-replayed 32-layer steps",
                      "clocks": clocks}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["flux", "reference"], default="flux")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baselines")
    ap.add_argument("--quick", action="store_true",
                    help="decode and Llama prefill only (no Qwen prefill, geometry or sweep)")
    ap.add_argument("--sweep", action="store_true",
                    help="full routing-mix x context x batch sweep (graph-replayed 32-layer steps)")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.warmup + args.steps > 256 - 1:
        raise SystemExit("warm-up + steps must stay within the 256 decode steps of capacity")
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_flux(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

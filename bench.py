"""Benchmark of the hybrid-attention hot path (Flux Attention: layer router + FA/SA
prefill + FA/SA decode) on B200.

Main line (`value`): decode tokens/s of the Llama-3.1-8B attention shape serving 16
sequences at a 32768-token context, 32 layers of which a fixed seeded 16 run SA
(sink 128 + window 2048, block 128).  One step = one decode token for every sequence:
per layer a KV append and an FA- or SA-routed split-KV decode, the 32 layers captured
once as a CUDA graph and replayed per step (the eager, launch-by-launch number is
reported beside it, and its FA decode launches give the HBM roofline).  The same run also
times the prefill phase (router + 32 x (KV append + FA/SA prefill) of an 8192-token
Llama-shaped prompt with router-chosen routes) and the decode step at every SA-layer
fraction of the routing mix.  Protocol: W warm-up then K timed steps (default 10 and
50), CUDA events on the launching stream, barrier + synchronize around the timed
region, max over ranks.

`--impl reference` times the fp64 CPU oracle on the host cores instead, on a bounded
sample of the same decode workload, and prints the same metric.

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
        self.path = os.path.join("/tmp", f"flux_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

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


# ------------------------------------------------------------------- workloads


def decode_geometry():
    from sparse_attention_layer_b200 import configs
    from sparse_attention_layer_b200.flux import AttnCfg
    w = configs.LLAMA_DECODE
    cfg = AttnCfg(w.n_layers, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.sink, w.window)
    return w, cfg


def decode_bytes_per_layer(w, cfg, T: int, fa: bool) -> int:
    """Algorithmic bytes of one decode launch: K and V rows of every visible key plus
    q in and o out, for all sequences."""
    if fa:
        n_vis = T
    else:
        t = T - 1
        qb = t // cfg.block
        win_lo = max(0, (qb - cfg.window // cfg.block + 1) * cfg.block)
        n_vis = (T - win_lo) + min(cfg.sink, win_lo)
    kv = 2 * 2 * w.batch * cfg.n_kv_heads * cfg.head_dim * n_vis
    qo = 2 * 2 * w.batch * cfg.n_q_heads * cfg.head_dim
    return kv + qo


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

    def step(self, fa_events=None, sa_events=None):
        """One decode token for every sequence through all layers.  With fa_events /
        sa_events, the flux_decode call of every FA / SA layer is bracketed by CUDA
        events."""
        from sparse_attention_layer_b200 import flux
        m = self.model
        for layer in range(self.w.n_layers):
            c = m.caches[layer]
            flux.flux_kv_append(self.cfg, c.k, c.v, c.seq_len, self.k_new[layer],
                                self.v_new[layer])
            events = fa_events if self.fa[layer] else sa_events
            timed = events is not None
            if timed:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
            flux.flux_decode(self.cfg, layer, m.fa_mask, self.q[layer], c.k, c.v, c.seq_len,
                             self.o[layer], m.workspace)
            if timed:
                e1.record()
                events.append((e0, e1))

    # kernels of this library per step: one-kernel append, decode split + combine
    launches_per_step = property(lambda self: self.w.n_layers * 3)


class PrefillBench:
    """Llama-shape prefill: router on x_Q, then 32 x (KV append + FA/SA prefill), S=8192."""

    def __init__(self, seed: int):
        from sparse_attention_layer_b200 import configs, inputs
        from sparse_attention_layer_b200.flux import AttnCfg
        from sparse_attention_layer_b200.runtime import HybridAttention
        w = configs.LLAMA_PREFILL
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
        L, B, S = w.n_layers, w.batch, w.seq
        self.q = torch.randn(L, B, S, w.n_q_heads, w.head_dim, device="cuda",
                             generator=gen).to(torch.bfloat16)
        self.k = torch.randn(L, B, S, w.n_kv_heads, w.head_dim, device="cuda",
                             generator=gen).to(torch.bfloat16)
        self.v = torch.randn(L, B, S, w.n_kv_heads, w.head_dim, device="cuda",
                             generator=gen).to(torch.bfloat16)
        self.o = torch.empty(B, S, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
        # route once to learn the mask (the timed steps route again)
        self.model.route(*self.router, self.xq, w.pool_len, w.tau)
        words = self.model.fa_mask.cpu()[0]
        self.fa = [bool((int(words[i // 32]) >> (i % 32)) & 1) for i in range(L)]

    def reset(self):
        for c in self.model.caches:
            c.seq_len.zero_()

    def step(self, fa_events=None, router_events=None):
        from sparse_attention_layer_b200 import flux
        m, w = self.model, self.w
        if router_events is not None:
            e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
        m.route(*self.router, self.xq, w.pool_len, w.tau)
        if router_events is not None:
            e1.record(); router_events.append((e0, e1))
        for layer in range(w.n_layers):
            c = m.caches[layer]
            flux.flux_kv_append(self.cfg, c.k, c.v, c.seq_len, self.k[layer], self.v[layer])
            if fa_events is not None and self.fa[layer]:
                e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
            flux.flux_prefill(self.cfg, layer, m.fa_mask, self.q[layer], c.k, c.v, c.seq_len,
                              self.o)
            if fa_events is not None and self.fa[layer]:
                e1.record(); fa_events.append((e0, e1))

    launches_per_step = property(lambda self: 1 + self.w.n_layers * 3)  # route 1, append 2, prefill 1


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


def cpu_oracle_prefill_sample(n_rows: int = 16, seed: int = 9):
    """Time the fp64 oracle on n_rows query rows, evenly spaced over the Llama
    8192-token prompt, of one FA and one SA layer (all 32 heads); returns seconds per
    query row per layer for each route."""
    import numpy as np

    from oracle import flux_oracle as orc
    from sparse_attention_layer_b200 import configs, inputs
    w = configs.LLAMA_PREFILL
    S = w.seq
    q = inputs.normal_bf16((1, S, w.n_q_heads, w.head_dim), seed).float().numpy().astype(np.float64)
    shape = (1, w.n_kv_heads, S, w.head_dim)
    kc = inputs.normal_bf16(shape, seed + 1).float().numpy().astype(np.float64)
    vc = inputs.normal_bf16(shape, seed + 2).float().numpy().astype(np.float64)
    rows = np.linspace(0, S - 1, n_rows).astype(np.int64)
    out = {}
    for fa in (True, False):
        t0 = time.perf_counter()
        orc.attention_layer(q, kc, vc, np.array([S]), np.array([fa]), w.block, w.sink, w.window,
                            rows=rows)
        out[fa] = (time.perf_counter() - t0) / n_rows
    return out


def cpu_baseline_decode_tok_s(w, n_sa, n_seq=2):
    per = cpu_oracle_decode_sample(n_seq)
    per_seq_step = (w.n_layers - n_sa) * per[True] + n_sa * per[False]
    return 1.0 / per_seq_step, per


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
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_seq_step * 1e3 * w.batch, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": decode_config(w, cfg, sa),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: one decode token of 1 of the 16 sequences at "
                                   "32768 context, one FA and one SA layer, scaled to 16 FA + "
                                   "16 SA layers; a batch of 16 costs 16x (sequences are "
                                   "independent)"},
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


def run_flux(args, world, rank, local):
    from sparse_attention_layer_b200 import flux
    peaks, peak_kind = load_peaks()
    db = DecodeBench(seed=1234 + rank)
    w, cfg = db.w, db.cfg
    sa_layers = list(db.sa_layers)

    # ---------------- decode: main metric
    db.reset()
    for _ in range(args.warmup):
        db.step()
    db.reset()
    sampler = ClockSampler(local)
    barrier(world)
    sampler.start()
    fa_events, sa_events = [], []
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(world)
    start.record()
    for _ in range(args.steps):
        db.step(fa_events=fa_events, sa_events=sa_events)
    end.record()
    barrier(world)
    st = flux.flux_get_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the decode steps")
    t_ms = max_over_ranks(start.elapsed_time(end), world)
    ms_step = t_ms / args.steps
    value = replica_tokens_per_s(world, w.batch, args.steps, t_ms)
    fa_ms = elapsed_ms(fa_events)
    # the timed steps run contexts 32769 .. 32768 + K; take the mean context
    T_mean = w.seq + (args.steps + 1) / 2.0
    fa_bytes = decode_bytes_per_layer(w, cfg, int(round(T_mean)), True)
    achieved = fa_bytes / (statistics.mean(fa_ms) / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": "flux_decode (split-KV + combine), FA layers",
                "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_kind": f"{peak_kind} hbm_gbs",
                "traffic": measured_traffic("decode_split", w.batch),
                "traffic_note": "ncu dram bytes of a 4-sequence capture scaled to 16",
                "launch_ms": statistics.mean(fa_ms),
                "algorithmic_bytes_per_launch": fa_bytes}
    sa_bytes = decode_bytes_per_layer(w, cfg, int(round(T_mean)), False)
    sa_ms = elapsed_ms(sa_events) if sa_events else None
    roofline_sa = None if not sa_ms else {
        "bound": "hbm", "kernel": "flux_decode (split-KV + combine), SA layers",
        "achieved": sa_bytes / (statistics.mean(sa_ms) / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
        "unit": "GB/s",
        "frac": sa_bytes / (statistics.mean(sa_ms) / 1e3) / 1e9 / peaks["hbm_gbs"],
        "peak_kind": f"{peak_kind} hbm_gbs", "launch_ms": statistics.mean(sa_ms),
        "algorithmic_bytes_per_launch": sa_bytes}
    step_bytes = sum(decode_bytes_per_layer(w, cfg, int(round(T_mean)), fa) for fa in db.fa)

    # ---------------- decode as one CUDA graph per step (the headline number)
    from sparse_attention_layer_b200.runtime import DecodeStepGraph
    db.reset()
    graph = DecodeStepGraph(db.model, db.q, db.k_new, db.v_new, db.o)
    db.reset()
    for _ in range(args.warmup):  # warm-up replays outside the timed region
        graph.replay()
    db.reset()
    barrier(world)
    gs = torch.cuda.Event(enable_timing=True)
    ge = torch.cuda.Event(enable_timing=True)
    gs.record()
    for _ in range(args.steps):
        graph.replay()
    ge.record()
    barrier(world)
    clocks = sampler.stop()  # sampled over the eager and the graph timed regions
    tg_ms = max_over_ranks(gs.elapsed_time(ge), world)
    eager = {"value": value, "ms_per_step": ms_step,
             "what": "the same steps as 3 x 32 separate launches from Python"}
    value = replica_tokens_per_s(world, w.batch, args.steps, tg_ms)
    ms_step = tg_ms / args.steps
    st = flux.flux_get_device_status()
    if st:
        raise RuntimeError(f"device status {st:#x} after the graph decode steps")

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
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
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
    freed = db.model.evict_sa_layers()
    torch.cuda.synchronize()
    kv_evicted = db.model.kv_bytes()
    db.reset()
    for c in db.model.caches:
        c.seq_len.fill_(db.ctx)
    ring_graph = DecodeStepGraph(db.model, db.q, db.k_new, db.v_new, db.o)
    for c in db.model.caches:
        c.seq_len.fill_(db.ctx)
    for _ in range(args.warmup):
        ring_graph.replay()
    for c in db.model.caches:
        c.seq_len.fill_(db.ctx)
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
    per_seq_full = kv_full / w.batch
    per_seq_evicted = kv_evicted / w.batch
    hbm_budget = 160 * gib  # leaves room for weights and activations on a 180 GB part
    eviction = {
        "kv_gib_full": kv_full / gib, "kv_gib_evicted": kv_evicted / gib,
        "saving": 1.0 - kv_evicted / kv_full,
        "decode_tokens_per_s": replica_tokens_per_s(world, w.batch, args.steps, tr_ms),
        "ms_per_step": tr_ms / args.steps,
        "max_batch_in_160_gib": {"full": int(hbm_budget // per_seq_full),
                                 "evicted": int(hbm_budget // per_seq_evicted)},
        "what": "the 16 SA layers' caches moved to rings of sink 128 + 2048 rows per "
                "(sequence, KV head) after prefill; the same graph-replayed decode step",
    }
    launches_per_step = db.launches_per_step
    del ring_graph, db
    torch.cuda.empty_cache()

    # ---------------- prefill phase (Llama shape, 8192 tokens, router-chosen routes)
    pb = PrefillBench(seed=99 + rank)
    for _ in range(max(1, min(args.warmup, 3))):
        pb.reset()
        pb.step()
    n_pf = max(3, min(10, args.steps))
    pf_ms, fa_ev, rt_ev = [], [], []
    barrier(world)
    for _ in range(n_pf):
        pb.reset()
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
        a.record()
        pb.step(fa_events=fa_ev, router_events=rt_ev)
        b.record()
        pf_ms.append((a, b))
    barrier(world)
    pf_step = max_over_ranks(statistics.mean(elapsed_ms(pf_ms)), world)
    fa_launch = statistics.mean(elapsed_ms(fa_ev))
    flops_fa = prefill_flops_per_layer(pb.cfg, pb.w.seq, True)
    flops_sa = prefill_flops_per_layer(pb.cfg, pb.w.seq, False)
    n_fa = sum(pb.fa)
    tflops = flops_fa / (fa_launch / 1e3) / 1e12
    prefill = {
        "workload": "llama3.1-8b-shape prefill, 1 x 8192 tokens, router 4096->256->32 "
                    f"(seeded; {w.n_layers - n_fa} SA layers), SA sink 128 + window 2048",
        "tokens_per_s": world * pb.w.batch * pb.w.seq / (pf_step / 1e3),
        "ms_per_step": pf_step, "steps": n_pf, "sa_layers": pb.w.n_layers - n_fa,
        "router_ms": statistics.mean(elapsed_ms(rt_ev)),
        "algorithmic_tflops_per_step": (n_fa * flops_fa + (pb.w.n_layers - n_fa) * flops_sa) / 1e12,
        # The FA launches are timed inside back-to-back 32-layer prefill steps (GPU busy
        # for the whole phase, at the power cap), so the peak is the sustained one; the
        # fraction of the burst peak (a kernel timed alone) is given beside it.
        "roofline": {"bound": "tensor", "kernel": "prefill_kernel<128> (tcgen05), FA layers",
                     "achieved": tflops, "peak": peaks["bf16_tflops_sustained"],
                     "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops_sustained"],
                     "peak_kind": f"{peak_kind} bf16_tflops_sustained (timed inside a long step)",
                     "frac_of_burst_peak": tflops / peaks["bf16_tflops"],
                     "traffic": measured_traffic("prefill", pb.w.batch),
                     "launch_ms": fa_launch, "algorithmic_flops_per_launch": flops_fa},
        "gpu_launches_per_step": pb.launches_per_step,
        "cpu_baseline": None,
    }
    if world == 1 and rank == 0 and not args.no_cpu:
        # the oracle on sampled query rows, extrapolated to the whole prompt (every row of
        # 32 layers with this step's routes); a baseline, not a target
        t0 = time.perf_counter()
        per_row = cpu_oracle_prefill_sample()
        sec = pb.w.seq * (n_fa * per_row[True] + (pb.w.n_layers - n_fa) * per_row[False])
        prefill["cpu_baseline"] = {
            "value": pb.w.seq / sec, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "extrapolated": True,
            "sample": "16 evenly spaced query rows x 32 heads of one FA and one SA layer of the "
                      "8192-token prompt (fp64 oracle), extrapolated to all rows of "
                      f"{n_fa} FA + {pb.w.n_layers - n_fa} SA layers; "
                      f"{time.perf_counter() - t0:.1f} s of CPU time"}
    del pb
    torch.cuda.empty_cache()

    # ---------------- CPU baseline (rank 0, N = 1 only)
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu:
        t0 = time.perf_counter()
        tok_s, per = cpu_baseline_decode_tok_s(w, len(sa_layers), n_seq=2)
        cpu = {"value": tok_s, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": "one decode token of 2 of the 16 sequences at 32768 context for one FA "
                         "and one SA layer (fp64 oracle), scaled to 16 FA + 16 SA layers; "
                         f"{time.perf_counter() - t0:.1f} s of CPU time"}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": decode_config(w, cfg, sa_layers),
        "roofline": roofline, "roofline_sa": roofline_sa,
        "decode_step": {"algorithmic_gb_per_step": step_bytes / 1e9,
                        "step_gb_per_s": step_bytes / (ms_step / 1e3) / 1e9,
                        "fa_layer_bytes": fa_bytes, "sa_layer_bytes": sa_bytes},
        "cpu_baseline": cpu, "e2e": e2e, "decode_eager": eager,
        "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
        "prefill": prefill, "routing_mix": mix, "sa_kv_eviction": eviction,
    }
    if rank == 0:
        print(json.dumps(line))



def run_sweep(args):
    """Routing-mix x context x batch sweep of the Llama-3.1-8B shape (32 layers, 32/8
    heads, d 128, sink 128 + window 2048, block 128).  Every point is a measured
    32-layer step replayed from a CUDA graph with the given fraction of layers routed to
    SA (a fixed seeded choice of layers):
      decode  -- KV append + FA/SA decode per layer; the layers cycle over n distinct
                 KV caches, n = 32 where they fit in 120 GB and at least 512 MB of
                 cache is read between two visits of the same cache (so repeated
                 layers are not served from L2);
      prefill -- batch 1, KV append + FA/SA prefill on 32 separate caches.
    Per-layer FA and SA times are the 0 % and 100 % steps divided by 32."""
    from sparse_attention_layer_b200 import configs, inputs
    from sparse_attention_layer_b200.flux import AttnCfg
    from sparse_attention_layer_b200.runtime import HybridAttention
    torch.cuda.set_device(0)
    n_layers = 32
    cfg = AttnCfg(n_layers, 32, 8, 128, 128, 128, 2048)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    fracs = configs.SWEEP_SA_FRACTIONS
    out = {"decode": [], "prefill": []}

    def graph_ms(graph, warm, reps):
        for _ in range(warm):
            graph.replay()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for a, b in ev:
            a.record(); graph.replay(); b.record()
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    def mask_for(model, batch, frac):
        sa = inputs.fixed_sa_layers(n_layers, int(round(frac * n_layers)), seed=11)
        model.set_mask(inputs.pack_bits_u32(inputs.fa_bits_from_sa_layers(batch, n_layers, sa)).cuda())

    warm, reps = 3, 10
    sampler = ClockSampler(0)
    sampler.start()
    for T in configs.SWEEP_CONTEXTS:
        for B in configs.SWEEP_BATCHES:
            cap = T + n_layers * (warm + reps + 1) + 64
            cache_bytes = 2 * B * cfg.n_kv_heads * cap * cfg.head_dim * 2
            n_cache = max(1, min(n_layers, -(-512 * 2**20 // cache_bytes), (120 << 30) // cache_bytes))
            m = HybridAttention(cfg, B, cap, "cuda", layers=n_cache)
            for c in m.caches:
                c.k.normal_(generator=gen)
                c.v.normal_(generator=gen)
            q = torch.randn(B, 32, 128, device="cuda", generator=gen).to(torch.bfloat16)
            kn = torch.randn(B, 1, 8, 128, device="cuda", generator=gen).to(torch.bfloat16)
            o = torch.empty_like(q)

            def step():
                for layer in range(n_layers):
                    m.decode_layer(layer, q, kn, kn, o, cache_index=layer % n_cache)
            for c in m.caches:
                c.seq_len.fill_(T)
            step()
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            row = {"context": T, "batch": B, "distinct_caches": n_cache}
            for f in fracs:
                mask_for(m, B, f)
                for c in m.caches:
                    c.seq_len.fill_(T)
                ms = graph_ms(graph, warm, reps)
                row[f"{int(f * 100)}%"] = {"ms_per_step": ms, "tokens_per_s": B / (ms / 1e3)}
            base = row["0%"]["ms_per_step"]
            for f in fracs:
                row[f"{int(f * 100)}%"]["speedup_vs_all_fa"] = base / row[f"{int(f * 100)}%"]["ms_per_step"]
            row["fa_layer_ms"] = base / n_layers
            row["sa_layer_ms"] = row["100%"]["ms_per_step"] / n_layers
            out["decode"].append(row)
            del graph, m, q, kn, o
            torch.cuda.empty_cache()
        # prefill: batch 1, 32 layers on separate caches whose lengths are views of one
        # tensor, so a single memset in the graph restarts every layer at length 0
        m = HybridAttention(cfg, 1, T, "cuda")
        lens = torch.zeros(n_layers, 1, dtype=torch.int32, device="cuda")
        for i, c in enumerate(m.caches):
            c.seq_len = lens[i]
        qp = torch.randn(1, T, 32, 128, device="cuda", generator=gen).to(torch.bfloat16)
        kp = torch.randn(1, T, 8, 128, device="cuda", generator=gen).to(torch.bfloat16)
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
        pw, pr = (1, 3) if T >= 65536 else (3, 5)
        for f in fracs:
            mask_for(m, 1, f)
            ms = graph_ms(graph, pw, pr)
            row[f"{int(f * 100)}%"] = {"ms": ms, "tokens_per_s": T / (ms / 1e3)}
        base = row["0%"]["ms"]
        for f in fracs:
            row[f"{int(f * 100)}%"]["speedup_vs_all_fa"] = base / row[f"{int(f * 100)}%"]["ms"]
        row["fa_layer_ms"] = base / n_layers
        row["sa_layer_ms"] = row["100%"]["ms"] / n_layers
        row["fa_tflops"] = prefill_flops_per_layer(cfg, T, True) / (row["fa_layer_ms"] / 1e3) / 1e12
        out["prefill"].append(row)
        del graph, m, lens, qp, kp, op
        torch.cuda.empty_cache()
    clocks = sampler.stop()
    from sparse_attention_layer_b200 import flux
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
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--sweep", action="store_true",
                    help="routing-mix x context x batch sweep (graph-replayed 32-layer steps)")
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

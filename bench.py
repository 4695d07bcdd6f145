"""Benchmark of the LightTransfer-Test prefill hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config gqa1p2b] [--impl ours|reference]

One step is one pass of the whole path over one prefill of the workload: for
every layer the causal GQA attention with its LSE fused with the lazy ratio
(lt_prefill_attn_ratio), the push of the layer's ratios into the device-resident
layer queue (lt_dqueue_push) and the compaction of the layer the queue demotes,
if any (lt_compact_kv_pending).  The whole step is one CUDA graph (no host round
trip).  The per-layer Q/K/V of all layers are resident in HBM before timing
(together far larger than the 126 MB L2, so no L2 flush is needed).  The plain
attention (lt_prefill_attn), the separate ratio pass from the LSE
(lt_lazy_ratio), the host queue and compaction (lt_compact_kv) are timed beside
it.

Rank 0 prints one JSON line.  With --gpus N > 1 (torchrun) every rank runs an
independent replica of the workload by default (--shard replicas): weak
scaling, value = work of all ranks / max-over-ranks device time.  With
--shard heads the ranks split ONE prefill by KV heads and all-gather the
per-head ratios of every layer (NCCL, inside the step's graph) before the
queue push: strong scaling, value = work of the one prefill / max-over-ranks
device time; per-kernel figures are then those of this rank's head slice.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "prefill attn+lazy-ratio TFLOP/s & % BF16 tensor peak; compaction GB/s; ratio ovh %"
ATTN_SOURCES = ["kv_cache_compression_tcgen05_b200/csrc/attn_fwd64.cuh", "kv_cache_compression_tcgen05_b200/csrc/attn_fwd.cuh",
                "kv_cache_compression_tcgen05_b200/csrc/lt_device.cuh"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_digest(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(config_name):
    """DRAM bytes per attention launch from the committed ncu summary, or None if
    the kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"attn_fwd64_{config_name}.traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha") != source_digest(ATTN_SOURCES):
        return None
    return rec.get("dram_bytes_per_launch")


def attention_flops(cfg):
    """Algorithmic causal FLOPs of one layer: 4 d per (query, key <= query, head)."""
    return 4.0 * cfg.d * cfg.hq * cfg.causal_pairs()


def ratio_flops(cfg):
    """2 d FLOPs per (observed row, head, key in K_i)."""
    total = 0
    for n in cfg.seqlens:
        nb = min(cfg.n_obs, n)
        for i in range(n - nb, n):
            total += min(cfg.S + cfg.W, i + 1)
    return 2.0 * cfg.d * cfg.hq * total


def ratio_unique_bytes(cfg):
    """Bytes the separate ratio pass must touch once per layer: the observed Q
    rows and their LSE, and the union of the key rows they see (sinks plus the
    window band of all observed rows)."""
    total = 0
    for n in cfg.seqlens:
        obs = min(cfg.n_obs, n)
        band = min(n, cfg.S + cfg.W + obs - 1)
        total += obs * cfg.hq * (2 * cfg.d + 4) + band * cfg.hkv * 2 * cfg.d
    return total


def compaction_bytes(cfg, n_layers):
    """Bytes read + written by compacting n_layers demoted layers (K and V)."""
    rows = sum(min(n, cfg.S + cfg.W) for n in cfg.seqlens)
    return 2.0 * 2.0 * rows * cfg.hkv * cfg.d * 2 * n_layers


def kv_fraction_after_prefill(order, pool_len, seqlens, layers):
    """KV cache rows kept after the prefill over the rows of keeping every layer
    full: per sequence b, the (layers - demoted) full layers keep N_b rows each
    and each demoted layer the pool_len rows of its streaming cache.
    order: [batch, budget] demoted layers (-1 past the count), pool_len:
    [budget, batch] rows in demotion slot k; both host tensors."""
    kept = total = 0
    for b, n in enumerate(seqlens):
        demoted = [k for k in range(order.shape[1]) if int(order[b, k]) >= 0]
        kept += (layers - len(demoted)) * n + sum(int(pool_len[k, b]) for k in demoted)
        total += layers * n
    return kept / total if total else 1.0


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus, need_group=False):
    """One process per GPU; a NCCL process group when several ranks run, or
    when the heads are split (a single rank then still takes the collective
    path)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local if world > 1 else 0)
    if world > 1 or need_group:
        import datetime
        if world == 1 and "MASTER_ADDR" not in os.environ:
            import socket
            with socket.socket() as sock:
                sock.bind(("127.0.0.1", 0))
                port = sock.getsockname()[1]
            os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="1")
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def max_over_ranks(x, world, device="cuda"):
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------ our arm

class Prefill:
    """The whole path over every layer of one prefill, inputs resident on the GPU.
    With a process group the heads are split over its ranks (this rank's slice
    of every layer's Q/K/V); otherwise this GPU holds all heads."""

    def __init__(self, cfg, lt, device="cuda", group=None, seqs=None):
        self.cfg, self.lt = cfg, lt
        if group is not None:
            q0, q1, k0, k1 = lt.head_shard(cfg.hq, cfg.hkv, torch.distributed.get_rank(group),
                                           torch.distributed.get_world_size(group))
        else:
            q0, q1, k0, k1 = 0, cfg.hq, 0, cfg.hkv
        self.seqs = list(range(cfg.batch)) if seqs is None else list(seqs)
        layers = []
        for l in range(cfg.layers):
            Q, K, V = synth.layer_inputs(cfg, l, device)
            if group is not None:
                Q, K, V = Q[:, q0:q1].contiguous(), K[:, k0:k1].contiguous(), V[:, k0:k1].contiguous()
            if seqs is not None:
                Q, K, V = (lt.pack_sequences(t, cfg.cu_seqlens(), self.seqs)[0] for t in (Q, K, V))
            layers.append((Q, K, V))
        self.heads = (q0, q1, k0, k1)
        # this rank's shape: its heads and its sequences
        self.local = dataclasses.replace(cfg, hq=q1 - q0, hkv=k1 - k0,
                                         seqlens=tuple(cfg.seqlens[b] for b in self.seqs))
        lc = self.local
        cu = torch.tensor(lc.cu_seqlens(), dtype=torch.int32, device=device) if lc.batch > 1 else None
        self.step = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, cu_seqlens=cu,
                                   max_seqlen=lc.max_seqlen, group=group)
        st = self.step
        self.layers, self.O, self.LSE, self.ratio = st.layers, st.O, st.LSE, st.ratio
        self.K_pool, self.V_pool, self.pool_len = st.K_pool, st.V_pool, st.pool_len
        self.Kp, self.Vp, self.dq, self.kw = st.Kp, st.Vp, st.dq, st.kw

    def enqueue_step(self, stream, events=None):
        """Enqueue one whole step on `stream`; `events` collects an (start, end)
        pair of external timing events around every attention launch."""
        self.step.enqueue(stream, events=events)


def run_ours(args, cfg, rank, world):
    import kv_cache_compression_tcgen05_b200 as lt
    lt.library()
    peaks, peak_src = load_peaks()
    sharded = args.shard != "replicas"
    pf = Prefill(cfg, lt, group=torch.distributed.group.WORLD if args.shard == "heads" else None,
                 seqs=lt.sequence_shard(cfg.seqlens, rank, world) if args.shard == "sequences" else None)
    lc = pf.local   # this rank's shape: all heads and sequences, or its slice when sharded
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())   # the inputs were made on the default stream
    with torch.cuda.stream(stream):
        pf.enqueue_step(stream)           # eager warm-up: per-device set-up happens outside capture
    torch.cuda.synchronize()
    if args.decode_only:
        # One prefill step for the demotions, then the decode leg alone (a
        # short command for profiling the decode kernel).
        return {"metric": "decode after prefill", "config": cfg.name, **measure_decode(lc, lt, pf, peaks)}
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        pf.enqueue_step(stream)
    # K whole steps in one graph for the timed region; a second graph with
    # timing events around every attention launch gives the per-launch
    # duration (event nodes between kernels would also end the programmatic
    # launch overlap, so they stay out of the timed graph).
    g_timed = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_timed, stream=stream):
        for _ in range(args.steps):
            pf.enqueue_step(stream)
    g_events = torch.cuda.CUDAGraph()
    fused_ev = []
    with torch.cuda.graph(g_events, stream=stream):
        for _ in range(2):
            pf.enqueue_step(stream, events=fused_ev)
    for _ in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize()
    barrier(world)

    # Device-timed region: K whole steps (one graph replay).
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        with torch.cuda.stream(stream):
            torch.cuda.synchronize()
            start.record(stream)
            g_timed.replay()
            stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    launches = args.steps * pf.step.kernel_launches()
    ms = max_over_ranks(start.elapsed_time(stop), world) / args.steps
    with torch.cuda.stream(stream):
        g_events.replay()
    torch.cuda.synchronize()
    del g_step, g_timed, g_events   # before any process-group teardown (they may hold NCCL calls)
    t_fused = statistics.mean(a.elapsed_time(b) for a, b in fused_ev) * 1e-3
    # The demotions of the timed steps equal the host queue's on the same ratios
    # (all heads' ratios: the gathered ones when the heads are split), and every
    # rank demotes the same layers.
    mask_dev, order_dev = pf.dq.result()
    host_order = []
    r = pf.step.all_head_ratios().cpu().numpy()
    for b in range(lc.batch):
        q = lt.LayerQueue(cfg.layers, cfg.budget)
        host_order.append([x for x in (q.push(l, lt.lt_layer_score(r[l, b])) for l in range(cfg.layers)) if x >= 0])
        q.close()
    queue_agrees = all(order_dev[b].tolist() == host_order[b] for b in range(lc.batch))
    kv_frac = kv_fraction_after_prefill(order_dev.cpu(), pf.pool_len.cpu(), lc.seqlens, cfg.layers)
    ranks_agree = True
    if world > 1 and args.shard == "heads":
        orders = [torch.empty_like(order_dev) for _ in range(world)]
        torch.distributed.all_gather(orders, order_dev.contiguous())
        ranks_agree = all(torch.equal(o, orders[0]) for o in orders)

    # Beside the step: the plain attention and the separate ratio pass per layer.
    kw = pf.kw
    attn_ev, ratio_ev = [], []
    for rep in range(2):
        for l in range(cfg.layers):
            Q, K, V = pf.layers[l]
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record()
            lt.lt_prefill_attn(Q, K, V, out=pf.O, lse=pf.LSE, **kw)
            e1.record()
            lt.lt_lazy_ratio(Q, K, pf.LSE, cfg.S, cfg.W, cfg.n_obs, out=pf.ratio[l], **kw)
            e2.record()
            if rep > 0:
                attn_ev.append((e0, e1))
                ratio_ev.append((e1, e2))
    torch.cuda.synchronize()
    t_attn = statistics.mean(a.elapsed_time(b) for a, b in attn_ev) * 1e-3
    t_ratio = statistics.mean(a.elapsed_time(b) for a, b in ratio_ev) * 1e-3

    if args.kernels_only:
        return {"metric": METRIC, "ms_per_step": round(ms, 4), "fused_us_per_layer": round(t_fused * 1e6, 2),
                "attn_us_per_layer": round(t_attn * 1e6, 2), "ratio_us_per_layer": round(t_ratio * 1e6, 2),
                "kv_cache_fraction_after_prefill": round(kv_frac, 4), "gpu_launches": launches}

    # Compaction timed on its own: every demoted layer of one step (inputs > L2 apart).
    mask1 = torch.ones(lc.batch, dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    c_times = []
    for rep in range(5):
        for l in range(cfg.budget):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            Q, K, V = pf.layers[l]
            e0.record()
            lt.lt_compact_kv(K, V, mask1, lc.S, lc.W, k_stream=pf.K_pool[0], v_stream=pf.V_pool[0],
                             stream_len=pf.pool_len[0], **kw)
            e1.record()
            torch.cuda.synchronize()
            if rep > 0:
                c_times.append(e0.elapsed_time(e1) * 1e-3)
    # All demoted layers of the step in one launch (the per-layer launch above is latency bound).
    _, order_now = pf.dq.result()
    demoted_layers = order_now[0].to(torch.int32).contiguous()
    n_dem = int((demoted_layers >= 0).sum())
    cb_times = []
    for rep in range(6):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lt.lt_compact_kv_layers(pf.Kp, pf.Vp, demoted_layers, lc.S, lc.W, pf.K_pool, pf.V_pool, pf.pool_len,
                                lc.total_tokens, lc.hkv, lc.d, **kw)
        e1.record()
        torch.cuda.synchronize()
        if rep > 0:
            cb_times.append(e0.elapsed_time(e1) * 1e-3)
    del flush
    t_comp = statistics.mean(c_times)
    t_comp_batch = statistics.median(cb_times)

    # Per-kernel figures are this rank's; the job is world whole prefills
    # (replicas) or the one prefill split over the ranks.
    fl_attn, fl_ratio = attention_flops(lc), ratio_flops(lc)
    job_flops = cfg.layers * (attention_flops(cfg) + ratio_flops(cfg)) * (1 if sharded else world)
    value = job_flops / (ms * 1e-3) / 1e12
    achieved = fl_attn / t_fused / 1e12
    peak_sus = float(peaks["bf16_tflops_sustained"])
    peak_burst = float(peaks["bf16_tflops"])
    traffic = recorded_traffic(cfg.name) if lc == cfg else None   # the record is of the all-heads launch
    comp_gbs = compaction_bytes(lc, 1) / t_comp / 1e9

    decode = measure_decode(lc, lt, pf, peaks)
    e2e = measure_e2e(args, lc, lt, pf, world, job_flops)
    cpu = cpu_baseline(cfg) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    clocks = clk.summary()
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V with per-layer sink bias; pages' datasets/weights absent)",
        "config": {
            "workload": f"{cfg.name}: {cfg.layers} layers, batch {cfg.batch}, seq {cfg.max_seqlen}, "
                        f"{cfg.hq} q heads / {cfg.hkv} KV heads, head_dim {cfg.d}, S={cfg.S}, W={cfg.W}, "
                        f"n_obs={cfg.n_obs}, budget {cfg.budget}",
            "layers": cfg.layers, "batch": cfg.batch, "seq_len": cfg.max_seqlen, "hq": cfg.hq, "hkv": cfg.hkv,
            "head_dim": cfg.d, "S": cfg.S, "W": cfg.W, "n_obs": cfg.n_obs, "budget": cfg.budget,
            "l2": "inputs of one step (all layers' Q/K/V) exceed L2; no flush between steps",
            "step": "one CUDA graph: queue init, all layers' ratio accumulators zeroed once, then per layer fused "
                    "attention+ratio, device queue push, device-driven compaction (programmatic dependent launch)",
            "parallelism": (f"heads split over {world} rank(s): this rank's q heads {pf.heads[0]}..{pf.heads[1] - 1}, "
                            f"KV heads {pf.heads[2]}..{pf.heads[3] - 1}; ratios all-gathered per layer (NCCL)"
                            if args.shard == "heads" else
                            f"sequences split over {world} rank(s) by causal work: rank 0's sequences {pf.seqs}; "
                            f"no exchange" if args.shard == "sequences" else
                            f"replicas x{world}" if world > 1 else "single GPU"),
        },
        "attn_tflops": round(achieved, 2),
        "attn_pct_of_burst_peak": round(100 * achieved / peak_burst, 2),
        "fused_attn_ratio_us_per_layer": round(t_fused * 1e6, 2),
        "attn_only_us_per_layer": round(t_attn * 1e6, 2),
        "attn_only_tflops": round(fl_attn / t_attn / 1e12, 2),
        "fused_ratio_overhead_pct": round(100 * (t_fused - t_attn) / t_attn, 3),
        "separate_ratio_us_per_layer": round(t_ratio * 1e6, 2),
        "separate_ratio_overhead_pct": round(100 * t_ratio / t_attn, 3),
        "compaction_gbs": round(comp_gbs, 1),
        "compaction_us_per_layer": round(t_comp * 1e6, 2),
        "compaction_batched_layers": n_dem,
        "compaction_batched_gbs": round(compaction_bytes(lc, n_dem) / t_comp_batch / 1e9, 1),
        "separate_ratio_unique_gbs": round(ratio_unique_bytes(lc) / t_ratio / 1e9, 1),
        "device_queue_matches_host_queue": queue_agrees,
        "kv_cache_fraction_after_prefill": round(kv_frac, 4),
        "ranks_demote_same_layers": ranks_agree,
        **decode,
        "roofline": {"kernel": "attn_fwd64_kernel (head_dim 64, fused with the lazy ratio)", "bound": "tensor",
                     "achieved": round(achieved, 2), "peak": peak_sus, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_sus, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
    }
    return line


def measure_decode(cfg, lt, pf, peaks):
    """One decode step (one new query per sequence, every layer) after the
    prefill: demoted layers read their S+W streaming cache, kept layers their
    full prefill cache.  Timed against the same step with every layer full.
    The demotions are sequence 0's (the benchmark workload has batch 1).  Each
    replay is timed alone with the 126 MB L2 flushed before it."""
    _, order = pf.dq.result()
    demoted = [int(x) for x in order[0].tolist() if x >= 0]
    slot_of = {l: k for k, l in enumerate(demoted)}
    B, d = cfg.batch, cfg.d
    g = torch.Generator(device="cuda").manual_seed(5)
    q = torch.randn((B, cfg.hq, d), generator=g, device="cuda").bfloat16()
    O = torch.empty_like(q)
    LSE = torch.empty((B, cfg.hq), dtype=torch.float32, device="cuda")
    cu_h = cfg.cu_seqlens()
    starts = torch.tensor(cu_h[:-1], dtype=torch.int32, device="cuda")
    lens = torch.tensor([cu_h[b + 1] - cu_h[b] for b in range(B)], dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()

    def full(l, s):
        _, K, V = pf.layers[l]
        lt.lt_decode_attn(q, K, V, lens, seq_start=starts, max_len=cfg.max_seqlen, out=O, lse=LSE, stream=s)

    def streaming(l, s):
        k = slot_of[l]
        lt.lt_stream_decode(q, pf.K_pool[k], pf.V_pool[k], pf.pool_len[k], out=O, lse=LSE, stream=s)

    def hybrid_step(s):
        for l in range(cfg.layers):
            (streaming if l in slot_of else full)(l, s)

    def full_step(s):
        for l in range(cfg.layers):
            full(l, s)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def timed(fn, reps=10):
        with torch.cuda.stream(stream):
            fn(stream)                       # eager warm-up outside capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            fn(stream)
        out = []
        for r in range(reps + 2):
            flush.zero_()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                graph.replay()
                e1.record(stream)
            torch.cuda.synchronize()
            if r >= 2:
                out.append(e0.elapsed_time(e1) * 1e-3)
        return statistics.median(out)

    t_hybrid = timed(hybrid_step)
    t_full = timed(full_step)
    t_full_layer = timed(lambda s: full(0, s), reps=20)
    t_stream_layer = timed(lambda s: streaming(demoted[0], s), reps=20) if demoted else None
    del flush
    n_rows = sum(cu_h[b + 1] - cu_h[b] for b in range(B))
    full_bytes = n_rows * cfg.hkv * d * 2 * 2 + 2 * B * cfg.hq * d * 2 + B * cfg.hq * 4
    peak_hbm = float(peaks["hbm_gbs"])
    gbs = full_bytes / t_full_layer / 1e9
    out = {
        "decode_layers_streaming": len(demoted),
        "decode_hybrid_us_per_token": round(t_hybrid * 1e6, 2),
        "decode_all_full_us_per_token": round(t_full * 1e6, 2),
        "decode_speedup_vs_all_full": round(t_full / t_hybrid, 3),
        "decode_full_layer_us": round(t_full_layer * 1e6, 2),
        "decode_full_layer_gbs": round(gbs, 1),
        "decode_full_layer_frac_of_hbm": round(gbs / peak_hbm, 4),
    }
    if t_stream_layer is not None:
        slots = cfg.S + cfg.W
        s_bytes = B * cfg.hkv * min(slots, max(cu_h[b + 1] - cu_h[b] for b in range(B))) * d * 2 * 2
        out["decode_stream_layer_us"] = round(t_stream_layer * 1e6, 2)
        out["decode_stream_layer_gbs"] = round(s_bytes / t_stream_layer / 1e9, 1)
    return out


def measure_e2e(args, cfg, lt, pf, world, job_flops):
    """Same metric through the public calls with host buffers: every step copies
    each layer's Q/K/V from pinned host memory to the device and reads back each
    layer's O and LSE, the ratios and the streaming KV pool, all inside the
    device-timed region.  Uploads run one layer ahead on a side stream and
    read-backs on another, so copies overlap the kernels; the queue lives on the
    device, so no step waits for the host.  The full K/V of every layer stay on
    the device (the KV cache the queue manages); Q is double buffered.  `cfg` is
    this rank's shape (its slice when the heads or sequences are split);
    job_flops the work of the whole job per step."""
    host = [tuple(t.cpu().pin_memory() for t in lay) for lay in pf.layers]
    T, H, d = cfg.total_tokens, cfg.hq, cfg.d
    dev_q = [torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    dev_kv = [tuple(torch.empty_like(t) for t in lay[1:]) for lay in pf.layers]
    step = lt.PrefillStep([(dev_q[l % 2],) + dev_kv[l] for l in range(cfg.layers)], cfg.budget, cfg.S, cfg.W,
                          cfg.n_obs, group=pf.step.group, **pf.kw)
    o_host = torch.empty((cfg.layers, T, H, d), dtype=torch.bfloat16, pin_memory=True)
    lse_host = torch.empty((cfg.layers, H, T), dtype=torch.float32, pin_memory=True)
    ratio_host = torch.empty(step.ratio.shape, dtype=torch.float32, pin_memory=True)
    ks_host = torch.empty(step.K_pool.shape, dtype=torch.bfloat16, pin_memory=True)
    vs_host = torch.empty_like(ks_host)
    O = [torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    LSE = [torch.empty((H, T), dtype=torch.float32, device="cuda") for _ in range(2)]
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()
    h2d = sum(t.numel() * t.element_size() for lay in host for t in lay)
    d2h = o_host.numel() * 2 + lse_host.numel() * 4 + ratio_host.numel() * 4 + 2 * ks_host.numel() * 2

    def one_step():
        ready = [torch.cuda.Event() for _ in range(cfg.layers)]
        done = [torch.cuda.Event() for _ in range(cfg.layers)]
        computed = [torch.cuda.Event() for _ in range(cfg.layers)]

        def upload(l):
            with torch.cuda.stream(copy_in):
                if l >= 2:
                    copy_in.wait_event(done[l - 2])   # Q buffer and O/LSE of layer l-2 consumed
                dev_q[l % 2].copy_(host[l][0], non_blocking=True)
                dev_kv[l][0].copy_(host[l][1], non_blocking=True)
                dev_kv[l][1].copy_(host[l][2], non_blocking=True)
                ready[l].record(copy_in)

        step.begin(main)
        upload(0)
        for l in range(cfg.layers):
            if l + 1 < cfg.layers:
                upload(l + 1)
            main.wait_event(ready[l])
            step.layer(l, main, O=O[l % 2], LSE=LSE[l % 2])
            computed[l].record(main)
            with torch.cuda.stream(copy_out):
                copy_out.wait_event(computed[l])
                o_host[l].copy_(O[l % 2], non_blocking=True)
                lse_host[l].copy_(LSE[l % 2], non_blocking=True)
                done[l].record(copy_out)
        with torch.cuda.stream(copy_out):
            copy_out.wait_stream(main)
            ratio_host.copy_(step.ratio, non_blocking=True)
            ks_host.copy_(step.K_pool, non_blocking=True)
            vs_host.copy_(step.V_pool, non_blocking=True)
        main.wait_stream(copy_out)
        main.wait_stream(copy_in)

    for _ in range(2):
        one_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(1, min(args.steps, 5))
    e0.record()
    for _ in range(steps):
        one_step()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    return {"value": round(job_flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 3)}


# ------------------------------------------------------------- CPU (oracle)

def oracle_sample(cfg, seconds, seed=0):
    """Time the fp64 oracle on a bounded random sample of the workload's rows:
    attention rows (uniform over tokens and heads) of layer 0 plus the lazy
    ratio of a proportional share of the observed rows.  Returns
    (TFLOP/s, cores, description)."""
    import oracle
    Q, K, V = synth.layer_inputs(cfg, 0, "cpu")
    q, k, v = synth.bf16_bits(Q), synth.bf16_bits(K), synth.bf16_bits(V)
    cu = np.array(cfg.cu_seqlens(), np.int32)
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(seed)
    starts = np.array(cfg.cu_seqlens()[:-1])

    def run(n):
        toks = rng.integers(0, cfg.total_tokens, n).astype(np.int32)
        heads = rng.integers(0, cfg.hq, n).astype(np.int32)
        pos = toks - starts[np.searchsorted(starts, toks, side="right") - 1]
        t0 = time.perf_counter()
        oracle.attn(cu, q, k, v, tokens=toks, heads=heads, nthreads=cores)
        t = time.perf_counter() - t0
        return 4.0 * cfg.d * float(np.sum(pos + 1)), t

    fl, t = run(64)
    n = int(min(200000, max(64, 64 * seconds / max(t, 1e-3))))
    fl, t = run(n)
    return fl / t / 1e12, cores, f"{n} random (token, head) attention rows of layer 0 ({fl / 1e9:.1f} GFLOP, {t:.1f} s)"


def cpu_baseline(cfg, seconds=10.0):
    v, cores, desc = oracle_sample(cfg, seconds)
    return {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return None
    vals = []
    desc = ""
    for _ in range(args.warmup):
        oracle_sample(cfg, 2.0, seed=1)
    t0 = time.perf_counter()
    for s in range(args.steps):
        v, cores, desc = oracle_sample(cfg, 5.0, seed=100 + s)
        vals.append(v)
    ms = (time.perf_counter() - t0) * 1e3 / max(1, args.steps)
    value = statistics.mean(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name} (fp64 CPU oracle on a bounded random row sample per step)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="gqa1p2b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="one prefill step, then only the decode measurement (for profiling the decode kernel)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads", "sequences"],
                    help="with several GPUs: independent replicas (weak scaling, default); one prefill with its "
                         "KV heads split over the ranks and the ratios all-gathered per layer; or a packed batch "
                         "split by whole sequences, no exchange (both strong scaling)")
    ap.add_argument("--kernels-only", action="store_true",
                    help="time only the device steps (no e2e, CPU baseline or compaction leg); for profiling")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    cfg = synth.CONFIGS[args.config]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, cfg, rank, args.gpus)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    rank, world, _ = dist_setup(args.gpus, need_group=args.shard == "heads")
    line = run_ours(args, cfg, rank, world)   # frees its CUDA graphs (they may hold NCCL calls) on return
    torch.cuda.synchronize()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

"""Benchmark of the LightTransfer-Test prefill hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config long128k] [--impl ours|reference]

One step is one pass of the whole path over one prefill of the workload: for
every layer the causal GQA attention with its LSE fused with the lazy ratio and
the push of the layer's ratios into the device-resident layer queue
(lt_prefill_attn_ratio_push: the attention's last CTA pushes), then the
compaction of the layer the queue demotes.  On the long-context workload
(long128k, the default: the largest that one GPU holds, and the one whose
prefill runs the queue online under the peak-memory cap) the step keeps the
full KV of at most C + 1 layers: lt_kv_pool_commit reduces the demoted layer
to its streaming rows and stores the current layer in the freed slot.  The
whole step is one CUDA graph (no host round trip).  The per-layer Q/K/V of all
layers are resident in HBM before timing (far larger than the 126 MB L2, so no
L2 flush is needed between steps); in the capped mode they stand for the
projections' outputs, each read only while its layer runs.  The plain
attention (lt_prefill_attn), the separate ratio pass from the LSE
(lt_lazy_ratio) and compaction (lt_compact_kv) are timed beside it.

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
                "kv_cache_compression_tcgen05_b200/csrc/lt_device.cuh", "kv_cache_compression_tcgen05_b200/csrc/dqueue.cuh"]
# A per-launch time averaged over at least this long is taken under the
# sustained (power-capped) tensor peak; shorter ones under the burst peak.
SUSTAINED_REGION_S = 1.0


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


def recorded_traffic(config_name, d):
    """DRAM bytes per attention launch from the committed ncu summary of the
    head_dim-d kernel on this workload, or None if there is none or the kernel
    source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"attn_fwd{d}_{config_name}.traffic.txt")
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


def choose_peak(peaks, region_s):
    """(peak TFLOP/s, source) for a kernel whose per-launch time was averaged
    over region_s seconds of back-to-back work: the measured sustained bf16
    peak (a seconds-long loop under the power cap) when that region lasts
    seconds, else the burst peak."""
    if region_s >= SUSTAINED_REGION_S:
        return float(peaks["bf16_tflops_sustained"]), (
            f"bf16_tflops_sustained: per-launch time averaged over {region_s:.1f} s of back-to-back launches "
            f"(>= {SUSTAINED_REGION_S:.0f} s)")
    return float(peaks["bf16_tflops"]), (
        f"bf16_tflops (burst): per-launch time averaged over {region_s:.3f} s (< {SUSTAINED_REGION_S:.0f} s)")


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
    of every layer's Q/K/V); otherwise this GPU holds all heads.  kv_pool: the
    step keeps the full KV of at most C + 1 layers (the capped prefill)."""

    def __init__(self, cfg, lt, device="cuda", group=None, seqs=None, kv_pool=False):
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
        # Device memory the step itself takes (its buffers and anything it
        # allocates while running), from here to the end of the first step.
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        self.mem_base = torch.cuda.memory_allocated()
        self.step = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, cu_seqlens=cu,
                                   max_seqlen=lc.max_seqlen, group=group, kv_pool=kv_pool)
        st = self.step
        self.kv_pool = kv_pool
        self.layers, self.O, self.LSE, self.ratio = st.layers, st.O, st.LSE, st.ratio
        self.K_pool, self.V_pool, self.pool_len = st.K_pool, st.V_pool, st.pool_len
        self.Kp, self.Vp, self.dq, self.kw = st.Kp, st.Vp, st.dq, st.kw

    def enqueue_step(self, stream, events=None):
        """Enqueue one whole step on `stream`; `events` collects an (start, end)
        pair of external timing events around every attention launch."""
        self.step.enqueue(stream, events=events)

    def kv_report(self, step_alloc_bytes):
        """The KV cache the step keeps (the method's memory outcome) and the
        device memory the step took, measured by the allocator."""
        st, cfg = self.step, self.local
        full, stream, held = st.kv_bytes()
        owned = sum(t.numel() * t.element_size() for t in (st.O, st.LSE, st.ratio, st.K_pool, st.V_pool,
                                                            st.pool_len, st.dq.state))
        if st.kv_pool:
            owned += 2 * st.K_full.numel() * st.K_full.element_size()
            peak = held + full            # the C slots, the working layer's own K/V, the streaming caches
        else:
            owned += 2 * st.Kp.numel() * 8
            peak = cfg.layers * full + cfg.budget * stream   # every layer stays full in the caller's tensors
        return {
            "mode": ("capped: C = L - budget full-KV slots plus the working layer's K/V" if st.kv_pool else
                     "every layer's full K/V resident (caller's tensors) plus the streaming caches"),
            "full_layer_bytes": full, "stream_layer_bytes": stream,
            "peak_kv_bytes": peak, "all_full_kv_bytes": cfg.layers * full,
            "peak_kv_fraction_of_all_full": round(peak / (cfg.layers * full), 4),
            "bound_bytes": (cfg.layers - cfg.budget + 1) * full + cfg.budget * stream,
            "step_alloc_bytes_measured": int(step_alloc_bytes), "step_buffer_bytes": int(owned),
        }


def workload_config(cfg, kv_pool, world, shard):
    """The `config` of the JSON line (both arms): the workload and how a step
    runs it."""
    import kv_cache_compression_tcgen05_b200 as lt
    if shard == "heads":
        q0, q1, k0, k1 = lt.head_shard(cfg.hq, cfg.hkv, 0, world)
        par = (f"heads split over {world} rank(s): rank 0's q heads {q0}..{q1 - 1}, KV heads {k0}..{k1 - 1}; "
               f"ratios all-gathered per layer (NCCL)")
    elif shard == "sequences":
        par = (f"sequences split over {world} rank(s) by causal work: rank 0's sequences "
               f"{lt.sequence_shard(cfg.seqlens, 0, world)}; no exchange")
    else:
        par = f"replicas x{world}" if world > 1 else "single GPU"
    return {
        "workload": f"{cfg.name}: {cfg.layers} layers, batch {cfg.batch}, seq {cfg.max_seqlen}, "
                    f"{cfg.hq} q heads / {cfg.hkv} KV heads, head_dim {cfg.d}, S={cfg.S}, W={cfg.W}, "
                    f"n_obs={cfg.n_obs}, budget {cfg.budget}"
                    + (", online queue under the peak-memory cap (C+1 full-KV layers)" if kv_pool else ""),
        "layers": cfg.layers, "batch": cfg.batch, "seq_len": cfg.max_seqlen, "hq": cfg.hq, "hkv": cfg.hkv,
        "head_dim": cfg.d, "S": cfg.S, "W": cfg.W, "n_obs": cfg.n_obs, "budget": cfg.budget,
        "kv_pool": kv_pool,
        "l2": "inputs of one step (all layers' Q/K/V) exceed L2; no flush between steps",
        "step": "one CUDA graph: queue init, all layers' ratio accumulators zeroed once, then per layer fused "
                "attention+ratio+queue push, then " + ("the slot commit (compaction of the demoted layer, "
                                                       "store of the current one)" if kv_pool else
                                                       "device-driven compaction")
                + " (programmatic dependent launch)",
        "parallelism": par,
    }


def run_ours(args, cfg, rank, world):
    import kv_cache_compression_tcgen05_b200 as lt
    lt.library()
    peaks, peak_src = load_peaks()
    sharded = args.shard != "replicas"
    kv_pool = cfg.online if args.kv_pool == "auto" else args.kv_pool == "on"
    pf = Prefill(cfg, lt, group=torch.distributed.group.WORLD if args.shard == "heads" else None,
                 seqs=lt.sequence_shard(cfg.seqlens, rank, world) if args.shard == "sequences" else None,
                 kv_pool=kv_pool)
    lc = pf.local   # this rank's shape: all heads and sequences, or its slice when sharded
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())   # the inputs were made on the default stream
    t0 = time.perf_counter()
    with torch.cuda.stream(stream):
        pf.enqueue_step(stream)           # eager warm-up: per-device set-up happens outside capture
    torch.cuda.synchronize()
    t_eager = time.perf_counter() - t0
    step_alloc = torch.cuda.max_memory_allocated() - pf.mem_base
    if args.decode_only:
        # One prefill step for the demotions, then the decode leg alone (a
        # short command for profiling the decode kernel).
        return {"metric": "decode after prefill", "config": cfg.name, **measure_decode(lc, lt, pf, peaks)}
    long_step = t_eager > 0.5             # seconds-long steps: fewer repetitions beside the timed region
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
        for _ in range(1 if long_step else 2):
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
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        g_events.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    events_region_s = ev0.elapsed_time(ev1) * 1e-3
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

    # Beside the step: the plain attention and the separate ratio pass per
    # layer (all layers for short steps, the first four for long ones), captured
    # in one CUDA graph with external timing events around every launch, so the
    # times are the device's alone (no host gaps between eager launches).  The
    # fused kernel is timed in the same graph (its accumulate form, as in the
    # step), right after the plain one on the same inputs, so the ratio's
    # overhead compares the two kernels under the same conditions (clock,
    # power, L2).  Medians over the layers (every layer twice for short steps).
    kw = pf.kw
    side_layers = list(range(min(cfg.layers, 4))) if long_step else list(range(cfg.layers))
    attn_ev, ratio_ev, fused_eager_ev = [], [], []
    ratio_out = torch.empty_like(pf.ratio[0])
    side_events = []   # every event the graph records into lives until the graph is released

    def ev():
        e = torch.cuda.Event(enable_timing=True, external=True)
        side_events.append(e)
        return e

    g_side = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_side, stream=stream):
        for l in side_layers * (1 if long_step else 2):
            Q, K, V = pf.layers[l]
            e0, e1, e2, e2b, e3 = ev(), ev(), ev(), ev(), ev()
            e0.record(stream)
            lt.lt_prefill_attn(Q, K, V, out=pf.O, lse=pf.LSE, stream=stream, **kw)
            e1.record(stream)
            lt.lt_lazy_ratio(Q, K, pf.LSE, cfg.S, cfg.W, cfg.n_obs, out=ratio_out, stream=stream, **kw)
            e2.record(stream)
            ratio_out.zero_()      # outside the fused launch's events (accumulate form, as in the step)
            e2b.record(stream)
            lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, out=pf.O, lse=pf.LSE, ratio=ratio_out,
                                     accumulate=True, stream=stream, **kw)
            e3.record(stream)
            if not long_step or l > 0:
                attn_ev.append((e0, e1))
                ratio_ev.append((e1, e2))
                fused_eager_ev.append((e2b, e3))
    with torch.cuda.stream(stream):
        for _ in range(1 if long_step else 2):     # the last replay's events are read
            g_side.replay()
    torch.cuda.synchronize()
    t_attn = statistics.median(a.elapsed_time(b) for a, b in attn_ev) * 1e-3
    t_ratio = statistics.median(a.elapsed_time(b) for a, b in ratio_ev) * 1e-3
    t_fused_eager = statistics.median(a.elapsed_time(b) for a, b in fused_eager_ev) * 1e-3
    del g_side
    del side_events
    kv = pf.kv_report(step_alloc)

    if args.kernels_only:
        return {"metric": METRIC, "config": {"workload": cfg.name, "kv_pool": kv_pool},
                "ms_per_step": round(ms, 4), "fused_us_per_layer": round(t_fused * 1e6, 2),
                "fused_eager_us_per_layer": round(t_fused_eager * 1e6, 2),
                "fused_ratio_overhead_pct": round(100 * (t_fused_eager - t_attn) / t_attn, 3),
                "attn_us_per_layer": round(t_attn * 1e6, 2), "ratio_us_per_layer": round(t_ratio * 1e6, 2),
                "kv_cache_fraction_after_prefill": round(kv_frac, 4), "kv_cache": kv, "gpu_launches": launches,
                "events_region_s": round(events_region_s, 3)}

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
    Kp = pf.Kp if pf.Kp is not None else lt.layer_pointer_table([lay[1] for lay in pf.layers])
    Vp = pf.Vp if pf.Vp is not None else lt.layer_pointer_table([lay[2] for lay in pf.layers])
    cb_times = []
    for rep in range(6):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lt.lt_compact_kv_layers(Kp, Vp, demoted_layers, lc.S, lc.W, pf.K_pool, pf.V_pool, pf.pool_len,
                                lc.total_tokens, lc.hkv, lc.d, **kw)
        e1.record()
        torch.cuda.synchronize()
        if rep > 0:
            cb_times.append(e0.elapsed_time(e1) * 1e-3)
    del flush
    t_comp = statistics.mean(c_times)
    t_comp_batch = statistics.median(cb_times)
    # The step's own buffers (pools, queue) hold its result again for the legs below.
    with torch.cuda.stream(stream):
        pf.enqueue_step(stream)
    torch.cuda.synchronize()

    # Per-kernel figures are this rank's; the job is world whole prefills
    # (replicas) or the one prefill split over the ranks.
    fl_attn, fl_ratio = attention_flops(lc), ratio_flops(lc)
    job_flops = cfg.layers * (attention_flops(cfg) + ratio_flops(cfg)) * (1 if sharded else world)
    value = job_flops / (ms * 1e-3) / 1e12
    achieved = fl_attn / t_fused / 1e12
    peak, peak_why = choose_peak(peaks, events_region_s)
    peak_burst = float(peaks["bf16_tflops"])
    traffic = recorded_traffic(cfg.name, cfg.d) if lc == cfg else None   # the record is of the all-heads launch
    comp_gbs = compaction_bytes(lc, 1) / t_comp / 1e9

    decode = measure_decode(lc, lt, pf, peaks)
    e2e = measure_e2e(args, lc, lt, pf, world, job_flops, long_step)
    cpu = cpu_baseline(cfg) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    clocks = clk.summary()
    kernel = (f"attn_fwd64_kernel<fused> (head_dim 64, fused with the lazy ratio and the queue push)" if cfg.d == 64
              else f"attn_fwd_kernel<128, fused> (head_dim 128, fused with the lazy ratio and the queue push)")
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
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V with per-layer sink and recency biases; pages' datasets/weights "
                "absent)",
        "config": workload_config(cfg, kv_pool, world, args.shard),
        "attn_tflops": round(achieved, 2),
        "attn_pct_of_burst_peak": round(100 * achieved / peak_burst, 2),
        "fused_attn_ratio_push_us_per_layer_in_step": round(t_fused * 1e6, 2),
        "fused_attn_ratio_us_per_layer": round(t_fused_eager * 1e6, 2),
        "attn_only_us_per_layer": round(t_attn * 1e6, 2),
        "attn_only_tflops": round(fl_attn / t_attn / 1e12, 2),
        "fused_ratio_overhead_pct": round(100 * (t_fused_eager - t_attn) / t_attn, 3),
        "separate_ratio_us_per_layer": round(t_ratio * 1e6, 2),
        "separate_ratio_overhead_pct": round(100 * t_ratio / t_attn, 3),
        "compaction_gbs": round(comp_gbs, 1),
        "compaction_us_per_layer": round(t_comp * 1e6, 2),
        "compaction_batched_layers": n_dem,
        "compaction_batched_gbs": round(compaction_bytes(lc, n_dem) / t_comp_batch / 1e9, 1),
        "separate_ratio_unique_gbs": round(ratio_unique_bytes(lc) / t_ratio / 1e9, 1),
        "device_queue_matches_host_queue": queue_agrees,
        "kv_cache_fraction_after_prefill": round(kv_frac, 4),
        "kv_cache": kv,
        "ranks_demote_same_layers": ranks_agree,
        **decode,
        "roofline": {"kernel": kernel, "bound": "tensor",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "frac_of_burst": round(achieved / peak_burst, 4),
                     "traffic": traffic, "peak_source": f"{peak_src} {peak_why}",
                     "algorithmic_flop_per_launch": fl_attn},
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

    # Kept layers read their full cache: the layer's own tensors, or its
    # full-KV slot in the capped mode.
    slots = pf.dq.slots() if pf.kv_pool else None
    full_cache = {}
    for l in range(cfg.layers):
        if pf.kv_pool and l in slot_of:
            continue
        K, V, st = pf.step.kept_layer_cache(l, slots)
        full_cache[l] = (K, V, st if pf.kv_pool else starts)

    workspace = torch.empty(max(16, lt.lt_decode_splitk_workspace_bytes(B, cfg.hq, d, cfg.max_seqlen)),
                            dtype=torch.uint8, device="cuda")

    def full_cluster(l, s):
        K, V, st = full_cache[l] if l in full_cache else (pf.layers[l][1], pf.layers[l][2], starts)
        lt.lt_decode_attn(q, K, V, lens, seq_start=st, max_len=cfg.max_seqlen, out=O, lse=LSE, stream=s)

    def full_splitk(l, s):
        K, V, st = full_cache[l] if l in full_cache else (pf.layers[l][1], pf.layers[l][2], starts)
        lt.lt_decode_attn_splitk(q, K, V, lens, seq_start=st, max_len=cfg.max_seqlen, out=O, lse=LSE,
                                 workspace=workspace, stream=s)

    full_paths = {"cluster": full_cluster, "splitk": full_splitk}
    choice = {"path": "cluster"}

    def full(l, s):
        full_paths[choice["path"]](l, s)

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

    l0 = min(full_cache) if full_cache else 0
    t_path = {name: timed(lambda s, fn=fn: fn(l0, s), reps=20) for name, fn in full_paths.items()}
    choice["path"] = min(t_path, key=t_path.get)       # the faster full-cache decode for this length
    t_hybrid = timed(hybrid_step)
    t_full = timed(full_step)
    t_full_layer = t_path[choice["path"]]
    t_stream_layer = timed(lambda s: streaming(demoted[0], s), reps=20) if demoted else None
    del flush
    n_rows = sum(cu_h[b + 1] - cu_h[b] for b in range(B))
    full_bytes = n_rows * cfg.hkv * d * 2 * 2 + 2 * B * cfg.hq * d * 2 + B * cfg.hq * 4
    # K/V bytes a decode token reads: every layer full, or the demoted ones on
    # their streaming caches (the ratio the hybrid speed-up tends to when HBM bound).
    stream_rows = sum(min(cu_h[b + 1] - cu_h[b], cfg.S + cfg.W) for b in range(B))
    full_step_bytes = cfg.layers * n_rows * cfg.hkv * d * 4
    hybrid_step_bytes = ((cfg.layers - len(demoted)) * n_rows + len(demoted) * stream_rows) * cfg.hkv * d * 4
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
        "decode_full_layer_path": choice["path"],
        "decode_full_layer_us_by_path": {k: round(v * 1e6, 2) for k, v in t_path.items()},
        "decode_speedup_analytic_bytes": round(full_step_bytes / hybrid_step_bytes, 3),
    }
    if t_stream_layer is not None:
        slots = cfg.S + cfg.W
        s_bytes = B * cfg.hkv * min(slots, max(cu_h[b + 1] - cu_h[b] for b in range(B))) * d * 2 * 2
        out["decode_stream_layer_us"] = round(t_stream_layer * 1e6, 2)
        out["decode_stream_layer_gbs"] = round(s_bytes / t_stream_layer / 1e9, 1)
    return out


def measure_e2e(args, cfg, lt, pf, world, job_flops, long_step):
    """Same metric through the public calls with host buffers: every step copies
    each layer's Q/K/V from pinned host memory to the device and reads back the
    step's result -- the last layer's O and LSE, every layer's ratios and the
    demoted layers' streaming KV with its lengths -- all inside the
    device-timed region.  Uploads run one layer ahead on a side stream (two
    device buffers for Q, each reused every other layer) and the read-back on
    another, so copies overlap the kernels; the queue lives on the device, so
    no step waits for the host.  In the capped mode K/V take the same two
    device buffers (the step keeps its own C full-KV slots); otherwise every
    layer's K/V stays on the device (the KV cache the queue manages).  `cfg`
    is this rank's shape (its slice when the heads or sequences are split);
    job_flops the work of the whole job per step."""
    # Every rank of a node pins its own copy of the inputs: check that the host
    # has room for all of them before pinning (a failed pin would end the run).
    need = sum(t.numel() * t.element_size() for lay in pf.layers for t in lay)
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = None
    local = int(os.environ.get("LOCAL_WORLD_SIZE", world))
    skip = avail is not None and need * local > 0.7 * avail
    if max_over_ranks(1.0 if skip else 0.0, world) > 0:     # every rank takes the same branch
        avail = avail or 0
        return {"value": None, "unit": "TFLOP/s", "h2d_bytes_per_step": int(need), "d2h_bytes_per_step": 0,
                "skipped": f"{local} rank(s) x {need / 2**30:.1f} GiB of pinned inputs exceed 70% of the host's "
                           f"{avail / 2**30:.0f} GiB available"}
    host = []
    for lay in pf.layers:
        host.append(tuple(torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t) for t in lay))
    T, H, d = cfg.total_tokens, cfg.hq, cfg.d
    dev_q = [torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    if pf.kv_pool:
        bufs = [tuple(torch.empty_like(t) for t in pf.layers[0][1:]) for _ in range(2)]
        dev_kv = [bufs[l % 2] for l in range(cfg.layers)]
    else:
        dev_kv = [tuple(torch.empty_like(t) for t in lay[1:]) for lay in pf.layers]
    step = lt.PrefillStep([(dev_q[l % 2],) + dev_kv[l] for l in range(cfg.layers)], cfg.budget, cfg.S, cfg.W,
                          cfg.n_obs, group=pf.step.group, kv_pool=pf.kv_pool, **pf.kw)
    o_host = torch.empty((T, H, d), dtype=torch.bfloat16, pin_memory=True)
    lse_host = torch.empty((H, T), dtype=torch.float32, pin_memory=True)
    ratio_host = torch.empty(step.ratio.shape, dtype=torch.float32, pin_memory=True)
    ks_host = torch.empty(step.K_pool.shape, dtype=torch.bfloat16, pin_memory=True)
    vs_host = torch.empty_like(ks_host)
    len_host = torch.empty(step.pool_len.shape, dtype=torch.int32, pin_memory=True)
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()
    h2d = sum(t.numel() * t.element_size() for lay in host for t in lay)
    d2h = sum(t.numel() * t.element_size() for t in (o_host, lse_host, ratio_host, ks_host, vs_host, len_host))

    def one_step():
        ready = [torch.cuda.Event() for _ in range(cfg.layers)]
        computed = [torch.cuda.Event() for _ in range(cfg.layers)]

        def upload(l):
            with torch.cuda.stream(copy_in):
                if l >= 2:
                    copy_in.wait_event(computed[l - 2])   # layer l-2 no longer reads these buffers
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
            step.layer(l, main)
            computed[l].record(main)
        with torch.cuda.stream(copy_out):
            copy_out.wait_stream(main)
            o_host.copy_(step.O, non_blocking=True)
            lse_host.copy_(step.LSE, non_blocking=True)
            ratio_host.copy_(step.ratio, non_blocking=True)
            ks_host.copy_(step.K_pool, non_blocking=True)
            vs_host.copy_(step.V_pool, non_blocking=True)
            len_host.copy_(step.pool_len, non_blocking=True)
        main.wait_stream(copy_out)
        main.wait_stream(copy_in)

    for _ in range(1 if long_step else 2):
        one_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(1, min(args.steps, 2 if long_step else 5))
    e0.record()
    for _ in range(steps):
        one_step()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    ok = bool(torch.equal(step.ratio, pf.step.ratio))     # same result as the device-resident step
    return {"value": round(job_flops / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 3),
            "steps": steps, "ratios_match_device_inputs_step": ok}


# ------------------------------------------------------------- CPU (oracle)

_ORACLE_INPUTS = {}


def oracle_sample(cfg, seconds, seed=0):
    """Time the fp64 oracle, as it stands, on a bounded random sample of one
    layer's work in the metric's unit (algorithmic attention + lazy-ratio
    FLOPs per second): random (token, head) attention rows of layer 0 and
    random (observed row, head) lazy-ratio rows of layer 0, the latter in
    the proportion of the layer's ratio FLOPs to its attention FLOPs (at least
    one).  The oracle's ratio row takes its LSE from a full attention row
    (route A without a given LSE), so it costs about as much as one.
    Returns (TFLOP/s, cores, description)."""
    import oracle
    if cfg.name not in _ORACLE_INPUTS:   # drawn once per process: a long workload's layer takes seconds on the host
        _ORACLE_INPUTS.clear()
        _ORACLE_INPUTS[cfg.name] = tuple(synth.bf16_bits(t) for t in synth.layer_inputs(cfg, 0, "cpu"))
    q, k, v = _ORACLE_INPUTS[cfg.name]
    cu = np.array(cfg.cu_seqlens(), np.int32)
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(seed)
    starts = np.array(cfg.cu_seqlens()[:-1])
    obs = [(cu[b] + i, i) for b, n in enumerate(cfg.seqlens) for i in range(n - min(cfg.n_obs, n), n)]
    share = ratio_flops(cfg) / attention_flops(cfg)

    def run(n):
        toks = rng.integers(0, cfg.total_tokens, n).astype(np.int32)
        heads = rng.integers(0, cfg.hq, n).astype(np.int32)
        pos = toks - starts[np.searchsorted(starts, toks, side="right") - 1]
        n_r = max(1, int(round(n * share)))
        pick = rng.integers(0, len(obs), n_r)
        rt = np.array([obs[i][0] for i in pick], np.int32)
        rp = np.array([obs[i][1] for i in pick], np.int64)
        rh = rng.integers(0, cfg.hq, n_r).astype(np.int32)
        t0 = time.perf_counter()
        oracle.attn(cu, q, k, v, tokens=toks, heads=heads, nthreads=cores)
        oracle.lazy_ratio_rows(cu, q, k, cfg.S, cfg.W, rt, rh, nthreads=cores)
        t = time.perf_counter() - t0
        fl = 4.0 * cfg.d * float(np.sum(pos + 1))
        fl += 2.0 * cfg.d * float(np.sum(np.minimum(cfg.S + cfg.W, rp + 1)))
        return fl, t, n, n_r

    fl, t, _, _ = run(64)
    n = int(min(200000, max(64, 64 * seconds / max(t, 1e-3))))
    fl, t, n, n_r = run(n)
    return fl / t / 1e12, cores, (f"{n} random (token, head) attention rows and {n_r} random observed (row, head) "
                                  f"lazy-ratio rows of layer 0 ({fl / 1e9:.1f} GFLOP, {t:.1f} s)")


def cpu_baseline(cfg, seconds=10.0):
    v, cores, desc = oracle_sample(cfg, seconds)
    return {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc}


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return None
    vals = []
    desc = ""
    oracle_sample(cfg, 0.1, seed=0)        # draws the inputs once, outside the timed steps
    for _ in range(args.warmup):
        oracle_sample(cfg, 1.0, seed=1)
    t0 = time.perf_counter()
    for s in range(args.steps):
        v, cores, desc = oracle_sample(cfg, 4.0, seed=100 + s)
        vals.append(v)
    ms = (time.perf_counter() - t0) * 1e3 / max(1, args.steps)
    value = statistics.mean(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, cfg.online if args.kv_pool == "auto" else args.kv_pool == "on", world,
                                  args.shard),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {desc}; the fp64 oracle on the host cores"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="long128k",
                    help="workload (synth.CONFIGS); long128k is the largest that one GPU holds")
    ap.add_argument("--kv-pool", default="auto", choices=["auto", "on", "off"],
                    help="keep the full KV of at most C+1 layers (auto: on for the online, memory-capped workload)")
    ap.add_argument("--layers", type=int, default=0,
                    help="a smaller case: only the workload's first N layers (budget scaled to N); for profiling")
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
    if args.layers:
        n = max(1, min(args.layers, cfg.layers))
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}-first{n}layers", layers=n,
                                  budget=int(round(cfg.budget * n / cfg.layers)))
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

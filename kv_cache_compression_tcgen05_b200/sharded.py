"""The prefill step over all layers, on one GPU or with the heads split over GPUs.

`PrefillStep` enqueues the whole LightTransfer-Test prefill path of one
prefill on a stream: per layer the causal GQA attention fused with the lazy
ratio (lt_prefill_attn_ratio, accumulate mode), the push of the layer's ratios
into the device-resident layer queue and the compaction of the layer the push
demotes (LightTransfer project page, Methodology, LightTransfer-Test; the
LightTransfer write-up, second solution).  No step waits for the host, so the
whole step can be captured in one CUDA graph.

Sequence sharding of a packed batch (sequence_shard, pack_sequences): each rank
takes whole sequences and runs its own PrefillStep on them; the sequences'
queues are independent, so nothing is exchanged.

Head sharding (one process per GPU; the pages describe a single GPU, both
splits are this library's reading): rank r of N holds KV heads [r Hkv/N, (r+1) Hkv/N)
and the query heads of their groups -- the contiguous slices a column-sharded
QKV projection produces -- and runs attention, the ratio and the compaction on
those heads alone.  The layer score is the mean of the ratios of all Hq query
heads, so the one exchange per layer is an all-gather of the per-head ratios
(batch * Hq * 4 bytes).  Every rank pushes the same gathered buffer into its
own device queue with lt_dqueue_push_gathered, which sums the heads in global
order: every rank demotes the same layers, bit for bit the ones a single GPU
holding all heads demotes, with no further exchange, and compacts its own
heads of each demoted layer.
"""
from __future__ import annotations

import torch

from . import binding as _b


def head_shard(hq: int, hkv: int, rank: int, world: int):
    """(q0, q1, kv0, kv1): the query and KV head ranges of `rank` out of `world`.
    KV head of query head h is h // (hq // hkv), so the query heads of KV heads
    [kv0, kv1) are [kv0 g, kv1 g)."""
    if hq < 1 or hkv < 1 or hq % hkv:
        raise ValueError("hq must be a positive multiple of hkv")
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if hkv % world:
        raise ValueError(f"{world} ranks cannot split {hkv} KV heads evenly")
    g, per = hq // hkv, hkv // world
    kv0 = rank * per
    return kv0 * g, (kv0 + per) * g, kv0, kv0 + per


def sequence_shard(seqlens, rank: int, world: int):
    """Sequences of `rank` when a packed batch is split over `world` ranks by
    whole sequences (independent prefills: no exchange, every rank keeps its own
    sequences' queues).  Sequences are dealt largest causal work N(N+1)/2 first,
    each to the rank with the least work so far (ties: lower sequence index,
    lower rank), so the slowest rank stays near 1/world of the batch's work.
    Returned in increasing order; the same on every rank."""
    seqlens = [int(n) for n in seqlens]
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if len(seqlens) < world:
        raise ValueError(f"{len(seqlens)} sequences cannot feed {world} ranks")
    load, owner = [0] * world, [0] * len(seqlens)
    for b in sorted(range(len(seqlens)), key=lambda b: (-seqlens[b] * (seqlens[b] + 1), b)):
        r = min(range(world), key=lambda r: (load[r], r))
        owner[b] = r
        load[r] += seqlens[b] * (seqlens[b] + 1) // 2
    return [b for b in range(len(seqlens)) if owner[b] == rank]


def pack_sequences(t: torch.Tensor, cu_seqlens, seqs):
    """Rows of the listed sequences of a packed [T, ...] tensor, packed in the
    listed order, and their cu_seqlens (a list, from 0)."""
    cu = [int(x) for x in cu_seqlens]
    parts, local_cu = [], [0]
    for b in seqs:
        parts.append(t[cu[b]:cu[b + 1]])
        local_cu.append(local_cu[-1] + cu[b + 1] - cu[b])
    return torch.cat(parts, dim=0).contiguous(), local_cu


def gather_ratios(ratio_local: torch.Tensor, gathered: torch.Tensor, group=None) -> None:
    """All-gather every rank's [batch, hq_shard] ratios into gathered
    [world, batch, hq_shard] (rank n's slice at index n), on the current stream."""
    world, batch, hq_s = gathered.shape
    if tuple(ratio_local.shape) != (batch, hq_s):
        raise ValueError("ratio_local must be [batch, hq_shard] of gathered [world, batch, hq_shard]")
    if not (ratio_local.is_contiguous() and gathered.is_contiguous()):
        raise ValueError("ratio_local and gathered must be contiguous")
    if world == 1 and not torch.distributed.is_initialized():
        gathered[0].copy_(ratio_local)
        return
    # [world * batch, hq_shard] is the memory of [world, batch, hq_shard].
    torch.distributed.all_gather_into_tensor(gathered.view(world * batch, hq_s), ratio_local, group=group)


def head_ratios(gathered: torch.Tensor) -> torch.Tensor:
    """[..., world, batch, hq_shard] gathered ratios as [..., batch, world * hq_shard]
    in global head order."""
    *lead, world, batch, hq_s = gathered.shape
    return gathered.movedim(-3, -2).reshape(*lead, batch, world * hq_s)


class PrefillStep:
    """Every layer of one prefill on this GPU's heads.

    layers: one (Q [T, hq, d], K [T, hkv, d], V [T, hkv, d]) bf16 device tuple
    per layer -- all heads, or this rank's head slice when `group` is a process
    group of several ranks.  The per-layer Q/K/V stay owned by the caller; the
    step owns O/LSE scratch, the per-layer ratios, the device queue and the
    streaming-KV pool [budget, batch, hkv, S+W, d] of the demoted layers (this
    rank's heads).  The step's buffers are created on the current stream: a
    step enqueued on another stream must be ordered after them and after the
    inputs (e.g. stream.wait_stream(torch.cuda.current_stream()))."""

    def __init__(self, layers, budget, S, W, n_obs, cu_seqlens=None, max_seqlen=None, group=None):
        if not layers:
            raise ValueError("at least one layer is required")
        if any(len(lay) != 3 for lay in layers):
            raise ValueError("every layer must be a (Q, K, V) triple")
        if cu_seqlens is not None and max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        Q0, K0, _ = layers[0]
        T, hq, d = Q0.shape
        hkv = K0.shape[1]
        for Q, K, V in layers:
            if Q.shape != Q0.shape or K.shape != K0.shape or V.shape != K0.shape:
                raise ValueError("every layer must have the same Q/K/V shapes")
        self.layers = list(layers)
        self.L, self.budget, self.S, self.W, self.n_obs = len(layers), int(budget), int(S), int(W), int(n_obs)
        self.T, self.hq, self.hkv, self.d = T, hq, hkv, d
        self.group = group
        self.world = torch.distributed.get_world_size(group) if group is not None else 1
        self.batch = cu_seqlens.numel() - 1 if cu_seqlens is not None else 1
        dev = Q0.device
        self.kw = dict(cu_seqlens=cu_seqlens, max_seqlen=max_seqlen if cu_seqlens is not None else None)
        self.O = torch.empty((T, hq, d), dtype=torch.bfloat16, device=dev)
        self.LSE = torch.empty((hq, T), dtype=torch.float32, device=dev)
        self.ratio = torch.zeros((self.L, self.batch, hq), dtype=torch.float32, device=dev)
        self.gathered = (torch.zeros((self.L, self.world, self.batch, hq), dtype=torch.float32, device=dev)
                         if group is not None else None)
        pool = (self.budget, self.batch, hkv, self.S + self.W, d)
        self.K_pool = torch.zeros(pool, dtype=torch.bfloat16, device=dev)
        self.V_pool = torch.zeros_like(self.K_pool)
        self.pool_len = torch.zeros((self.budget, self.batch), dtype=torch.int32, device=dev)
        self.Kp = _b.layer_pointer_table([lay[1] for lay in self.layers], device=dev)
        self.Vp = _b.layer_pointer_table([lay[2] for lay in self.layers], device=dev)
        self.dq = _b.DeviceQueue(self.L, self.budget, self.batch, device=dev)

    def layer(self, l, stream, O=None, LSE=None, events=None):
        """Attention + ratio, ratio exchange (sharded), queue push and compaction
        of layer l; O / LSE default to the step's own scratch."""
        Q, K, V = self.layers[l]
        if events is not None:
            e0 = torch.cuda.Event(enable_timing=True, external=True)
            e1 = torch.cuda.Event(enable_timing=True, external=True)
            e0.record(stream)
        _b.lt_prefill_attn_ratio(Q, K, V, self.S, self.W, self.n_obs, out=self.O if O is None else O,
                                 lse=self.LSE if LSE is None else LSE, ratio=self.ratio[l], stream=stream,
                                 accumulate=True, **self.kw)
        if events is not None:
            e1.record(stream)
            events.append((e0, e1))
        if self.gathered is None:
            _b.lt_dqueue_push(self.dq.state, self.L, self.batch, l, self.ratio[l], stream)
        else:
            with torch.cuda.stream(stream):
                gather_ratios(self.ratio[l], self.gathered[l], self.group)
            _b.lt_dqueue_push_gathered(self.dq.state, self.L, self.batch, l, self.gathered[l], stream)
        if self.budget > 0:   # with budget 0 no layer is ever demoted
            _b.lt_compact_kv_pending(self.Kp, self.Vp, self.dq, self.S, self.W, self.K_pool, self.V_pool,
                                     self.pool_len, self.T, self.hkv, self.d, stream=stream, **self.kw)

    def begin(self, stream):
        """Queue reset and all layers' ratio accumulators zeroed (once per step)."""
        _b.lt_dqueue_init(self.dq.state, self.L, self.budget, self.batch, stream)
        with torch.cuda.stream(stream):
            self.ratio.zero_()

    def enqueue(self, stream, events=None):
        """One whole step on `stream`; `events` collects a (start, end) pair of
        external timing events around every attention launch."""
        self.begin(stream)
        for l in range(self.L):
            self.layer(l, stream, events=events)

    def all_head_ratios(self) -> torch.Tensor:
        """[L, batch, Hq] ratios of all query heads (this rank's alone when not sharded)."""
        return self.ratio if self.gathered is None else head_ratios(self.gathered)

    def kernel_launches(self) -> int:
        """Library kernels one step launches: the queue reset, then attention,
        push and compaction per layer (the ratio zeroing and the all-gather
        are torch / NCCL work)."""
        return 1 + (3 if self.budget > 0 else 2) * self.L

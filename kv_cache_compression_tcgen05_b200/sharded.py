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
    group of several ranks.  The per-layer Q/K/V stay owned by the caller.

    Two ways to keep the KV cache (LightTransfer project page, Methodology,
    LightTransfer-Test, Figure 2 caption; the write-up's second solution):

    * kv_pool=False: every layer's full K/V stays in the caller's tensors; a
      demoted layer's streaming rows are gathered into the streaming pool
      (lt_compact_kv_pending) and the caller may release its full K/V.
    * kv_pool=True (the prefill under the peak-memory cap): the step owns a
      pool of C = L - budget full-KV slots [C, T, hkv, d].  A layer's K/V is
      read from the caller's tensors only while the layer runs; after its
      queue push, lt_kv_pool_commit reduces the demoted layer to its
      streaming rows and stores the current layer in the slot that freed (or
      a never-used one), unless the current layer was demoted itself.  At
      most C + 1 layers' full K/V then exist at any time: the C slots and the
      current layer's own buffer, so the caller can produce every layer's K/V
      into one working buffer.  An entry of `layers` may then be None, with
      the layer's tensors handed to layer(..., qkv=) and `dims` = (T, hq,
      hkv, d) giving the shapes.

    The step owns O/LSE scratch, the per-layer ratios, the device queue and
    the streaming-KV pool [budget, batch, hkv, S+W, d] of the demoted layers
    (this rank's heads).  A layer is three library launches (attention with
    the ratio, queue push, compaction or slot commit), or two with
    fused_push=True.  The step's buffers are created on the current stream: a step
    enqueued on another stream must be ordered after them and after the
    inputs (e.g. stream.wait_stream(torch.cuda.current_stream()))."""

    def __init__(self, layers, budget, S, W, n_obs, cu_seqlens=None, max_seqlen=None, group=None, kv_pool=False,
                 dims=None, fused_push=False):
        if not layers:
            raise ValueError("at least one layer is required")
        if any(lay is not None and len(lay) != 3 for lay in layers):
            raise ValueError("every layer must be a (Q, K, V) triple")
        if any(lay is None for lay in layers) and not kv_pool:
            raise ValueError("layers given later (None entries) need kv_pool=True")
        if cu_seqlens is not None and max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        known = [lay for lay in layers if lay is not None]
        if dims is None:
            if not known:
                raise ValueError("dims=(T, hq, hkv, d) is required when no layer's tensors are given")
            T, hq, d = known[0][0].shape
            hkv = known[0][1].shape[1]
        else:
            T, hq, hkv, d = (int(x) for x in dims)
        for Q, K, V in known:
            if tuple(Q.shape) != (T, hq, d) or tuple(K.shape) != (T, hkv, d) or V.shape != K.shape:
                raise ValueError("every layer must have the same Q/K/V shapes")
        if cu_seqlens is not None:
            # One host read at set-up: tiles past max_seqlen are never scheduled,
            # so a max_seqlen below the longest sequence would leave rows unwritten.
            cu = [int(x) for x in cu_seqlens.cpu()]
            lens = [b - a for a, b in zip(cu[:-1], cu[1:])]
            if cu[0] != 0 or cu[-1] != T or min(lens, default=0) < 0:
                raise ValueError("cu_seqlens must rise from 0 to the token count")
            if int(max_seqlen) < max(lens, default=0):
                raise ValueError(f"max_seqlen {max_seqlen} is below the longest sequence ({max(lens)})")
        self.layers = list(layers)
        self.L, self.budget, self.S, self.W, self.n_obs = len(layers), int(budget), int(S), int(W), int(n_obs)
        if not 0 <= self.budget <= self.L:
            raise ValueError("budget must lie in [0, L]")
        self.T, self.hq, self.hkv, self.d = T, hq, hkv, d
        self.group = group
        self.kv_pool = bool(kv_pool)
        # fused_push: the queue push rides on the attention kernel's last CTA
        # (lt_prefill_attn_ratio_push; two launches per layer) instead of its
        # own launch.  Off by default: measured on B200 the separate push,
        # launched programmatically behind the attention, costs less than the
        # completion count every CTA then takes (gqa1p2b step 1.88 against
        # 1.91 ms; equal at long128k).  With the heads split the push follows
        # the ratio exchange, so it is always separate.
        self.fused_push = bool(fused_push) and group is None
        self.world = torch.distributed.get_world_size(group) if group is not None else 1
        self.batch = cu_seqlens.numel() - 1 if cu_seqlens is not None else 1
        dev = known[0][0].device if known else torch.device("cuda", torch.cuda.current_device())
        self.device = dev
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
        if self.kv_pool:
            full = (self.L - self.budget, T, hkv, d)
            self.K_full = torch.empty(full, dtype=torch.bfloat16, device=dev)
            self.V_full = torch.empty_like(self.K_full)
            self.Kp = self.Vp = None
        else:
            self.K_full = self.V_full = None
            self.Kp = _b.layer_pointer_table([lay[1] for lay in self.layers], device=dev)
            self.Vp = _b.layer_pointer_table([lay[2] for lay in self.layers], device=dev)
        self.dq = _b.DeviceQueue(self.L, self.budget, self.batch, device=dev)

    def kv_bytes(self):
        """(full-KV bytes of one layer, streaming-KV bytes of one demoted layer,
        bytes the step holds for the KV cache: the full-KV slots, or none when
        the caller keeps every layer, plus the streaming pool)."""
        per_row = self.hkv * self.d * 2 * 2       # K and V, bf16
        full = self.T * per_row
        stream = self.batch * (self.S + self.W) * per_row
        held = self.budget * stream + ((self.L - self.budget) * full if self.kv_pool else 0)
        return full, stream, held

    def layer(self, l, stream, O=None, LSE=None, events=None, qkv=None):
        """Attention + ratio + queue push, ratio exchange (sharded), and the
        compaction / slot store of layer l; O / LSE default to the step's own
        scratch.  qkv: this layer's (Q, K, V), instead of the registered ones
        (kv_pool mode only)."""
        if qkv is not None and not self.kv_pool:
            raise ValueError("qkv= needs kv_pool=True (the registered K/V feed the compaction)")
        Q, K, V = qkv if qkv is not None else self.layers[l]
        out = self.O if O is None else O
        lse = self.LSE if LSE is None else LSE
        if events is not None:
            e0 = torch.cuda.Event(enable_timing=True, external=True)
            e1 = torch.cuda.Event(enable_timing=True, external=True)
            e0.record(stream)
        if self.fused_push:
            _b.lt_prefill_attn_ratio_push(Q, K, V, self.S, self.W, self.n_obs, self.dq, l, self.ratio[l], out=out,
                                          lse=lse, stream=stream, **self.kw)
        else:
            _b.lt_prefill_attn_ratio(Q, K, V, self.S, self.W, self.n_obs, out=out, lse=lse, ratio=self.ratio[l],
                                     stream=stream, accumulate=True, **self.kw)
        if events is not None:
            e1.record(stream)
            events.append((e0, e1))
        if self.gathered is not None:
            with torch.cuda.stream(stream):
                gather_ratios(self.ratio[l], self.gathered[l], self.group)
            _b.lt_dqueue_push_gathered(self.dq.state, self.L, self.batch, l, self.gathered[l], stream)
        elif not self.fused_push:
            _b.lt_dqueue_push(self.dq.state, self.L, self.batch, l, self.ratio[l], stream)
        if self.kv_pool:
            _b.lt_kv_pool_commit(K, V, self.dq, l, self.S, self.W, self.K_full, self.V_full, self.K_pool,
                                 self.V_pool, self.pool_len, stream=stream, **self.kw)
        elif self.budget > 0:   # with budget 0 no layer is ever demoted
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

    def kept_layer_cache(self, l, slots=None):
        """Full K/V of a layer the queue kept, for lt_decode_attn: (K, V,
        seq_start) with sequence b's rows starting at row seq_start[b].  In
        kv_pool mode K/V are the slot pool viewed as [(L - budget) T, hkv, d]
        and seq_start = slot * T + cu_seqlens[b] (slots: the queue's slot
        table, read here when not given); otherwise the layer's own tensors."""
        cu = self.kw["cu_seqlens"]
        starts = (cu[:-1] if cu is not None else torch.zeros(1, dtype=torch.int32, device=self.device))
        if not self.kv_pool:
            _, K, V = self.layers[l]
            return K, V, starts.to(torch.int32).contiguous()
        slots = self.dq.slots() if slots is None else slots
        s = slots[:, l].to(torch.int64)
        if bool((s < 0).any()):
            raise ValueError(f"layer {l} holds no full-KV slot (demoted, or not pushed) in some sequence")
        rows = (self.L - self.budget) * self.T
        seq_start = (s * self.T + starts.to(torch.int64)).to(torch.int32).contiguous()
        return (self.K_full.view(rows, self.hkv, self.d), self.V_full.view(rows, self.hkv, self.d), seq_start)

    def kernel_launches(self) -> int:
        """Library kernels one step launches: the queue reset, then per layer
        the attention (with the queue push when not sharded), the push (when
        sharded) and the compaction or the slot commit (the ratio zeroing and
        the all-gather are torch / NCCL work)."""
        per_layer = 1 + (0 if self.fused_push else 1) + (1 if self.kv_pool or self.budget > 0 else 0)
        return 1 + per_layer * self.L

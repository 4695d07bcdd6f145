"""Sharding on the CPU.  Heads: the head ranges, the global head order of
gathered ratios, and two gloo ranks that each compute their own heads' lazy
ratios (with the oracle), all-gather them with the library's gather_ratios and
run the library's host queue on the gathered scores; both ranks must demote the
same layers as one process holding all heads, with bit-identical layer scores.
Sequences: every sequence dealt to one rank, the slowest rank's work within the
greedy bound, and packing of a rank's sequences.  Failure: a rank that leaves
before a layer's exchange makes the other rank's exchange fail with an error
within the process group's timeout instead of hanging."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import kv_cache_compression_tcgen05_b200 as lt


@pytest.mark.parametrize("hq,hkv,world", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8), (40, 8, 4), (4, 4, 2),
                                          (8, 2, 2)])
def test_head_shard_covers_every_head_once(hq, hkv, world):
    g = hq // hkv
    q_seen, kv_seen = [], []
    for r in range(world):
        q0, q1, k0, k1 = lt.head_shard(hq, hkv, r, world)
        assert q1 - q0 == hq // world and k1 - k0 == hkv // world
        # every query head of the slice maps (h // g) to a KV head of the same slice
        assert all(k0 <= h // g < k1 for h in range(q0, q1))
        q_seen += range(q0, q1)
        kv_seen += range(k0, k1)
    assert q_seen == list(range(hq)) and kv_seen == list(range(hkv))


def test_head_shard_rejects_bad_splits():
    with pytest.raises(ValueError):
        lt.head_shard(32, 8, 0, 3)        # 8 KV heads over 3 ranks
    with pytest.raises(ValueError):
        lt.head_shard(30, 8, 0, 2)        # hq not a multiple of hkv
    with pytest.raises(ValueError):
        lt.head_shard(32, 8, 2, 2)        # rank out of range


def test_head_ratios_restores_global_head_order():
    L, B, H, world = 3, 2, 8, 4
    full = torch.arange(L * B * H, dtype=torch.float32).reshape(L, B, H)
    hs = H // world
    gathered = torch.stack([full[:, :, r * hs:(r + 1) * hs] for r in range(world)], dim=1)   # [L, world, B, hs]
    assert torch.equal(lt.head_ratios(gathered), full)
    assert torch.equal(lt.head_ratios(gathered[1]), full[1])


def test_gather_ratios_single_process_copies():
    ratio = torch.rand(2, 5)
    gathered = torch.zeros(1, 2, 5)
    lt.gather_ratios(ratio, gathered)
    assert torch.equal(gathered[0], ratio)
    with pytest.raises(ValueError):
        lt.gather_ratios(torch.rand(2, 4), gathered)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _config():
    import synth
    # 4 KV heads so that two ranks hold 2 each; sink-biased layers 1, 3, 4
    return synth.custom(name="shard", layers=6, seqlens=(192,), hq=8, hkv=4, d=64, S=4, W=16, n_obs=16, budget=3,
                        seed=11, lazy_layers=(1, 3, 4))


def _ratios(cfg, layer, q0, q1, k0, k1):
    import oracle
    import synth
    Q, K, _ = synth.layer_inputs(cfg, layer)
    Q, K = Q[:, q0:q1].contiguous(), K[:, k0:k1].contiguous()
    cu = np.array(cfg.cu_seqlens(), np.int32)
    r = oracle.lazy_ratio(cu, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, cfg.n_obs, nthreads=1)
    return r.astype(np.float32)      # [batch, heads of the slice], as the kernel stores it


def _demotions(cfg, head_ratio_of_layer):
    q = lt.LayerQueue(cfg.layers, cfg.budget)
    order, scores = [], []
    for layer in range(cfg.layers):
        s = lt.lt_layer_score(np.ascontiguousarray(head_ratio_of_layer(layer)[0]))
        scores.append(s)
        d = q.push(layer, s)
        if d >= 0:
            order.append(d)
    q.close()
    return order, scores


def _rank_main(rank, world, port, out):
    import datetime

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = _config()
        q0, q1, k0, k1 = lt.head_shard(cfg.hq, cfg.hkv, rank, world)
        gathered = torch.zeros((cfg.layers, world, cfg.batch, q1 - q0))
        for layer in range(cfg.layers):
            local = torch.from_numpy(_ratios(cfg, layer, q0, q1, k0, k1))
            lt.gather_ratios(local, gathered[layer])
        heads = lt.head_ratios(gathered).numpy()
        out[rank] = _demotions(cfg, lambda layer: heads[layer])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_demote_as_one_process():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    cfg = _config()
    single = _demotions(cfg, lambda layer: _ratios(cfg, layer, 0, cfg.hq, 0, cfg.hkv))
    assert len(single[0]) == cfg.budget
    assert out[0] == out[1] == single     # same demotion order and bit-identical scores


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_sequence_shard_deals_every_sequence_once_and_balances(world):
    import synth
    seqlens = synth.CONFIGS["batched"].seqlens
    parts = [lt.sequence_shard(seqlens, r, world) for r in range(world)]
    assert sorted(b for p in parts for b in p) == list(range(len(seqlens)))
    assert all(p == sorted(p) and p for p in parts)
    work = [n * (n + 1) // 2 for n in seqlens]
    loads = [sum(work[b] for b in p) for p in parts]
    # greedy largest-first bound: the slowest rank exceeds the mean by at most one sequence's work
    assert max(loads) <= sum(work) / world + max(work)
    assert parts == [lt.sequence_shard(list(seqlens), r, world) for r in range(world)]   # deterministic


def test_sequence_shard_examples_and_errors():
    # works 55, 820, 210, 465: 40 -> r0 (820); 30 -> r1 (465); 20 -> r1 (675); 10 -> r1 (730)
    assert lt.sequence_shard([10, 40, 20, 30], 0, 2) == [1]
    assert lt.sequence_shard([10, 40, 20, 30], 1, 2) == [0, 2, 3]
    assert lt.sequence_shard([5, 5, 5], 2, 3) == [2]
    with pytest.raises(ValueError):
        lt.sequence_shard([5, 5], 0, 3)
    with pytest.raises(ValueError):
        lt.sequence_shard([5, 5], 2, 2)


def test_pack_sequences_keeps_rows_and_lengths():
    cu = [0, 3, 7, 12]
    t = torch.arange(12 * 2).reshape(12, 2)
    packed, local_cu = lt.pack_sequences(t, cu, [2, 0])
    assert local_cu == [0, 5, 8]
    assert torch.equal(packed, torch.cat([t[7:12], t[0:3]]))


def test_prefill_step_rejects_bad_layer_lists_before_allocating():
    Q = torch.zeros((8, 4, 64), dtype=torch.bfloat16)
    K = torch.zeros((8, 2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        lt.PrefillStep([], 1, 4, 8, 4)
    with pytest.raises(ValueError):
        lt.PrefillStep([(Q, K)], 1, 4, 8, 4)
    with pytest.raises(ValueError):
        lt.PrefillStep([(Q, K, K), (Q, K, K[:4])], 1, 4, 8, 4)
    with pytest.raises(ValueError):
        lt.PrefillStep([(Q, K, K)], 1, 4, 8, 4, cu_seqlens=torch.tensor([0, 3, 8], dtype=torch.int32))


def _rank_dies_main(rank, world, port, out):
    import datetime
    import time

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(0)                       # leaves between steps, before the layer's exchange
    gathered = torch.zeros((world, 1, 2))
    t0 = time.monotonic()
    try:
        lt.gather_ratios(torch.ones((1, 2)), gathered)
        out[rank] = ("no error", time.monotonic() - t0)
    except RuntimeError as e:             # the exchange reports the missing rank
        out[rank] = (type(e).__name__, time.monotonic() - t0)


def test_exchange_fails_instead_of_hanging_when_a_rank_leaves():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=60)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank hung on the exchange"
    kind, seconds = out[0]
    assert kind == "RuntimeError" and seconds < 30

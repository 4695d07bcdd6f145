"""The multi-process path of bench.py on CPU: two gloo ranks, each an
independent replica of the tiny workload (synthetic inputs, oracle ratios, the
library's host queue).  Checks the max-over-ranks timing reduction and that the
replicas agree (the path has no exchange step, so replicas must not depend on
the rank)."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import kv_cache_compression_tcgen05_b200 as lt
        import oracle
        import synth

        cfg = synth.CONFIGS["tiny"]
        cu = np.array(cfg.cu_seqlens(), np.int32)
        q = lt.LayerQueue(cfg.layers, cfg.budget)
        demoted = []
        for layer in range(cfg.layers):
            Q, K, _ = synth.layer_inputs(cfg, layer)
            r = oracle.lazy_ratio(cu, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, cfg.n_obs, nthreads=1)
            d = q.push(layer, lt.lt_layer_score(r[0].astype(np.float32)))
            if d >= 0:
                demoted.append(d)
        q.close()
        slowest = bench.max_over_ranks(1.0 + rank, world, device="cpu")
        bench.barrier(world)
        out[rank] = (sorted(demoted), slowest)
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == [1, 3]
    assert out[0][1] == out[1][1] == 2.0

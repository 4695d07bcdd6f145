"""The package's prefill step (PrefillStep) and its head-split path, on one GPU.

- lt_dqueue_push_gathered on ratios laid out [shards, batch, hq_shard] makes
  exactly the pushes lt_dqueue_push makes on the same ratios as [batch, hq];
- PrefillStep over all heads matches the oracle (ratios, demotions, streaming
  KV);
- head slices run one after another on one GPU (no collective: the gathered
  buffer is assembled by the test), each pushing the gathered ratios of all
  slices into its own queue, demote the layers the all-heads step demotes and
  compact exactly their own heads of them, with bit-identical O and LSE;
- the step with a one-rank NCCL process group (so the ratios take the
  collective path) captured in a CUDA graph agrees with the step without one;
- ranks that take whole sequences of a packed batch reproduce the batch's rows.
"""
import socket

import numpy as np
import pytest
import torch

import kv_cache_compression_tcgen05_b200 as lt
import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lt.library()
    yield
    assert lt.lt_device_status(True) == lt.LT_OK


def _cfg():
    # 600 tokens: several 128-row tiles and a ragged tail; sink-biased layers 1, 3, 4
    return synth.custom(name="shard", layers=6, seqlens=(600,), hq=8, hkv=4, d=64, S=4, W=64, n_obs=32, budget=3,
                        seed=11, lazy_layers=(1, 3, 4))


def _layers(cfg, q0=0, q1=None, k0=0, k1=None):
    out = []
    for l in range(cfg.layers):
        Q, K, V = synth.layer_inputs(cfg, l, "cuda")
        out.append((Q[:, q0:q1].contiguous(), K[:, k0:k1].contiguous(), V[:, k0:k1].contiguous()))
    return out


def _step(cfg, layers, group=None):
    return lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, group=group)


def _run(step):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())     # inputs and the step's buffers were made there
    step.enqueue(s)
    torch.cuda.synchronize()
    assert step.dq.error() == 0
    _, order = step.dq.result()
    torch.cuda.synchronize()
    return order


@pytest.mark.parametrize("shards", [1, 2, 4, 8])
def test_push_gathered_equals_push(shards):
    L, B, H, budget = 8, 3, 32, 4
    g = torch.Generator(device="cuda").manual_seed(shards)
    ratios = torch.rand((L, B, H), generator=g, device="cuda")
    ratios[5] = ratios[2]                                   # tied layer scores
    hs = H // shards
    gathered = ratios.view(L, B, shards, hs).permute(0, 2, 1, 3).contiguous()   # [L, shards, B, hs]
    a, b = lt.DeviceQueue(L, budget, B), lt.DeviceQueue(L, budget, B)
    for l in range(L):
        a.push(l, ratios[l])
        b.push_gathered(l, gathered[l])
    ma, oa = a.result()
    mb, ob = b.result()
    torch.cuda.synchronize()
    assert a.error() == 0 and b.error() == 0
    assert torch.equal(oa, ob) and torch.equal(ma, mb)


def test_prefill_step_matches_oracle():
    cfg = _cfg()
    layers = _layers(cfg)
    step = _step(cfg, layers)
    order = _run(step)[0].tolist()
    cu = np.array(cfg.cu_seqlens(), np.int32)
    ref = [oracle.lazy_ratio(cu, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, cfg.n_obs)
           for Q, K, _ in layers]
    assert np.abs(step.ratio.cpu().numpy() - np.stack(ref)).max() <= 2e-3
    scores = np.array([r[0].mean() for r in ref])
    assert order == oracle.queue_online(scores, cfg.budget).tolist()
    assert sorted(order) == [1, 3, 4]
    for k, m in enumerate(order):
        oks, ovs, oln = oracle.compact_kv(cu, synth.bf16_bits(layers[m][1]), synth.bf16_bits(layers[m][2]),
                                          np.ones(1, np.uint8), cfg.S, cfg.W)
        assert np.array_equal(synth.bf16_bits(step.K_pool[k, 0]), oks[0])
        assert np.array_equal(synth.bf16_bits(step.V_pool[k, 0]), ovs[0])
        assert int(step.pool_len[k, 0]) == int(oln[0])


@pytest.mark.parametrize("world", [2, 4])
def test_head_slices_on_one_gpu_match_all_heads(world):
    cfg = _cfg()
    full = _step(cfg, _layers(cfg))
    order_full = _run(full)
    shards = [lt.head_shard(cfg.hq, cfg.hkv, r, world) for r in range(world)]
    steps = [_step(cfg, _layers(cfg, *sh)) for sh in shards]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    for st in steps:                        # each slice's attention + ratios (its own queue is not used)
        st.enqueue(s)
    torch.cuda.synchronize()
    gathered = torch.stack([st.ratio for st in steps], dim=1).contiguous()    # [L, world, B, hq_shard]
    assert torch.equal(lt.head_ratios(gathered), full.ratio)
    for (q0, q1, k0, k1), st in zip(shards, steps):
        assert torch.equal(st.O, full.O[:, q0:q1]) and torch.equal(st.LSE, full.LSE[q0:q1])   # the last layer's
        # the slice's queue fed every slice's ratios, as after an all-gather
        with torch.cuda.stream(s):
            st.K_pool.zero_()
            st.V_pool.zero_()
        lt.lt_dqueue_init(st.dq.state, st.L, st.budget, st.batch, s)
        for l in range(st.L):
            lt.lt_dqueue_push_gathered(st.dq.state, st.L, st.batch, l, gathered[l], s)
            lt.lt_compact_kv_pending(st.Kp, st.Vp, st.dq, st.S, st.W, st.K_pool, st.V_pool, st.pool_len, st.T,
                                     st.hkv, st.d, stream=s)
        torch.cuda.synchronize()
        _, order = st.dq.result()
        torch.cuda.synchronize()
        assert torch.equal(order, order_full)
        assert torch.equal(st.K_pool, full.K_pool[:, :, k0:k1]) and torch.equal(st.V_pool, full.V_pool[:, :, k0:k1])
        assert torch.equal(st.pool_len, full.pool_len)


def _free_port():
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


def test_step_with_single_rank_group_in_a_graph():
    cfg = _cfg()
    layers = _layers(cfg)
    plain = _step(cfg, layers)
    order_plain = _run(plain)
    dist = torch.distributed
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    graph = None
    try:
        step = _step(cfg, layers, group=dist.group.WORLD)
        assert step.gathered is not None
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step.enqueue(s)                 # eager: communicator set-up outside capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            step.enqueue(s)
        step.K_pool.zero_()
        step.ratio.fill_(-1.0)
        step.gathered.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert step.dq.error() == 0
        _, order = step.dq.result()
        torch.cuda.synchronize()
        assert torch.equal(order, order_plain)
        assert torch.equal(step.gathered[:, 0], plain.ratio) and torch.equal(step.ratio, plain.ratio)
        assert torch.equal(step.K_pool, plain.K_pool) and torch.equal(step.V_pool, plain.V_pool)
    finally:
        graph = None                        # a graph holding NCCL calls goes before the process group
        torch.cuda.synchronize()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_slices_match_full_batch(world):
    """Ranks that take whole sequences of a packed batch (run one after another
    here) reproduce the full batch's rows: bit-identical O, LSE, demotions and
    streaming KV per sequence; the ratios agree to float-atomic order (the
    observed rows of a sequence can span two query tiles)."""
    cfg = synth.custom(name="seqs", layers=5, seqlens=(300, 77, 520, 190), hq=4, hkv=2, d=64, S=4, W=48, n_obs=24,
                       budget=2, seed=13, lazy_layers=(1, 3))
    layers = _layers(cfg)
    cu_h = cfg.cu_seqlens()
    full = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs,
                          cu_seqlens=torch.tensor(cu_h, dtype=torch.int32, device="cuda"), max_seqlen=cfg.max_seqlen)
    order_full = _run(full)
    for r in range(world):
        seqs = lt.sequence_shard(cfg.seqlens, r, world)
        packed = [tuple(lt.pack_sequences(t, cu_h, seqs)[0] for t in lay) for lay in layers]
        local_cu = lt.pack_sequences(layers[0][0], cu_h, seqs)[1]
        cu = torch.tensor(local_cu, dtype=torch.int32, device="cuda") if len(seqs) > 1 else None
        st = lt.PrefillStep(packed, cfg.budget, cfg.S, cfg.W, cfg.n_obs, cu_seqlens=cu,
                            max_seqlen=max(cfg.seqlens[b] for b in seqs))
        order = _run(st)
        for i, b in enumerate(seqs):
            assert torch.equal(order[i], order_full[b])
            assert torch.allclose(st.ratio[:, i], full.ratio[:, b], rtol=0, atol=1e-6)
            assert torch.equal(st.K_pool[:, i], full.K_pool[:, b]) and torch.equal(st.V_pool[:, i], full.V_pool[:, b])
            assert torch.equal(st.pool_len[:, i], full.pool_len[:, b])
            l0, l1, g0, g1 = local_cu[i], local_cu[i + 1], cu_h[b], cu_h[b + 1]
            assert torch.equal(st.O[l0:l1], full.O[g0:g1]) and torch.equal(st.LSE[:, l0:l1], full.LSE[:, g0:g1])


def test_prefill_step_with_budget_zero_demotes_nothing():
    cfg = _cfg()
    step = lt.PrefillStep(_layers(cfg), 0, cfg.S, cfg.W, cfg.n_obs)
    assert step.kernel_launches() == 1 + 2 * cfg.layers      # attention and push; no compaction launches
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    step.enqueue(s)
    torch.cuda.synchronize()
    mask, order = step.dq.result()
    torch.cuda.synchronize()
    assert step.dq.error() == 0 and order.shape == (1, 0) and not bool(mask.any())
    assert step.K_pool.numel() == 0

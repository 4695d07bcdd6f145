"""Device-resident layer queue and the compaction it drives, against the host
queue and the fp64 oracle; and a whole tiny prefill captured in a CUDA graph."""
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


def _host_pops(ratios, budget, push_order):
    """Host queue pops of each sequence; ratios [L, B, H] float32 (numpy)."""
    L, B, H = ratios.shape
    out = []
    for b in range(B):
        q = lt.LayerQueue(L, budget)
        pops = [d for d in (q.push(l, lt.lt_layer_score(ratios[l, b])) for l in push_order) if d >= 0]
        q.close()
        out.append(pops)
    return out


@pytest.mark.parametrize("L,B,H,budget", [(16, 5, 8, 8), (4, 1, 2, 2), (64, 3, 40, 32), (7, 2, 3, 0), (5, 4, 4, 5)])
def test_device_queue_matches_host_and_oracle(L, B, H, budget):
    rng = np.random.default_rng(L * 100 + B)
    ratios = rng.random((L, B, H)).astype(np.float32)
    ratios[2 % L, :, :] = ratios[1 % L, :, :]           # tied layer scores
    for push_order in (list(range(L)), list(rng.permutation(L))):
        dq = lt.DeviceQueue(L, budget, B)
        r_dev = torch.tensor(ratios, device="cuda")
        for l in push_order:
            dq.push(l, r_dev[l])
        mask, order = dq.result()
        torch.cuda.synchronize()
        assert dq.error() == 0
        host = _host_pops(ratios, budget, push_order)
        for b in range(B):
            assert order[b].tolist() == host[b], (b, order[b].tolist(), host[b])
            scores = np.array([lt.lt_layer_score(ratios[l, b]) for l in range(L)], np.float64)
            o_lazy, _ = oracle.select_layers(scores, budget)
            assert np.array_equal(mask[b].cpu().numpy(), o_lazy)


def test_device_queue_flags_bad_pushes():
    L, B, H = 6, 2, 4
    ratios = torch.rand((L, B, H), device="cuda")
    dq = lt.DeviceQueue(L, 3, B)
    dq.push(0, ratios[0])
    dq.push(0, ratios[0])            # twice
    torch.cuda.synchronize()
    assert dq.error() & 1
    dq.reset()
    dq.push(7, ratios[0])            # out of range
    torch.cuda.synchronize()
    assert dq.error() & 1
    dq.reset()
    bad = ratios[1].clone()
    bad[1, 0] = float("nan")         # sequence 1 gets a non-finite score
    dq.push(1, bad)
    torch.cuda.synchronize()
    assert dq.error() & 1
    for l in (0, 2, 3, 4, 5):
        dq.push(l, ratios[l])
    mask, _ = dq.result()
    torch.cuda.synchronize()
    # sequence 0 saw all six layers and demoted 3; sequence 1 missed layer 1.
    assert int(mask[0].sum()) == 3 and int(mask[1, 1]) == 0


def test_compact_pending_matches_oracle():
    spec = dict(seqlens=(300, 41, 1000, 7), hq=4, hkv=2, d=64, S=4, W=60)
    cfg = synth.custom(layers=6, seqlens=spec["seqlens"], hq=spec["hq"], hkv=spec["hkv"], d=spec["d"], S=spec["S"],
                       W=spec["W"], seed=71)
    L, B, budget = cfg.layers, cfg.batch, 3
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(L)]
    Kp = lt.layer_pointer_table([lay[1] for lay in layers])
    Vp = lt.layer_pointer_table([lay[2] for lay in layers])
    slots = cfg.S + cfg.W
    K_pool = torch.full((budget, B, cfg.hkv, slots, cfg.d), -3.0, dtype=torch.bfloat16, device="cuda")
    V_pool = K_pool.clone()
    pool_len = torch.full((budget, B), -1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(5)
    ratios = rng.random((L, B, cfg.hq)).astype(np.float32)
    r_dev = torch.tensor(ratios, device="cuda")
    cu = torch.tensor(cfg.cu_seqlens(), dtype=torch.int32, device="cuda")
    dq = lt.DeviceQueue(L, budget, B)
    for l in range(L):
        dq.push(l, r_dev[l])
        lt.lt_compact_kv_pending(Kp, Vp, dq, cfg.S, cfg.W, K_pool, V_pool, pool_len, cfg.total_tokens, cfg.hkv, cfg.d,
                                 cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    _, order = dq.result()
    torch.cuda.synchronize()
    host = _host_pops(ratios, budget, range(L))
    cu_h = np.array(cfg.cu_seqlens(), np.int32)
    for b in range(B):
        assert order[b].tolist() == host[b]
        for k, m in enumerate(host[b]):
            mask = np.zeros(B, np.uint8)
            mask[b] = 1
            oks, ovs, oln = oracle.compact_kv(cu_h, synth.bf16_bits(layers[m][1]), synth.bf16_bits(layers[m][2]), mask,
                                              cfg.S, cfg.W)
            assert np.array_equal(synth.bf16_bits(K_pool[k, b]), oks[b])
            assert np.array_equal(synth.bf16_bits(V_pool[k, b]), ovs[b])
            assert int(pool_len[k, b]) == int(oln[b])


def test_graph_captured_tiny_prefill():
    """The whole tiny prefill (fused attention + ratio, device queue, device-
    driven compaction for every layer) captured once in a CUDA graph and
    replayed: demotes the designed layers {1, 3} with their streaming KV."""
    cfg = synth.CONFIGS["tiny"]
    L = cfg.layers
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(L)]
    Kp = lt.layer_pointer_table([lay[1] for lay in layers])
    Vp = lt.layer_pointer_table([lay[2] for lay in layers])
    T, H, d = cfg.total_tokens, cfg.hq, cfg.d
    O = torch.empty((T, H, d), dtype=torch.bfloat16, device="cuda")
    LSE = torch.empty((H, T), dtype=torch.float32, device="cuda")
    ratio = torch.empty((L, 1, H), dtype=torch.float32, device="cuda")
    slots = cfg.S + cfg.W
    K_pool = torch.zeros((cfg.budget, 1, cfg.hkv, slots, d), dtype=torch.bfloat16, device="cuda")
    V_pool = torch.zeros_like(K_pool)
    pool_len = torch.zeros((cfg.budget, 1), dtype=torch.int32, device="cuda")
    dq = lt.DeviceQueue(L, cfg.budget, 1)

    def prefill(stream):
        lt.lt_dqueue_init(dq.state, L, cfg.budget, 1, stream)
        for l in range(L):
            Q, K, V = layers[l]
            lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, out=O, lse=LSE, ratio=ratio[l], stream=stream)
            lt.lt_dqueue_push(dq.state, L, 1, l, ratio[l], stream)
            lt.lt_compact_kv_pending(Kp, Vp, dq, cfg.S, cfg.W, K_pool, V_pool, pool_len, T, cfg.hkv, d, stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())   # the inputs were made on the default stream
    with torch.cuda.stream(s):
        prefill(s)            # warm-up outside capture (first calls set up per-device state)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        prefill(s)
    K_pool.zero_()
    V_pool.zero_()
    g.replay()
    torch.cuda.synchronize()
    mask, order = dq.result()
    torch.cuda.synchronize()
    assert order[0].tolist() == [1, 3] or sorted(order[0].tolist()) == [1, 3]
    cu_h = np.array(cfg.cu_seqlens(), np.int32)
    for k, m in enumerate(order[0].tolist()):
        oks, ovs, oln = oracle.compact_kv(cu_h, synth.bf16_bits(layers[m][1]), synth.bf16_bits(layers[m][2]),
                                          np.ones(1, np.uint8), cfg.S, cfg.W)
        assert np.array_equal(synth.bf16_bits(K_pool[k, 0]), oks[0])
        assert np.array_equal(synth.bf16_bits(V_pool[k, 0]), ovs[0])
    # The ratios computed inside the graph match the oracle.
    for l in range(L):
        Q, K, _ = layers[l]
        ref = oracle.lazy_ratio(cu_h, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, cfg.n_obs)
        assert np.abs(ratio[l].cpu().numpy() - ref).max() <= 2e-3


def test_compact_kv_layers_matches_oracle():
    """Several layers compacted in one launch equal the oracle's per-layer
    compaction; a slot whose layer index is -1 is left untouched."""
    cfg = synth.custom(layers=5, seqlens=(300, 41, 1000, 7), hq=4, hkv=2, d=128, S=4, W=60, seed=37)
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(cfg.layers)]
    Kp = lt.layer_pointer_table([lay[1] for lay in layers])
    Vp = lt.layer_pointer_table([lay[2] for lay in layers])
    pick = [3, -1, 0, 4]
    slots = cfg.S + cfg.W
    K_pool = torch.full((len(pick), cfg.batch, cfg.hkv, slots, cfg.d), -5.0, dtype=torch.bfloat16, device="cuda")
    V_pool = K_pool.clone()
    pool_len = torch.full((len(pick), cfg.batch), -7, dtype=torch.int32, device="cuda")
    cu = torch.tensor(cfg.cu_seqlens(), dtype=torch.int32, device="cuda")
    lt.lt_compact_kv_layers(Kp, Vp, torch.tensor(pick, dtype=torch.int32, device="cuda"), cfg.S, cfg.W, K_pool, V_pool,
                            pool_len, cfg.total_tokens, cfg.hkv, cfg.d, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    torch.cuda.synchronize()
    cu_h = np.array(cfg.cu_seqlens(), np.int32)
    ones = np.ones(cfg.batch, np.uint8)
    for k, m in enumerate(pick):
        if m < 0:
            assert bool((K_pool[k] == -5.0).all()) and bool((pool_len[k] == -7).all())
            continue
        oks, ovs, oln = oracle.compact_kv(cu_h, synth.bf16_bits(layers[m][1]), synth.bf16_bits(layers[m][2]), ones,
                                          cfg.S, cfg.W)
        assert np.array_equal(synth.bf16_bits(K_pool[k]), oks)
        assert np.array_equal(synth.bf16_bits(V_pool[k]), ovs)
        assert np.array_equal(pool_len[k].cpu().numpy(), oln)

"""The prefill under the peak-memory cap (PrefillStep(kv_pool=True)) and the
queue push fused into the attention kernel, on one GPU, through the C ABI.

LightTransfer project page (Methodology, LightTransfer-Test, Figure 2
caption): once the queue is full the layer with the highest ratio is made
lazy and its KV cache reduced, "freeing memory for storing the KV cache of the
current layer"; the write-up's second solution: the prefill's peak memory stays
at most 50% full KV + 50% streaming KV.  Checked here:

- lt_prefill_attn_ratio_push leaves the queue exactly as the separate push
  does (demotions, slots), with the same ratios, O and LSE, also with no tokens;
- the pool step demotes the oracle's layers (online queue on the oracle's
  ratios), its streaming KV equals the oracle's compaction bit for bit, and
  every kept layer's full K/V sits in its slot bit for bit;
- with each layer's Q/K/V produced just before its turn and released after
  it, the allocator's high-water mark over the whole prefill is the step's own
  buffers plus one layer's inputs: the C full-KV slots and the working layer
  (C + 1 full layers) plus the streaming caches, against L full layers;
- per-sequence slots of a packed batch, budget 0 and budget L, decode over a
  kept layer's slot, and the pool step replayed from a CUDA graph.
"""
import numpy as np
import pytest
import torch

import kv_cache_compression_tcgen05_b200 as lt
import oracle
import synth
from tests.gpu_common import RATIO_ABS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lt.library()
    yield
    assert lt.lt_device_status(True) == lt.LT_OK


def _cu(cfg):
    return torch.tensor(cfg.cu_seqlens(), dtype=torch.int32, device="cuda") if cfg.batch > 1 else None


def _kw(cfg):
    cu = _cu(cfg)
    return dict(cu_seqlens=cu, max_seqlen=cfg.max_seqlen if cu is not None else None)


def _run(step, qkv=None):
    s = torch.cuda.current_stream()
    step.begin(s)
    for l in range(step.L):
        step.layer(l, s, qkv=None if qkv is None else qkv(l))
    torch.cuda.synchronize()
    assert step.dq.error() == 0
    mask, order = step.dq.result()
    torch.cuda.synchronize()
    return mask, order


def _oracle_orders(cfg, host_layers):
    """Demotion order of every sequence from the oracle's ratios (online queue)."""
    cu = np.array(cfg.cu_seqlens(), np.int32)
    ratios = np.stack([oracle.lazy_ratio(cu, q, k, cfg.S, cfg.W, cfg.n_obs) for q, k, _ in host_layers])
    scores = oracle.layer_scores(ratios)                     # [batch, L]
    return ratios, scores, [oracle.queue_online(scores[b], cfg.budget).tolist() for b in range(cfg.batch)]


def _check_against_oracle(cfg, step, order, host_layers):
    """Ratios, demotions (ties within the ratio bar may swap), streaming KV and
    the kept layers' slots against the oracle and the inputs."""
    ratios, scores, want = _oracle_orders(cfg, host_layers)
    assert np.abs(step.ratio.cpu().numpy() - ratios).max() <= RATIO_ABS
    cu = np.array(cfg.cu_seqlens(), np.int32)
    slots = step.dq.slots().cpu().numpy()
    order = order.cpu().numpy()
    for b in range(cfg.batch):
        got = [int(x) for x in order[b] if x >= 0]
        if got != want[b]:
            # only layers whose oracle scores tie within the bar may trade places
            for x, y in zip(got, want[b]):
                assert x == y or abs(scores[b, x] - scores[b, y]) <= 2 * RATIO_ABS, (got, want[b])
        for k, m in enumerate(got):
            mask = np.zeros(cfg.batch, np.uint8)
            mask[b] = 1
            oks, ovs, oln = oracle.compact_kv(cu, host_layers[m][1], host_layers[m][2], mask, cfg.S, cfg.W)
            assert np.array_equal(synth.bf16_bits(step.K_pool[k, b]), oks[b]), (b, k, m)
            assert np.array_equal(synth.bf16_bits(step.V_pool[k, b]), ovs[b]), (b, k, m)
            assert int(step.pool_len[k, b]) == int(oln[b])
        kept = [l for l in range(cfg.layers) if l not in got]
        assert sorted(slots[b][kept].tolist()) == list(range(cfg.layers - cfg.budget))
        assert all(slots[b][m] == -1 for m in got)
        lo, hi = cu[b], cu[b + 1]
        for l in kept:
            s = int(slots[b][l])
            assert np.array_equal(synth.bf16_bits(step.K_full[s, lo:hi]), host_layers[l][1][lo:hi]), (b, l)
            assert np.array_equal(synth.bf16_bits(step.V_full[s, lo:hi]), host_layers[l][2][lo:hi]), (b, l)


# ------------------------------------------------------------- fused push

@pytest.mark.parametrize("spec", [
    dict(seqlens=(600,), hq=8, hkv=4, d=64, budget=3),
    dict(seqlens=(300, 77, 520, 190), hq=4, hkv=2, d=128, budget=2),
    dict(seqlens=(0,), hq=4, hkv=2, d=64, budget=1),
], ids=["one-seq-d64", "packed-d128", "empty"])
def test_fused_push_equals_separate_push(spec):
    cfg = synth.custom(name="push", layers=5, seqlens=spec["seqlens"], hq=spec["hq"], hkv=spec["hkv"], d=spec["d"],
                       S=4, W=48, n_obs=24, budget=spec["budget"], seed=17, lazy_layers=(1, 3))
    kw = _kw(cfg)
    a = lt.DeviceQueue(cfg.layers, cfg.budget, cfg.batch)
    b = lt.DeviceQueue(cfg.layers, cfg.budget, cfg.batch)
    for l in range(cfg.layers):
        Q, K, V = synth.layer_inputs(cfg, l, "cuda")
        ra = torch.zeros((cfg.batch, cfg.hq), dtype=torch.float32, device="cuda")
        rb = torch.zeros_like(ra)
        Oa, La, _ = lt.lt_prefill_attn_ratio_push(Q, K, V, cfg.S, cfg.W, cfg.n_obs, a, l, ra, **kw)
        Ob, Lb, _ = lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, ratio=rb, accumulate=True, **kw)
        b.push(l, rb)
        torch.cuda.synchronize()
        assert torch.equal(ra, rb) and torch.equal(Oa, Ob) and torch.equal(La, Lb)
    ma, oa = a.result()
    mb, ob = b.result()
    torch.cuda.synchronize()
    assert a.error() == 0 and b.error() == 0
    assert torch.equal(ma, mb) and torch.equal(oa, ob) and torch.equal(a.slots(), b.slots())
    assert int((ma.sum(dim=1) == cfg.budget).all()) == 1


def test_fused_push_flags_a_second_push_of_a_layer():
    cfg = synth.custom(name="push2", layers=3, seqlens=(200,), hq=4, hkv=2, d=64, S=4, W=16, n_obs=8, budget=1,
                       seed=19)
    q = lt.DeviceQueue(cfg.layers, cfg.budget, cfg.batch)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    r = torch.zeros((1, cfg.hq), dtype=torch.float32, device="cuda")
    lt.lt_prefill_attn_ratio_push(Q, K, V, cfg.S, cfg.W, cfg.n_obs, q, 0, r)
    r.zero_()
    lt.lt_prefill_attn_ratio_push(Q, K, V, cfg.S, cfg.W, cfg.n_obs, q, 0, r)
    torch.cuda.synchronize()
    assert q.error() & 1
    with pytest.raises(lt.LtError):
        lt.lt_prefill_attn_ratio_push(Q, K, V, cfg.S, cfg.W, cfg.n_obs, q, 3, r)    # layer out of range


# --------------------------------------------------------- pool vs oracle

def _pool_cfg():
    # 600 tokens: several 128-row tiles and a ragged tail; sink-biased layers 1, 3, 4
    return synth.custom(name="pool", layers=6, seqlens=(600,), hq=8, hkv=4, d=64, S=4, W=64, n_obs=32, budget=3,
                        seed=11, lazy_layers=(1, 3, 4))


def test_pool_step_matches_oracle_and_resident_step():
    cfg = _pool_cfg()
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(cfg.layers)]
    host = [tuple(synth.bf16_bits(t) for t in lay) for lay in layers]
    pool = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, kv_pool=True)
    _, order = _run(pool)
    assert sorted(order[0].tolist()) == [1, 3, 4]
    _check_against_oracle(cfg, pool, order, host)
    resident = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs)
    _, order_r = _run(resident)
    assert torch.equal(order, order_r) and torch.equal(pool.ratio, resident.ratio)
    assert torch.equal(pool.K_pool, resident.K_pool) and torch.equal(pool.V_pool, resident.V_pool)
    assert torch.equal(pool.pool_len, resident.pool_len)
    assert pool.kernel_launches() == 1 + 3 * cfg.layers
    # The queue push fused into the attention kernel gives the same step, bit for bit.
    fused = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, kv_pool=True, fused_push=True)
    _, order_f = _run(fused)
    assert fused.kernel_launches() == 1 + 2 * cfg.layers
    assert torch.equal(order, order_f) and torch.equal(pool.ratio, fused.ratio)
    assert torch.equal(pool.K_full, fused.K_full) and torch.equal(pool.K_pool, fused.K_pool)


def test_pool_step_packed_batch_per_sequence_slots():
    """Each sequence has its own queue and slots; a layer can be kept for one
    sequence and demoted for another."""
    cfg = synth.custom(name="poolb", layers=6, seqlens=(300, 77, 520, 190, 5), hq=4, hkv=2, d=128, S=4, W=48,
                       n_obs=24, budget=3, recency=True, seed=23)
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(cfg.layers)]
    host = [tuple(synth.bf16_bits(t) for t in lay) for lay in layers]
    step = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, kv_pool=True, **_kw(cfg))
    _, order = _run(step)
    _check_against_oracle(cfg, step, order, host)


@pytest.mark.parametrize("budget", [0, 6])
def test_pool_step_budget_edges(budget):
    cfg = synth.custom(name="poole", layers=6, seqlens=(600,), hq=8, hkv=4, d=64, S=4, W=64, n_obs=32,
                       budget=budget, seed=11, lazy_layers=(1, 3, 4))
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(cfg.layers)]
    host = [tuple(synth.bf16_bits(t) for t in lay) for lay in layers]
    step = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, kv_pool=True)
    _, order = _run(step)
    assert step.K_full.shape[0] == cfg.layers - budget and step.K_pool.shape[0] == budget
    _check_against_oracle(cfg, step, order, host)


# ----------------------------------------------------------- peak memory

def _nbytes(t):
    return t.numel() * t.element_size()


def _rounded(n):
    return (n + 511) // 512 * 512                 # the caching allocator's block granularity


@pytest.mark.parametrize("name", ["tiny", "gqa1p2b"])
def test_pool_prefill_peak_memory(name):
    """Every layer's Q/K/V is produced just before its turn (copied from host
    memory) and released after it, as a model's projections would: the device
    high-water mark over the prefill is the step's own buffers plus one
    layer's inputs, with C + 1 full KV layers in it, far below L full layers."""
    cfg = synth.CONFIGS[name]
    host_t = [synth.layer_inputs(cfg, l, "cpu") for l in range(cfg.layers)]
    host = [tuple(synth.bf16_bits(t) for t in lay) for lay in host_t]
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    step = lt.PrefillStep([None] * cfg.layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, kv_pool=True,
                          dims=(cfg.total_tokens, cfg.hq, cfg.hkv, cfg.d), **_kw(cfg))
    owned = sum(_rounded(_nbytes(t)) for t in (step.O, step.LSE, step.ratio, step.K_pool, step.V_pool,
                                                  step.pool_len, step.K_full, step.V_full, step.dq.state))
    after_init = torch.cuda.memory_allocated() - base
    assert after_init == owned, (after_init, owned)
    s = torch.cuda.current_stream()
    step.begin(s)
    for l in range(cfg.layers):
        Q, K, V = (t.to("cuda") for t in host_t[l])    # this layer's inputs, made now
        step.layer(l, s, qkv=(Q, K, V))
        del Q, K, V                                     # and released after its turn
    torch.cuda.synchronize()
    peak = torch.cuda.max_memory_allocated() - base
    one_layer = sum(_rounded(_nbytes(t)) for t in host_t[0])
    assert peak <= owned + one_layer + 4096, (peak, owned, one_layer)
    full, stream, held = step.kv_bytes()
    C = cfg.layers - cfg.budget
    assert held == C * full + cfg.budget * stream
    kv_peak = held + full                               # the C slots + the working layer + streaming caches
    assert kv_peak <= (C + 1) * full + cfg.budget * stream
    assert kv_peak < cfg.layers * full                  # every layer kept full
    # the pages' cap with budget = L/2: half the layers full (plus the working one), half streaming
    assert cfg.budget * 2 == cfg.layers and kv_peak <= (cfg.layers // 2 + 1) * full + (cfg.layers // 2) * stream
    assert step.dq.error() == 0
    _, order = step.dq.result()
    torch.cuda.synchronize()
    _check_against_oracle(cfg, step, order, host)
    if name == "tiny":
        assert sorted(order[0].tolist()) == [1, 3]


# ---------------------------------------------------------- decode, graph

def test_decode_over_a_kept_layer_slot_equals_its_own_cache():
    cfg = synth.custom(name="poold", layers=6, seqlens=(300, 520, 190), hq=4, hkv=2, d=64, S=4, W=48, n_obs=24,
                       budget=3, seed=29, lazy_layers=(0, 2, 5))
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(cfg.layers)]
    kw = _kw(cfg)
    step = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, kv_pool=True, **kw)
    _, order = _run(step)
    slots = step.dq.slots()
    q = torch.randn((cfg.batch, cfg.hq, cfg.d), device="cuda").bfloat16()
    lens = torch.tensor(cfg.seqlens, dtype=torch.int32, device="cuda")
    starts = kw["cu_seqlens"][:-1].contiguous()
    for l in range(cfg.layers):
        if bool((slots[:, l] < 0).any()):
            continue
        K, V, seq_start = step.kept_layer_cache(l, slots)
        O1, L1 = lt.lt_decode_attn(q, K, V, lens, seq_start=seq_start, max_len=cfg.max_seqlen)
        O2, L2 = lt.lt_decode_attn(q, layers[l][1], layers[l][2], lens, seq_start=starts, max_len=cfg.max_seqlen)
        torch.cuda.synchronize()
        assert torch.equal(O1, O2) and torch.equal(L1, L2), l


def test_pool_step_replayed_from_a_graph():
    cfg = _pool_cfg()
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(cfg.layers)]
    step = lt.PrefillStep(layers, cfg.budget, cfg.S, cfg.W, cfg.n_obs, kv_pool=True)
    _, order_eager = _run(step)
    k_full, v_full, k_pool = step.K_full.clone(), step.V_full.clone(), step.K_pool.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step.enqueue(s)
    for t in (step.K_full, step.V_full, step.K_pool):
        t.fill_(3.0)
    step.ratio.fill_(-1.0)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert step.dq.error() == 0
    _, order = step.dq.result()
    torch.cuda.synchronize()
    assert torch.equal(order, order_eager)
    assert torch.equal(step.K_full, k_full) and torch.equal(step.V_full, v_full) and torch.equal(step.K_pool, k_pool)

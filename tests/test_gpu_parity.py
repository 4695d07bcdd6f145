"""GPU parity: every step of the path through the C ABI against the fp64 oracle,
on the same seeded bf16 inputs.  Bars: O relative L2 <= 1e-2 per layer, LSE and
lazy ratio absolute error <= 2e-3, selection and compacted KV exact (except
layers whose oracle scores tie within 2e-3)."""
import numpy as np
import pytest
import torch

import kv_cache_compression_tcgen05_b200 as lt
import oracle
import synth
from tests.gpu_common import (LSE_ABS, O_REL_L2, RATIO_ABS, check_attention, cu_tensor, expected_uniform_ratio,
                              gpu_attention, gpu_ratio, oracle_ratio, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lt.library()
    yield
    assert lt.lt_device_status(True) == lt.LT_OK


# --------------------------------------------------------------- attention

def test_attention_tiny_every_layer_every_row():
    cfg = synth.CONFIGS["tiny"]
    for layer in range(cfg.layers):
        Q, K, V = synth.layer_inputs(cfg, layer, "cuda")
        O, LSE = gpu_attention(cfg, Q, K, V)
        torch.cuda.synchronize()
        rel, lse_err = check_attention(cfg, Q, K, V, O, LSE)
        assert rel <= O_REL_L2 and lse_err <= LSE_ABS, (layer, rel, lse_err)


RAGGED = [
    dict(seqlens=(1, 63, 129, 200, 300, 128, 256), hq=4, hkv=2, d=64),
    dict(seqlens=(1, 63, 129, 200, 300, 128, 256), hq=4, hkv=2, d=128),
    dict(seqlens=(383,), hq=6, hkv=1, d=64),
    dict(seqlens=(17, 640), hq=8, hkv=8, d=128),
    dict(seqlens=(0, 5, 0, 130), hq=2, hkv=1, d=64),
    # eight sequences with g = 8: long enough (>= 2 bands of 4 q-tiles) for the
    # banded work order, ragged lengths
    dict(seqlens=(1500, 1100, 1300, 1400, 1200, 1250, 1350, 1150), hq=16, hkv=2, d=64),
    dict(seqlens=(1500, 1100, 1300, 1400, 1200, 1250, 1350, 1150), hq=16, hkv=2, d=128),
]


@pytest.mark.parametrize("spec", RAGGED, ids=lambda s: f"{s['seqlens']}-{s['hq']}/{s['hkv']}-d{s['d']}")
def test_attention_ragged_batches(spec):
    cfg = synth.custom(seqlens=spec["seqlens"], hq=spec["hq"], hkv=spec["hkv"], d=spec["d"], seed=31)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    cu = cu_tensor(cfg)
    O, LSE = lt.lt_prefill_attn(Q, K, V, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    torch.cuda.synchronize()
    rel, lse_err = check_attention(cfg, Q, K, V, O, LSE)
    assert rel <= O_REL_L2 and lse_err <= LSE_ABS, (rel, lse_err)


@pytest.mark.parametrize("d", [64, 128])
def test_attention_uniform_closed_form(d):
    """q = 0: LSE_i = log(i+1) and O_i is the mean of v_0..v_i."""
    cfg = synth.custom(seqlens=(300,), hq=2, hkv=1, d=d, seed=32)
    _, K, V = synth.layer_inputs(cfg, 0, "cuda")
    Q = torch.zeros((cfg.total_tokens, cfg.hq, d), dtype=torch.bfloat16, device="cuda")
    O, LSE = gpu_attention(cfg, Q, K, V)
    torch.cuda.synchronize()
    i = torch.arange(cfg.total_tokens, dtype=torch.float64)
    assert (LSE.double().cpu() - torch.log(i + 1)[None, :]).abs().max().item() <= LSE_ABS
    means = V.double().cpu()[:, 0, :].cumsum(0) / (i + 1)[:, None]
    for h in range(cfg.hq):
        got = O.double().cpu()[:, h, :]
        assert ((got - means).norm() / means.norm()).item() <= O_REL_L2


def test_attention_scale_argument():
    cfg = synth.custom(seqlens=(200,), hq=4, hkv=2, d=64, seed=33)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    O, LSE = lt.lt_prefill_attn(Q, K, V, softmax_scale=0.05)
    torch.cuda.synchronize()
    cu = np.array(cfg.cu_seqlens(), np.int32)
    o_ref, lse_ref = oracle.attn(cu, synth.bf16_bits(Q), synth.bf16_bits(K), synth.bf16_bits(V), scale=0.05)
    assert np.abs(LSE.cpu().numpy() - lse_ref).max() <= LSE_ABS
    o = O.float().cpu().numpy()
    assert np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref) <= O_REL_L2


def test_attention_empty_batch_is_a_no_op():
    Q = torch.empty((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    K = torch.empty((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    O, LSE = lt.lt_prefill_attn(Q, K, K)
    assert O.shape == (0, 4, 64) and LSE.shape == (4, 0)


@pytest.mark.parametrize("name,n_random", [("gqa1p2b", 400), ("qwen32b", 64), ("batched", 64), ("long128k", 24)])
def test_attention_full_size_sampled_rows(name, n_random):
    """One layer at the workload's full size, in the launch configuration the
    benchmark times; the oracle checks sampled rows: every observed row (the
    last max(n_obs, 128) rows of every sequence, a ragged q-tile) of every
    head, the first rows, and random rows."""
    cfg = synth.CONFIGS[name]
    layer = 1
    Q, K, V = synth.layer_inputs(cfg, layer, "cuda")
    O, LSE = gpu_attention(cfg, Q, K, V)
    torch.cuda.synchronize()
    tokens, heads = sample_rows(cfg, n_random, seed=5, last_rows=max(cfg.n_obs, 128), heads_for_last=cfg.hq)
    rel, lse_err = check_attention(cfg, Q, K, V, O, LSE, tokens, heads)
    assert rel <= O_REL_L2 and lse_err <= LSE_ABS, (rel, lse_err)
    assert torch.isfinite(LSE).all() and torch.isfinite(O.float()).all()
    del Q, K, V, O, LSE
    torch.cuda.empty_cache()


# -------------------------------------------------------------- lazy ratio

def test_lazy_ratio_tiny_every_layer():
    cfg = synth.CONFIGS["tiny"]
    for layer in range(cfg.layers):
        Q, K, V = synth.layer_inputs(cfg, layer, "cuda")
        _, LSE = gpu_attention(cfg, Q, K, V)
        r = gpu_ratio(cfg, Q, K, LSE)
        torch.cuda.synchronize()
        ref = oracle_ratio(cfg, Q, K)
        assert np.abs(r.cpu().numpy() - ref).max() <= RATIO_ABS, layer


@pytest.mark.parametrize("spec", [
    dict(seqlens=(1, 63, 129, 200, 300), hq=4, hkv=2, d=64, S=4, W=32, n_obs=16),
    dict(seqlens=(1, 63, 129, 200, 300), hq=4, hkv=2, d=128, S=4, W=60, n_obs=100),
    dict(seqlens=(700,), hq=10, hkv=1, d=64, S=0, W=1, n_obs=130),
    dict(seqlens=(40, 9), hq=2, hkv=2, d=64, S=7, W=0, n_obs=64),
    dict(seqlens=(500,), hq=12, hkv=2, d=128, S=16, W=1000, n_obs=37),
], ids=lambda s: f"{s['seqlens']}-g{s['hq'] // s['hkv']}-d{s['d']}-S{s['S']}W{s['W']}n{s['n_obs']}")
def test_lazy_ratio_ragged(spec):
    cfg = synth.custom(seqlens=spec["seqlens"], hq=spec["hq"], hkv=spec["hkv"], d=spec["d"], S=spec["S"],
                       W=spec["W"], n_obs=spec["n_obs"], seed=41)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    _, LSE = gpu_attention(cfg, Q, K, V)
    r = gpu_ratio(cfg, Q, K, LSE)
    torch.cuda.synchronize()
    # End to end (GPU LSE) and with the oracle's own LSE handed to the kernel.
    ref = oracle_ratio(cfg, Q, K)
    assert np.abs(r.cpu().numpy() - ref).max() <= RATIO_ABS
    cu = np.array(cfg.cu_seqlens(), np.int32)
    _, lse_ref = oracle.attn(cu, synth.bf16_bits(Q), synth.bf16_bits(K), synth.bf16_bits(V))
    r2 = gpu_ratio(cfg, Q, K, torch.tensor(lse_ref, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert np.abs(r2.cpu().numpy() - oracle_ratio(cfg, Q, K, lse=lse_ref)).max() <= RATIO_ABS


def test_lazy_ratio_closed_forms():
    """Zero queries give min(S+W, i+1)/(i+1) averaged; S + W >= N gives 1."""
    cfg = synth.custom(seqlens=(50, 300, 1000), hq=4, hkv=1, d=64, S=4, W=60, n_obs=64, seed=42)
    _, K, V = synth.layer_inputs(cfg, 0, "cuda")
    Q = torch.zeros((cfg.total_tokens, cfg.hq, cfg.d), dtype=torch.bfloat16, device="cuda")
    cu = cu_tensor(cfg)
    _, LSE = lt.lt_prefill_attn(Q, K, V, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    r = lt.lt_lazy_ratio(Q, K, LSE, cfg.S, cfg.W, cfg.n_obs, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    torch.cuda.synchronize()
    want = expected_uniform_ratio(cfg)
    assert np.abs(r.cpu().numpy() - want[:, None]).max() <= RATIO_ABS
    Q2, K2, V2 = synth.layer_inputs(cfg, 0, "cuda")
    _, L2 = lt.lt_prefill_attn(Q2, K2, V2, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    r2 = lt.lt_lazy_ratio(Q2, K2, L2, 4, 2000, 64, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    torch.cuda.synchronize()
    assert np.abs(r2.cpu().numpy() - 1.0).max() <= RATIO_ABS


@pytest.mark.parametrize("name", ["gqa1p2b", "qwen32b", "batched", "long128k"])
def test_lazy_ratio_full_size(name):
    """Full size, in the launch configuration the benchmark times: the ratio
    kernel end to end (its LSE from the GPU attention) against the oracle with
    its own LSE (one full attention row per observed row and head), and as a
    unit against the oracle given the same LSE."""
    cfg = synth.CONFIGS[name]
    Q, K, V = synth.layer_inputs(cfg, 2, "cuda")
    _, LSE = gpu_attention(cfg, Q, K, V)
    r = gpu_ratio(cfg, Q, K, LSE)
    torch.cuda.synchronize()
    got = r.cpu().numpy()
    assert np.abs(got - oracle_ratio(cfg, Q, K)).max() <= RATIO_ABS
    ref = oracle_ratio(cfg, Q, K, lse=LSE.cpu().numpy().astype(np.float64))
    assert np.abs(got - ref).max() <= RATIO_ABS
    del Q, K, V, LSE
    torch.cuda.empty_cache()


# ------------------------------------------------------- selection / queue

def test_tiny_selection_end_to_end():
    """GPU ratios of the tiny workload select the designed lazy layers {1, 3},
    offline and through the online queue."""
    cfg = synth.CONFIGS["tiny"]
    ratios = []
    q = lt.LayerQueue(cfg.layers, cfg.budget)
    popped = []
    for layer in range(cfg.layers):
        Q, K, V = synth.layer_inputs(cfg, layer, "cuda")
        _, LSE = gpu_attention(cfg, Q, K, V)
        r = gpu_ratio(cfg, Q, K, LSE).cpu().numpy()
        ratios.append(r)
        dem = q.push(layer, lt.lt_layer_score(r[0]))
        if dem >= 0:
            popped.append(dem)
    lazy, order = lt.lt_select_layers(np.stack(ratios), cfg.budget)
    assert sorted(order[0].tolist()) == [1, 3] and sorted(popped) == [1, 3]


def test_selection_matches_oracle_gqa1p2b():
    cfg = synth.CONFIGS["gqa1p2b"]
    gpu, ref = [], []
    for layer in range(cfg.layers):
        Q, K, V = synth.layer_inputs(cfg, layer, "cuda")
        _, LSE = gpu_attention(cfg, Q, K, V)
        gpu.append(gpu_ratio(cfg, Q, K, LSE).cpu().numpy())
        ref.append(oracle_ratio(cfg, Q, K))
    gpu, ref = np.stack(gpu), np.stack(ref)
    assert np.abs(gpu - ref).max() <= RATIO_ABS
    _, order = lt.lt_select_layers(gpu, cfg.budget)
    sc = oracle.layer_scores(ref)[0]
    _, o_order = oracle.select_layers(sc, cfg.budget)
    got, want = set(order[0].tolist()), set(o_order.tolist())
    # Only layers whose oracle scores tie within the ratio tolerance may swap.
    boundary = np.sort(sc)[::-1][cfg.budget - 1: cfg.budget + 1]
    for l in got ^ want:
        assert abs(sc[l] - boundary).min() <= 2 * RATIO_ABS, (got, want)


# -------------------------------------------------------------- compaction

@pytest.mark.parametrize("spec", [
    dict(seqlens=(20, 3, 9, 0, 12, 300), hkv=2, d=64, S=2, W=5, mask=(1, 1, 0, 1, 1, 1)),
    dict(seqlens=(1000, 40), hkv=8, d=128, S=4, W=1020, mask=(1, 1)),
    dict(seqlens=(4096,), hkv=8, d=64, S=4, W=1020, mask=(1,)),
    dict(seqlens=(5000, 77), hkv=4, d=64, S=0, W=64, mask=(0, 1)),
], ids=lambda s: f"{s['seqlens']}-S{s['S']}W{s['W']}")
def test_compact_kv_bit_exact(spec):
    cfg = synth.custom(seqlens=spec["seqlens"], hq=spec["hkv"], hkv=spec["hkv"], d=spec["d"], S=spec["S"],
                       W=spec["W"], seed=51)
    _, K, V = synth.layer_inputs(cfg, 0, "cuda")
    B, slots = cfg.batch, cfg.S + cfg.W
    mask = torch.tensor(spec["mask"], dtype=torch.uint8, device="cuda")
    sentinel = torch.full((B, cfg.hkv, slots, cfg.d), -7.0, dtype=torch.bfloat16, device="cuda")
    ks, vs = sentinel.clone(), sentinel.clone()
    cu = cu_tensor(cfg)
    ks, vs, ln = lt.lt_compact_kv(K, V, mask, cfg.S, cfg.W, cu_seqlens=cu, max_seqlen=cfg.max_seqlen,
                                  k_stream=ks, v_stream=vs)
    torch.cuda.synchronize()
    sent_bits = synth.bf16_bits(sentinel)
    oks, ovs, oln = oracle.compact_kv(np.array(cfg.cu_seqlens(), np.int32), synth.bf16_bits(K), synth.bf16_bits(V),
                                      np.array(spec["mask"], np.uint8), cfg.S, cfg.W, Ks=sent_bits.copy(),
                                      Vs=sent_bits.copy())
    assert np.array_equal(synth.bf16_bits(ks), oks)
    assert np.array_equal(synth.bf16_bits(vs), ovs)
    assert np.array_equal(ln.cpu().numpy(), oln)


def test_device_status_clean():
    assert lt.lt_device_status(True) == lt.LT_OK


# ------------------------------------------------- fused attention + ratio

FUSED = [
    dict(name="tiny"),
    dict(seqlens=(1, 63, 129, 200, 300, 128, 256), hq=4, hkv=2, d=64, S=4, W=32, n_obs=16),
    dict(seqlens=(1, 63, 129, 200, 300), hq=4, hkv=2, d=128, S=4, W=60, n_obs=100),
    dict(seqlens=(700, 5), hq=10, hkv=2, d=64, S=0, W=1, n_obs=128),
    dict(seqlens=(500,), hq=6, hkv=2, d=128, S=16, W=1000, n_obs=37),
    dict(seqlens=(383, 260), hq=3, hkv=1, d=64, S=2, W=130, n_obs=128),
    dict(seqlens=(1500, 1100, 1300, 1400, 1200, 1250, 1350, 1150), hq=16, hkv=2, d=128, S=4, W=200, n_obs=40),
    # One sequence with more work items than SMs: the static longest-first
    # schedule, over q-tile pairs of one head (odd group) and over head pairs.
    dict(seqlens=(8000,), hq=12, hkv=4, d=64, S=4, W=700, n_obs=100),
    dict(seqlens=(5000,), hq=16, hkv=4, d=128, S=4, W=1500, n_obs=128),
    # One long sequence with an odd group: banded q-tile pairs, ragged last pair.
    dict(seqlens=(15000,), hq=10, hkv=2, d=64, S=4, W=3000, n_obs=100),
]


@pytest.mark.parametrize("spec", FUSED, ids=lambda s: s.get("name") or f"{s['seqlens']}-g{s['hq'] // s['hkv']}-d{s['d']}")
def test_fused_attention_ratio(spec):
    """The fused kernel gives the plain kernel's O and LSE bit for bit, and the
    oracle's ratio within the tolerance."""
    if "name" in spec:
        cfg = synth.CONFIGS[spec["name"]]
    else:
        cfg = synth.custom(seqlens=spec["seqlens"], hq=spec["hq"], hkv=spec["hkv"], d=spec["d"], S=spec["S"],
                           W=spec["W"], n_obs=spec["n_obs"], seed=61)
    from tests.gpu_common import gpu_fused
    for layer in range(min(cfg.layers, 4)):
        Q, K, V = synth.layer_inputs(cfg, layer, "cuda")
        O1, L1 = gpu_attention(cfg, Q, K, V)
        O2, L2, r = gpu_fused(cfg, Q, K, V)
        torch.cuda.synchronize()
        assert torch.equal(O1, O2) and torch.equal(L1, L2)
        rel, lse_err = check_attention(cfg, Q, K, V, O2, L2)
        assert rel <= O_REL_L2 and lse_err <= LSE_ABS, (rel, lse_err)
        ref = oracle_ratio(cfg, Q, K)
        assert np.abs(r.cpu().numpy() - ref).max() <= RATIO_ABS
        r_sep = gpu_ratio(cfg, Q, K, L2)
        torch.cuda.synchronize()
        assert np.abs(r.cpu().numpy() - r_sep.cpu().numpy()).max() <= 1e-4


@pytest.mark.parametrize("name", ["gqa1p2b", "qwen32b", "batched", "long128k"])
def test_fused_ratio_full_size(name):
    """The fused ratio at full size against the oracle with its own LSE (end to
    end), against the oracle given the kernel's LSE, and against the separate
    pass."""
    cfg = synth.CONFIGS[name]
    from tests.gpu_common import gpu_fused
    Q, K, V = synth.layer_inputs(cfg, 3, "cuda")
    O, LSE, r = gpu_fused(cfg, Q, K, V)
    r2 = gpu_ratio(cfg, Q, K, LSE)
    O1, L1 = gpu_attention(cfg, Q, K, V)
    torch.cuda.synchronize()
    assert torch.equal(O, O1) and torch.equal(LSE, L1)     # the plain kernel's O and LSE, bit for bit
    del O1, L1
    assert np.abs(r.cpu().numpy() - r2.cpu().numpy()).max() <= 1e-4
    assert np.abs(r.cpu().numpy() - oracle_ratio(cfg, Q, K)).max() <= RATIO_ABS
    ref = oracle_ratio(cfg, Q, K, lse=LSE.cpu().numpy().astype(np.float64))
    assert np.abs(r.cpu().numpy() - ref).max() <= RATIO_ABS
    # Run-to-run reproducibility of the fused ratio (n_obs <= 128).
    _, _, r3 = gpu_fused(cfg, Q, K, V)
    torch.cuda.synchronize()
    assert torch.equal(r, r3)


@pytest.mark.parametrize("d", [64, 128])
def test_fused_ratio_accumulate_mode(d):
    """lt_prefill_attn_ratio_acc adds into the caller's buffer: on a zeroed
    buffer it equals the zeroing call bit for bit, on a buffer holding c it
    gives c + ratio, and O / LSE are the same."""
    cfg = synth.custom(seqlens=(300, 77, 513), hq=4, hkv=2, d=d, S=4, W=60, n_obs=16, seed=61)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    cu = torch.tensor(cfg.cu_seqlens(), dtype=torch.int32, device="cuda")
    kw = dict(cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    O1, L1, r1 = lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, **kw)
    r0 = torch.zeros_like(r1)
    O2, L2, r2 = lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, ratio=r0, accumulate=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(r1, r2) and torch.equal(O1, O2) and torch.equal(L1, L2)
    rc = torch.full_like(r1, 0.25)
    lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, ratio=rc, accumulate=True, **kw)
    torch.cuda.synchronize()
    assert (rc - (r1 + 0.25)).abs().max().item() <= 1e-6
    with pytest.raises(ValueError):
        lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, accumulate=True, **kw)


def _schedule_sweep_specs():
    """Seeded single-sequence shapes whose launches take the static longest-first
    schedule (more work items than SMs, at most 1536): one per group size 1..6,
    both head dims, ragged lengths."""
    rng = np.random.default_rng(2024)
    specs = []
    for hq, hkv in [(16, 16), (32, 16), (24, 8), (32, 8), (40, 8), (12, 2)]:
        for _ in range(200):
            d = int(rng.choice([64, 128]))
            n = int(rng.integers(1200, 4200))
            S, W, n_obs = int(rng.integers(0, 9)), int(rng.integers(64, 1500)), int(rng.integers(16, 129))
            _, sched = lt.lt_attn_schedule(d, n, hq, hkv, 148, S=S, W=W, n_obs=n_obs, fused=True)
            if sched is not None:
                specs.append(dict(seqlens=(n,), hq=hq, hkv=hkv, d=d, S=S, W=W, n_obs=n_obs))
                break
    return specs


@pytest.mark.parametrize("spec", _schedule_sweep_specs(), ids=lambda s: f"{s['seqlens'][0]}-{s['hq']}x{s['hkv']}-d{s['d']}")
def test_static_schedule_parity_sweep(spec):
    """Launches that run the static schedule: plain and fused attention against the
    oracle on every row, the fused ratio against the oracle, and the fused kernel's
    O and LSE equal to the plain kernel's bit for bit."""
    cfg = synth.custom(seqlens=spec["seqlens"], hq=spec["hq"], hkv=spec["hkv"], d=spec["d"], S=spec["S"],
                       W=spec["W"], n_obs=spec["n_obs"], seed=77)
    from tests.gpu_common import gpu_fused
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    O1, L1 = gpu_attention(cfg, Q, K, V)
    O2, L2, r = gpu_fused(cfg, Q, K, V)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
    rel, lse_err = check_attention(cfg, Q, K, V, O2, L2)
    assert rel <= O_REL_L2 and lse_err <= LSE_ABS, (rel, lse_err)
    assert np.abs(r.cpu().numpy() - oracle_ratio(cfg, Q, K)).max() <= RATIO_ABS

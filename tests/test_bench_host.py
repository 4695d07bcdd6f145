"""Host logic of bench.py that the reported numbers rest on, checked without a GPU:
the algorithmic work counts (closed forms against brute-force enumeration of
the key sets the method defines), the KV-cache fraction a prefill leaves
(against the closed form (C + budget * min(1, (S+W)/N)) / L), and the parsing
of the nvidia-smi clock samples that decide whether a run is kept."""
import bench
import synth


def _key_set(i, S, W):
    """K_i: the sink keys [0, min(S, i+1)) and the window [max(S, i-W+1), i]."""
    return set(range(min(S, i + 1))) | set(range(max(S, i - W + 1), i + 1))


def _cases():
    yield synth.custom(name="a", seqlens=(37,), hq=4, hkv=2, d=64, S=4, W=8, n_obs=16)
    yield synth.custom(name="b", seqlens=(3, 50, 9), hq=6, hkv=3, d=128, S=4, W=5, n_obs=12)
    yield synth.custom(name="c", seqlens=(20,), hq=2, hkv=1, d=64, S=0, W=1, n_obs=30)
    yield synth.custom(name="d", seqlens=(12,), hq=2, hkv=1, d=64, S=6, W=40, n_obs=5)


def test_attention_flops_count_causal_pairs():
    for cfg in _cases():
        pairs = sum(1 for n in cfg.seqlens for i in range(n) for j in range(n) if j <= i)
        assert bench.attention_flops(cfg) == 4 * cfg.d * cfg.hq * pairs


def test_ratio_flops_count_the_observed_rows_key_sets():
    for cfg in _cases():
        keys = 0
        for n in cfg.seqlens:
            for i in range(max(0, n - cfg.n_obs), n):
                keys += len(_key_set(i, cfg.S, cfg.W))
        assert bench.ratio_flops(cfg) == 2 * cfg.d * cfg.hq * keys


def test_ratio_unique_bytes_count_the_union_of_touched_rows():
    for cfg in _cases():
        total = 0
        for n in cfg.seqlens:
            obs = range(max(0, n - cfg.n_obs), n)
            rows = set().union(*(_key_set(i, cfg.S, cfg.W) for i in obs))
            total += len(obs) * cfg.hq * (2 * cfg.d + 4) + len(rows) * cfg.hkv * 2 * cfg.d
        assert bench.ratio_unique_bytes(cfg) == total


def test_compaction_bytes_count_the_kept_rows():
    for cfg in _cases():
        kept = 0
        for n in cfg.seqlens:
            p = list(range(min(cfg.S, n))) + list(range(max(cfg.S, n - cfg.W), n))
            assert len(p) == len(set(p))
            kept += len(p)
        # K and V, each read and written, bf16
        assert bench.compaction_bytes(cfg, 3) == 3 * 2 * 2 * kept * cfg.hkv * cfg.d * 2


def test_clock_summary_reads_median_and_throttle_reasons():
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = cs.summary()
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    cs.lines = ["0, 1500, 1965, 900, 0x8, Active, Not Active, Active, Not Active"]
    assert cs.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_kv_fraction_after_prefill():
    import torch
    # one sequence, budget layers demoted, each keeping min(N, S+W) rows:
    # (C + budget * min(1, (S+W)/N)) / L with C = L - budget
    L, budget, N, S, W = 16, 8, 4096, 4, 1020
    order = torch.arange(budget, dtype=torch.int32).reshape(1, budget)
    pool_len = torch.full((budget, 1), min(N, S + W), dtype=torch.int32)
    want = ((L - budget) + budget * min(1.0, (S + W) / N)) / L
    assert abs(bench.kv_fraction_after_prefill(order, pool_len, (N,), L) - want) < 1e-12
    assert want == 0.625
    # ragged batch: sequence 1 demoted one layer only (-1 past its count), sequence 2 is short
    order = torch.tensor([[3, 1], [2, -1], [0, 1]], dtype=torch.int32)
    pool_len = torch.tensor([[24, 24, 9], [24, -7, 9]], dtype=torch.int32)    # [budget, batch]
    seqlens, L = (100, 50, 9), 4
    kept = (2 * 100 + 24 + 24) + (3 * 50 + 24) + (2 * 9 + 9 + 9)
    assert abs(bench.kv_fraction_after_prefill(order, pool_len, seqlens, L) - kept / (L * 159)) < 1e-12
    # budget 0: nothing demoted
    empty = torch.zeros((2, 0), dtype=torch.int32)
    assert bench.kv_fraction_after_prefill(empty, torch.zeros((0, 2), dtype=torch.int32), (5, 7), 3) == 1.0


def test_peak_choice_follows_the_averaging_region():
    """A per-launch time averaged over a short region is held against the
    burst tensor peak, one averaged over seconds against the sustained one."""
    peaks = {"bf16_tflops": 1679.2, "bf16_tflops_sustained": 1384.7, "hbm_gbs": 6455.9}
    peak, why = bench.choose_peak(peaks, 0.004)
    assert peak == 1679.2 and "burst" in why
    peak, why = bench.choose_peak(peaks, 5.0)
    assert peak == 1384.7 and "sustained" in why


def test_both_arms_describe_the_workload_alike():
    cfg = synth.CONFIGS["long128k"]
    a = bench.workload_config(cfg, True, 1, "replicas")
    b = bench.workload_config(cfg, True, 1, "replicas")
    assert a == b and a["kv_pool"] is True and "peak-memory cap" in a["workload"]
    assert a["parallelism"] == "single GPU"
    assert bench.workload_config(cfg, True, 2, "heads")["parallelism"].startswith("heads split over 2")

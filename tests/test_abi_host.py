"""Host-side checks of the C ABI: the library loads, exports every function the
header declares, rejects bad arguments before touching a device, and its host
queue / selection agree with the oracle.  No GPU needed."""
import ctypes
import itertools
import os
import re

import numpy as np
import pytest

import kv_cache_compression_tcgen05_b200 as lt
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    lt.build()
    return lt.library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "lt.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lt_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert {"lt_prefill_attn", "lt_lazy_ratio", "lt_select_layers", "lt_compact_kv", "lt_queue_push"} <= set(names)
    lib = ctypes.CDLL(lt.library_path())
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    assert lt.lt_status_string(lt.LT_OK) == "LT_OK"
    assert lt.lt_status_string(lt.LT_ERR_TIMEOUT) == "LT_ERR_TIMEOUT"
    assert lt.lt_version() >= 100


def _shape(**kw):
    s = lt.LtShape()
    s.batch, s.total_tokens, s.max_seqlen, s.hq, s.hkv, s.head_dim = 1, 256, 256, 4, 2, 64
    s.cu_seqlens = None
    for k, v in kw.items():
        setattr(s, k, v)
    return s


FAKE = 0x10000  # aligned, never dereferenced: every case below fails its checks first


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), lt.LT_ERR_UNSUPPORTED),
    (dict(head_dim=256), lt.LT_ERR_UNSUPPORTED),
    (dict(hq=3, hkv=2), lt.LT_ERR_INVALID_ARG),
    (dict(batch=0), lt.LT_ERR_INVALID_ARG),
    (dict(batch=2), lt.LT_ERR_INVALID_ARG),       # batch > 1 needs cu_seqlens
    (dict(total_tokens=-1), lt.LT_ERR_INVALID_ARG),
    (dict(hkv=0), lt.LT_ERR_INVALID_ARG),
])
def test_prefill_attn_rejects_bad_shapes(kw, status):
    s = _shape(**kw)
    rc = lt.library().lt_prefill_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, 0.0, None)
    assert rc == status


def test_calls_reject_null_and_misaligned_pointers():
    lib = lt.library()
    s = _shape()
    assert lib.lt_prefill_attn(None, FAKE, FAKE, FAKE, FAKE, FAKE, 0.0, None) == lt.LT_ERR_INVALID_ARG
    assert lib.lt_prefill_attn(ctypes.byref(s), None, FAKE, FAKE, FAKE, FAKE, 0.0, None) == lt.LT_ERR_INVALID_ARG
    assert lib.lt_prefill_attn(ctypes.byref(s), FAKE + 8, FAKE, FAKE, FAKE, FAKE, 0.0, None) == lt.LT_ERR_INVALID_ARG
    assert lib.lt_prefill_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE + 2, 0.0, None) == lt.LT_ERR_INVALID_ARG
    assert lib.lt_prefill_attn(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, float("nan"), None) == \
        lt.LT_ERR_INVALID_ARG


@pytest.mark.parametrize("S,W,n_obs", [(0, 0, 16), (-1, 4, 16), (4, -2, 16), (4, 32, 0), (4, 32, 5000)])
def test_lazy_ratio_rejects_bad_window(S, W, n_obs):
    s = _shape()
    rc = lt.library().lt_lazy_ratio(ctypes.byref(s), FAKE, FAKE, FAKE, 0.0, S, W, n_obs, FAKE, None)
    assert rc == lt.LT_ERR_INVALID_ARG


def test_lazy_ratio_rejects_grids_beyond_the_launch_limits():
    # one CTA cluster per (sequence, query head): hq and batch index grid dimensions of at most 65535
    s = _shape(hq=70000, hkv=1)
    assert lt.library().lt_lazy_ratio(ctypes.byref(s), FAKE, FAKE, FAKE, 0.0, 4, 32, 16, FAKE, None) == \
        lt.LT_ERR_INVALID_ARG


@pytest.mark.parametrize("S,W", [(0, 0), (-1, 3), (2, -1)])
def test_compact_rejects_bad_window(S, W):
    s = _shape()
    rc = lt.library().lt_compact_kv(ctypes.byref(s), FAKE, FAKE, FAKE, S, W, FAKE, FAKE, FAKE, None)
    assert rc == lt.LT_ERR_INVALID_ARG


def test_compact_rejects_null_mask():
    s = _shape()
    assert lt.library().lt_compact_kv(ctypes.byref(s), FAKE, FAKE, None, 4, 4, FAKE, FAKE, FAKE, None) == \
        lt.LT_ERR_INVALID_ARG


def test_layer_score_is_head_mean():
    r = np.array([0.25, 0.5, 0.75, 1.0], np.float32)
    assert abs(lt.lt_layer_score(r) - 0.625) < 1e-7


def test_select_layers_matches_oracle():
    rng = np.random.default_rng(3)
    for L, B, H in ((4, 1, 2), (16, 3, 8), (64, 8, 40)):
        ratios = rng.random((L, B, H)).astype(np.float32)
        for budget in (0, 1, L // 2, L):
            lazy, order = lt.lt_select_layers(ratios, budget)
            scores = ratios.astype(np.float64).mean(axis=2).T    # float64 head means, as the C code sums
            for b in range(B):
                o_lazy, o_order = oracle.select_layers(np.array([lt.lt_layer_score(ratios[l, b]) for l in range(L)]),
                                                       budget)
                assert np.array_equal(lazy[b], o_lazy)
                assert np.array_equal(order[b], o_order)
                assert abs(scores[b] - [lt.lt_layer_score(ratios[l, b]) for l in range(L)]).max() < 1e-6


def test_select_layers_rejects_non_finite_scores_and_bad_budget():
    r = np.ones((4, 1, 2), np.float32)
    with pytest.raises(lt.LtError):
        lt.lt_select_layers(r, 5)
    # NaN and +-inf are rejected, as the host and device queues reject them.
    for bad in (np.nan, np.inf, -np.inf):
        r = np.ones((4, 1, 2), np.float32)
        r[2, 0, 1] = bad
        with pytest.raises(lt.LtError):
            lt.lt_select_layers(r, 2)


def test_queue_matches_oracle_every_push_order():
    rng = np.random.default_rng(5)
    for L in range(1, 7):
        scores = np.round(rng.random(L), 1).astype(np.float32)   # rounding makes ties likely
        for budget in range(L + 1):
            for perm in itertools.permutations(range(L)):
                q = lt.LayerQueue(L, budget)
                popped = [x for x in (q.push(l, scores[l]) for l in perm) if x >= 0]
                want = oracle.queue_online(scores.astype(np.float64), budget, push_order=np.array(perm))
                assert popped == want.tolist(), (scores, perm, budget)
                assert len(q) == L - budget
                q.close()


def test_queue_rejects_bad_pushes():
    q = lt.LayerQueue(4, 2)
    assert q.push(0, 0.5) == -1
    for layer, score in ((0, 0.1), (4, 0.1), (-1, 0.1), (1, float("nan")), (1, float("inf"))):
        with pytest.raises(lt.LtError):
            q.push(layer, score)
    assert len(q) == 1
    with pytest.raises(lt.LtError):
        lt.lt_queue_create(3, 4)


def test_fused_accumulate_and_decode_calls_reject_bad_arguments():
    """The newer entry points check their arguments before any device call."""
    lib = lt.library()
    s = _shape()
    INV, UNS = lt.LT_ERR_INVALID_ARG, lt.LT_ERR_UNSUPPORTED
    # fused attention in accumulate mode needs a ratio buffer
    assert lib.lt_prefill_attn_ratio_acc(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, 0.0, 4, 32, 16, None,
                                         None) == INV
    # decode over a full cache: (q, K, V, seq_start, seq_capacity, len, batch, hq, hkv, d, max_len, O, LSE, scale)
    assert lib.lt_decode_attn(FAKE, FAKE, FAKE, None, 16, FAKE, 1, 4, 2, 64, 17, FAKE, FAKE, 0.0, None) == INV
    assert lib.lt_decode_attn(FAKE, FAKE, FAKE, None, 16, FAKE, 1, 5, 2, 64, 16, FAKE, FAKE, 0.0, None) == INV
    assert lib.lt_decode_attn(FAKE, FAKE, FAKE, None, 16, FAKE, 1, 4, 2, 64, 0, FAKE, FAKE, 0.0, None) == INV
    assert lib.lt_decode_attn(FAKE + 8, FAKE, FAKE, None, 16, FAKE, 1, 4, 2, 64, 16, FAKE, FAKE, 0.0, None) == INV
    assert lib.lt_decode_attn(FAKE, FAKE, FAKE, None, 16, FAKE, 1, 4, 2, 96, 16, FAKE, FAKE, 0.0, None) == UNS
    # decode over a streaming cache: (q, K, V, len, batch, hq, hkv, d, slots, O, LSE, scale)
    assert lib.lt_stream_decode(FAKE, FAKE, FAKE, FAKE, 0, 4, 2, 64, 8, FAKE, FAKE, 0.0, None) == INV
    assert lib.lt_stream_decode(FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 64, 0, FAKE, FAKE, 0.0, None) == INV
    assert lib.lt_stream_decode(FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 80, 8, FAKE, FAKE, 0.0, None) == UNS
    assert lib.lt_stream_decode(FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 64, 8, FAKE, FAKE, float("inf"), None) == INV
    # ring state
    assert lib.lt_stream_ring_init(FAKE, FAKE, 1, 4, 0, None) == INV
    assert lib.lt_stream_ring_init(FAKE + 2, FAKE, 1, 4, 8, None) == INV
    assert lib.lt_stream_append(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 96, 4, 8, None) == UNS


def test_queue_and_pool_calls_reject_bad_arguments():
    lib = lt.library()
    s = _shape()
    INV = lt.LT_ERR_INVALID_ARG
    assert lib.lt_dqueue_state_bytes(0, 1) == 0 and lib.lt_dqueue_state_bytes(4, 0) == 0
    assert lib.lt_dqueue_state_bytes(4, 2) > 0
    assert lib.lt_dqueue_init(FAKE, 4, 5, 1, None) == INV           # budget > L
    assert lib.lt_dqueue_init(FAKE + 4, 4, 2, 1, None) == INV       # state not 16-byte aligned
    assert lib.lt_dqueue_push(FAKE, 0, 1, 0, FAKE, 2, None) == INV   # L < 1
    assert lib.lt_dqueue_push(FAKE, 4, 1, 0, FAKE, 0, None) == INV   # hq < 1
    # (state, L, batch, layer, ratio, shards, hq_shard)
    assert lib.lt_dqueue_push_gathered(FAKE, 4, 1, 0, FAKE, 0, 4, None) == INV   # shards < 1
    assert lib.lt_dqueue_push_gathered(FAKE, 4, 1, 0, FAKE, 2, 0, None) == INV   # hq_shard < 1
    assert lib.lt_dqueue_push_gathered(FAKE, 4, 0, 0, FAKE, 2, 4, None) == INV   # batch < 1
    assert lib.lt_dqueue_push_gathered(FAKE, 4, 1, 0, FAKE + 2, 2, 4, None) == INV   # ratio not 4-byte aligned
    # (shape, K_layers, V_layers, state, L, budget, S, W, K_pool, V_pool, pool_len)
    assert lib.lt_compact_kv_pending(ctypes.byref(s), FAKE, FAKE, FAKE, 4, 0, 4, 8, FAKE, FAKE, FAKE, None) == INV
    assert lib.lt_compact_kv_pending(ctypes.byref(s), FAKE, FAKE, FAKE, 4, 2, 0, 0, FAKE, FAKE, FAKE, None) == INV
    # (shape, K_layers, V_layers, L, layers, n, S, W, K_pool, V_pool, pool_len)
    assert lib.lt_compact_kv_layers(ctypes.byref(s), FAKE, FAKE, 4, FAKE, 5, 4, 8, FAKE, FAKE, FAKE, None) == INV
    assert lib.lt_compact_kv_layers(ctypes.byref(s), FAKE, FAKE, 0, FAKE, 0, 4, 8, FAKE, FAKE, FAKE, None) == INV
    assert lib.lt_compact_kv_layers(ctypes.byref(s), FAKE, FAKE, 4, FAKE, 1, 0, 0, FAKE, FAKE, FAKE, None) == INV
    # nothing to compact: succeeds without a device
    assert lib.lt_compact_kv_layers(ctypes.byref(s), FAKE, FAKE, 4, None, 0, 4, 8, None, None, None, None) == lt.LT_OK
    assert lib.lt_selftest_wait_timeout(0, None) == INV


@pytest.mark.parametrize("max_len,splits", [(1, 1), (256, 1), (1024, 4), (4096, 16), (5000, 16), (8192, 16),
                                            (16384, 16), (32768, 32), (131072, 128), (1 << 20, 128)])
def test_splitk_workspace_follows_the_split_rule(max_len, splits):
    """The split-K decode splits each (sequence, KV head) into ceil(max_len / r)
    CTAs, r = ceil(max_len / 16) clamped to [256, 1024], at most 128; its
    workspace holds batch x hq x splits x (head_dim + 2) floats (host call)."""
    for batch, hq, d in [(1, 32, 128), (3, 8, 64)]:
        assert lt.lt_decode_splitk_workspace_bytes(batch, hq, d, max_len) == batch * hq * splits * (d + 2) * 4

"""Pins of the fp64 oracle against what the mathematics fixes.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with an
independent fact: a closed form, an invariant, a library routine (scipy's
logsumexp/softmax) applied to the fully materialised score matrix, or brute
force over every case of a tiny input.  None of them re-types the oracle's own
loops.  ``tests/test_oracle_pins.py`` runs them on the real oracle and
``tests/test_oracle_mutants.py`` runs them on deliberately broken copies of it.
"""
from __future__ import annotations

import itertools
import math

import numpy as np
from scipy.special import logsumexp, softmax

import oracle


# ----------------------------------------------------------------- helpers

def bits_of(x) -> np.ndarray:
    """bf16 bits of float values that bf16 holds exactly (asserted)."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def values_of(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def rand_bf16(rng, shape, scale=1.0):
    """Random normal values rounded down to bf16 by truncation (exact bits)."""
    f = (rng.standard_normal(shape) * scale).astype(np.float32)
    return ((f.view(np.uint32) >> 16).astype(np.uint16)).reshape(shape)


def rand_int_bf16(rng, shape, lo=-3, hi=3):
    return bits_of(rng.integers(lo, hi + 1, size=shape).astype(np.float32))


def cu_of(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)


def dense_reference(cu, Q, K, V, scale):
    """LSE [hq, T] and O [T, hq, d] from the materialised masked score matrix,
    reduced with scipy.special.logsumexp / softmax.  GQA is realised by
    repeating every KV head g times (np.repeat), not by index arithmetic."""
    q, k, v = values_of(Q), values_of(K), values_of(V)
    T, hq, d = q.shape
    g = hq // k.shape[1]
    k = np.repeat(k, g, axis=1)
    v = np.repeat(v, g, axis=1)
    lse = np.full((hq, T), np.nan)
    out = np.full((T, hq, d), np.nan)
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        n = s1 - s0
        if n == 0:
            continue
        for h in range(hq):
            S = scale * q[s0:s1, h, :] @ k[s0:s1, h, :].T
            S[np.triu(np.ones((n, n), bool), 1)] = -np.inf
            lse[h, s0:s1] = logsumexp(S, axis=1)
            out[s0:s1, h, :] = softmax(S, axis=1) @ v[s0:s1, h, :]
    return lse, out


def key_set(i, S, W):
    """K_i as a Python set: the sink keys and the W most recent keys."""
    sink = set(range(0, min(S, i + 1)))
    recent = set(range(max(0, i - W + 1), i + 1))
    return sink | recent


# ----------------------------------------------------------- attention pins

def pin_attention_matches_scipy_on_ragged_gqa():
    rng = np.random.default_rng(11)
    lengths = [5, 1, 13, 8]
    cu = cu_of(lengths)
    T, hq, hkv, d = int(cu[-1]), 4, 2, 8
    Q, K, V = rand_bf16(rng, (T, hq, d)), rand_bf16(rng, (T, hkv, d)), rand_bf16(rng, (T, hkv, d))
    scale = 1.0 / math.sqrt(d)
    O, LSE = oracle.attn(cu, Q, K, V, scale=scale, nthreads=2)
    lse_ref, o_ref = dense_reference(cu, Q, K, V, scale)
    assert np.allclose(LSE, lse_ref, rtol=0, atol=1e-12), np.abs(LSE - lse_ref).max()
    assert np.allclose(O, o_ref, rtol=0, atol=1e-12), np.abs(O - o_ref).max()


def pin_zero_queries_closed_form():
    """q = 0 makes attention uniform: LSE_i = log(i+1), O_i = mean(v_0..v_i)."""
    rng = np.random.default_rng(12)
    lengths = [9, 4]
    cu = cu_of(lengths)
    T, hq, hkv, d = int(cu[-1]), 2, 1, 4
    Q = np.zeros((T, hq, d), np.uint16)
    K, V = rand_bf16(rng, (T, hkv, d)), rand_bf16(rng, (T, hkv, d))
    O, LSE = oracle.attn(cu, Q, K, V)
    for b in range(len(lengths)):
        s0, s1 = cu[b], cu[b + 1]
        v = values_of(V[s0:s1, 0, :])
        means = np.cumsum(v, axis=0) / np.arange(1, s1 - s0 + 1)[:, None]
        for h in range(hq):
            assert np.allclose(LSE[h, s0:s1], np.log(np.arange(1, s1 - s0 + 1)), atol=1e-14)
            assert np.allclose(O[s0:s1, h, :], means, atol=1e-14)


def pin_first_row_and_two_keys():
    """Row 0 sees only key 0: O_0 = v_0, LSE_0 = s_00.  Row 1 (two keys):
    LSE = log(e^a + e^b), O = (e^a v_0 + e^b v_1) / (e^a + e^b)."""
    Qv = np.array([[[1, 2]], [[2, -1]]], np.float32)
    Kv = np.array([[[1, 1]], [[0, 2]]], np.float32)
    Vv = np.array([[[3, -4]], [[5, 8]]], np.float32)
    cu = cu_of([2])
    O, LSE = oracle.attn(cu, bits_of(Qv), bits_of(Kv), bits_of(Vv), scale=0.5)
    assert LSE[0, 0] == 0.5 * 3.0 and np.array_equal(O[0, 0], [3.0, -4.0])
    a, b = 0.5 * (2 * 1 + -1 * 1), 0.5 * (2 * 0 + -1 * 2)
    assert abs(LSE[0, 1] - math.log(math.exp(a) + math.exp(b))) < 1e-15
    wa, wb = math.exp(a) / (math.exp(a) + math.exp(b)), math.exp(b) / (math.exp(a) + math.exp(b))
    assert np.allclose(O[1, 0], [wa * 3 + wb * 5, wa * -4 + wb * 8], atol=1e-15)


def pin_key_shift_invariance():
    """k_j += t w for all keys raises LSE_i by scale t (q_i . w); O is unchanged."""
    rng = np.random.default_rng(13)
    T, hq, hkv, d = 12, 2, 2, 4
    cu = cu_of([T])
    Qf = rng.integers(-2, 3, (T, hq, d)).astype(np.float32)
    Kf = rng.integers(-2, 3, (T, hkv, d)).astype(np.float32)
    V = rand_bf16(rng, (T, hkv, d))
    w = np.array([1, 0, -1, 2], np.float32)
    O1, L1 = oracle.attn(cu, bits_of(Qf), bits_of(Kf), V, scale=0.5)
    O2, L2 = oracle.attn(cu, bits_of(Qf), bits_of(Kf + w), V, scale=0.5)
    shift = 0.5 * np.einsum("thd,d->ht", Qf.astype(np.float64), w.astype(np.float64))
    assert np.allclose(L2 - L1, shift, atol=1e-12)
    assert np.allclose(O1, O2, atol=1e-12)


def pin_gqa_head_mapping():
    """Query head h reads KV head floor(h / g): with KV head 0 all zero, heads
    0..g-1 attend uniformly and heads g..2g-1 do not."""
    rng = np.random.default_rng(14)
    T, hq, hkv, d = 10, 4, 2, 4
    cu = cu_of([T])
    Q = rand_bf16(rng, (T, hq, d), 2.0)
    Kf = np.zeros((T, hkv, d), np.float32)
    Kf[:, 1, :] = rng.integers(-3, 4, (T, d))
    V = rand_bf16(rng, (T, hkv, d))
    _, LSE = oracle.attn(cu, Q, bits_of(Kf), V)
    uniform = np.log(np.arange(1, T + 1))
    for h in range(hq):
        is_uniform = np.allclose(LSE[h], uniform, atol=1e-12)
        assert is_uniform == (h < 2), (h, LSE[h])


def pin_gqa_equals_repeated_heads():
    rng = np.random.default_rng(15)
    T, hq, hkv, d = 9, 6, 2, 8
    cu = cu_of([4, 5])
    Q, K, V = rand_bf16(rng, (T, hq, d)), rand_bf16(rng, (T, hkv, d)), rand_bf16(rng, (T, hkv, d))
    O1, L1 = oracle.attn(cu, Q, K, V)
    O2, L2 = oracle.attn(cu, Q, np.ascontiguousarray(np.repeat(K, 3, axis=1)),
                         np.ascontiguousarray(np.repeat(V, 3, axis=1)))
    assert np.array_equal(L1, L2) and np.array_equal(O1, O2)


def pin_packed_equals_separate():
    """A packed batch equals each sequence run on its own (no cross talk)."""
    rng = np.random.default_rng(16)
    lengths = [3, 7, 1, 6]
    cu = cu_of(lengths)
    T, hq, hkv, d = int(cu[-1]), 2, 1, 8
    Q, K, V = rand_bf16(rng, (T, hq, d)), rand_bf16(rng, (T, hkv, d)), rand_bf16(rng, (T, hkv, d))
    O, L = oracle.attn(cu, Q, K, V)
    for b in range(len(lengths)):
        s0, s1 = cu[b], cu[b + 1]
        Ob, Lb = oracle.attn(cu_of([s1 - s0]), np.ascontiguousarray(Q[s0:s1]), np.ascontiguousarray(K[s0:s1]),
                             np.ascontiguousarray(V[s0:s1]))
        assert np.array_equal(O[s0:s1], Ob) and np.array_equal(L[:, s0:s1], Lb)


def pin_causality():
    """Changing keys/values after row i leaves row i unchanged; changing key i
    itself (the diagonal) changes it."""
    rng = np.random.default_rng(17)
    T, hq, hkv, d = 8, 1, 1, 4
    cu = cu_of([T])
    Q, K, V = rand_bf16(rng, (T, hq, d)), rand_bf16(rng, (T, hkv, d)), rand_bf16(rng, (T, hkv, d))
    O, L = oracle.attn(cu, Q, K, V)
    i = 4
    K2, V2 = K.copy(), V.copy()
    K2[i + 1:] = rand_bf16(rng, K2[i + 1:].shape, 3.0)
    V2[i + 1:] = rand_bf16(rng, V2[i + 1:].shape, 3.0)
    O2, L2 = oracle.attn(cu, Q, K2, V2)
    assert np.array_equal(O2[: i + 1], O[: i + 1]) and np.array_equal(L2[:, : i + 1], L[:, : i + 1])
    K3 = K.copy()
    K3[i] = bits_of(values_of(K[i]).astype(np.float32) * 2)
    _, L3 = oracle.attn(cu, Q, K3, V)
    assert L3[0, i] != L[0, i] and np.array_equal(L3[0, :i], L[0, :i])


def pin_scale_parameter():
    """Doubling every query equals doubling the scale."""
    rng = np.random.default_rng(18)
    T, hq, hkv, d = 7, 2, 1, 8
    cu = cu_of([T])
    Q, K, V = rand_bf16(rng, (T, hq, d)), rand_bf16(rng, (T, hkv, d)), rand_bf16(rng, (T, hkv, d))
    O1, L1 = oracle.attn(cu, Q, K, V, scale=0.3)
    O2, L2 = oracle.attn(cu, bits_of(values_of(Q).astype(np.float32) * 2), K, V, scale=0.15)
    assert np.allclose(L1, L2, atol=1e-13) and np.allclose(O1, O2, atol=1e-13)


# ---------------------------------------------------------- lazy ratio pins

def _ratio_problem(seed, lengths=(40, 23), hq=4, hkv=2, d=8):
    rng = np.random.default_rng(seed)
    cu = cu_of(list(lengths))
    T = int(cu[-1])
    return cu, rand_bf16(rng, (T, hq, d), 1.5), rand_bf16(rng, (T, hkv, d), 1.5)


def _all_rows(cu, hq):
    return oracle.all_items(cu, hq)


def pin_ratio_is_one_when_key_set_covers_row():
    cu, Q, K = _ratio_problem(21)
    S, W = 3, 5
    tok, hd = _all_rows(cu, Q.shape[1])
    r = oracle.lazy_ratio_rows(cu, Q, K, S, W, tok, hd)
    pos = tok - cu[np.searchsorted(cu, tok, side="right") - 1]
    covered = S + W >= pos + 1
    assert covered.any() and (~covered).any()
    assert np.allclose(r[covered], 1.0, atol=1e-12)
    assert np.all(r[~covered] < 1.0 - 1e-9) and np.all(r > 0)


def pin_ratio_zero_queries_closed_form():
    """Uniform attention: r_i = min(S+W, i+1) / (i+1)."""
    cu, Q, K = _ratio_problem(22)
    Q = np.zeros_like(Q)
    for S, W in ((4, 7), (0, 3), (5, 0), (2, 50)):
        tok, hd = _all_rows(cu, Q.shape[1])
        r = oracle.lazy_ratio_rows(cu, Q, K, S, W, tok, hd)
        pos = (tok - cu[np.searchsorted(cu, tok, side="right") - 1]).astype(np.float64)
        assert np.allclose(r, np.minimum(S + W, pos + 1) / (pos + 1), atol=1e-14), (S, W)


def pin_ratio_routes_agree():
    cu, Q, K = _ratio_problem(23)
    tok, hd = _all_rows(cu, Q.shape[1])
    for S, W in ((4, 6), (1, 1), (0, 9)):
        ra = oracle.lazy_ratio_rows(cu, Q, K, S, W, tok, hd, route="A")
        rb = oracle.lazy_ratio_rows(cu, Q, K, S, W, tok, hd, route="B")
        assert np.allclose(ra, rb, atol=1e-12, rtol=0)


def pin_ratio_matches_scipy_softmax_over_key_set():
    """r_i = sum of scipy softmax weights of row i over the Python set K_i."""
    cu, Q, K = _ratio_problem(24)
    T, hq, d = Q.shape
    g = hq // K.shape[1]
    q, k = values_of(Q), np.repeat(values_of(K), g, axis=1)
    S, W = 3, 6
    tok, hd = _all_rows(cu, hq)
    r = oracle.lazy_ratio_rows(cu, Q, K, S, W, tok, hd)
    sc = 1.0 / math.sqrt(d)
    for n, (t, h) in enumerate(zip(tok, hd)):
        b = int(np.searchsorted(cu, t, side="right") - 1)
        i = int(t - cu[b])
        row = sc * k[cu[b]: t + 1, h, :] @ q[t, h, :]
        p = softmax(row)
        want = sum(p[j] for j in key_set(i, S, W))
        assert abs(r[n] - want) < 1e-12, (t, h, r[n], want)


def pin_ratio_diagonal_weight():
    """S = 0, W = 1 keeps only key i: r_i is the diagonal softmax weight."""
    cu, Q, K = _ratio_problem(25, lengths=(17,), hq=2, hkv=1)
    V = np.zeros_like(K)
    tok, hd = _all_rows(cu, 2)
    r = oracle.lazy_ratio_rows(cu, Q, K, 0, 1, tok, hd)
    _, LSE = oracle.attn(cu, Q, K, V)
    q, k = values_of(Q), values_of(K)
    sc = 1.0 / math.sqrt(Q.shape[2])
    diag = np.array([math.exp(sc * q[t, h] @ k[t, 0] - LSE[h, t]) for t, h in zip(tok, hd)])
    assert np.allclose(r, diag, atol=1e-13)


def pin_ratio_monotone_in_S_and_W():
    cu, Q, K = _ratio_problem(26)
    tok, hd = _all_rows(cu, Q.shape[1])
    prev = None
    for W in range(0, 12, 3):
        r = oracle.lazy_ratio_rows(cu, Q, K, 2, W, tok, hd)
        if prev is not None:
            assert np.all(r >= prev - 1e-15)
        prev = r
    prev = None
    for S in range(0, 10, 2):
        r = oracle.lazy_ratio_rows(cu, Q, K, S, 4, tok, hd)
        if prev is not None:
            assert np.all(r >= prev - 1e-15)
        prev = r
    r = oracle.lazy_ratio_rows(cu, Q, K, 0, 10**6, tok, hd)
    assert np.allclose(r, 1.0, atol=1e-12)


def pin_ratio_mean_over_last_rows():
    """ratio[b, h] is the mean of r_i over the last min(n_obs, N_b) rows, and
    using the oracle's own LSE as the given denominator changes nothing."""
    cu, Q, K = _ratio_problem(27, lengths=(30, 6, 19))
    T, hq, d = Q.shape
    S, W, n_obs = 2, 5, 8
    ratio = oracle.lazy_ratio(cu, Q, K, S, W, n_obs)
    tok, hd = _all_rows(cu, hq)
    r = oracle.lazy_ratio_rows(cu, Q, K, S, W, tok, hd).reshape(hq, T)
    for b in range(len(cu) - 1):
        nb = min(n_obs, cu[b + 1] - cu[b])
        want = r[:, cu[b + 1] - nb: cu[b + 1]].mean(axis=1)
        assert np.allclose(ratio[b], want, atol=1e-14)
    _, LSE = oracle.attn(cu, Q, K, np.zeros_like(K))
    assert np.allclose(oracle.lazy_ratio(cu, Q, K, S, W, n_obs, lse=LSE), ratio, atol=1e-14)


def pin_layer_scores_are_head_means():
    rng = np.random.default_rng(28)
    ratios = rng.random((5, 3, 4))
    assert np.allclose(oracle.layer_scores(ratios), ratios.mean(axis=2).T, atol=1e-15)


# --------------------------------------------------------------- queue pins

def _top_by_sort(scores, budget):
    ranked = sorted(range(len(scores)), key=lambda l: (-scores[l], l))
    return ranked[:budget]


def pin_queue_equals_full_sort_all_push_orders():
    """The online pops equal the top-`budget` of a full sort, for every push
    order of L <= 6 layers, with and without tied scores."""
    rng = np.random.default_rng(31)
    for L in range(1, 7):
        for trial in range(3):
            scores = rng.random(L) if trial < 2 else rng.integers(0, 3, L).astype(np.float64)
            for budget in range(0, L + 1):
                want = set(_top_by_sort(list(scores), budget))
                lazy, order = oracle.select_layers(scores, budget)
                assert list(order) == _top_by_sort(list(scores), budget)
                assert set(np.flatnonzero(lazy)) == want
                for perm in itertools.permutations(range(L)):
                    popped = oracle.queue_online(scores, budget, push_order=np.array(perm))
                    assert len(popped) == budget and set(popped.tolist()) == want, (scores, perm, popped)


def pin_queue_pops_max_of_current_queue():
    """Each pop is the best-ranked layer among those pushed and not yet popped,
    and no pop happens while at most C = L - budget layers are queued."""
    rng = np.random.default_rng(32)
    L, budget = 8, 3
    scores = rng.random(L)
    popped = list(oracle.queue_online(scores, budget))
    cap = L - budget
    queued, k = [], 0
    for l in range(L):
        queued.append(l)
        while len(queued) > cap:
            best = max(queued, key=lambda x: (scores[x], -x))
            assert popped[k] == best
            queued.remove(best)
            k += 1
    assert k == budget
    assert list(oracle.queue_online(scores, L)) == list(range(L))
    assert len(oracle.queue_online(scores, 0)) == 0


# ---------------------------------------------------------- compaction pins

def pin_compaction_matches_slicing():
    rng = np.random.default_rng(41)
    lengths = [20, 3, 9, 0, 12]
    cu = cu_of(lengths)
    T, hkv, d = int(cu[-1]), 2, 4
    K = rng.integers(0, 2**16, (T, hkv, d), dtype=np.uint16)
    V = rng.integers(0, 2**16, (T, hkv, d), dtype=np.uint16)
    S, W = 2, 5
    mask = np.array([1, 1, 0, 1, 1], np.uint8)
    sentinel = np.uint16(0xBEEF)
    Ks0 = np.full((len(lengths), hkv, S + W, d), sentinel, np.uint16)
    Ks, Vs, ln = oracle.compact_kv(cu, K, V, mask, S, W, Ks=Ks0.copy(), Vs=Ks0.copy())
    for b, n in enumerate(lengths):
        if not mask[b]:
            assert ln[b] == 0 and np.all(Ks[b] == sentinel) and np.all(Vs[b] == sentinel)
            continue
        keep = sorted(set(range(min(S, n))) | set(range(max(S, n - W), n)))
        assert ln[b] == len(keep) == min(n, S + W)
        rows = [cu[b] + p for p in keep]
        assert np.array_equal(Ks[b][:, : len(keep)], K[rows].transpose(1, 0, 2))
        assert np.array_equal(Vs[b][:, : len(keep)], V[rows].transpose(1, 0, 2))
        assert np.all(Ks[b][:, len(keep):] == 0) and np.all(Vs[b][:, len(keep):] == 0)


# ------------------------------------------------------ keyed-attention pins

def pin_keyed_attention_matches_scipy():
    rng = np.random.default_rng(51)
    n, m_max, d = 6, 9, 8
    q = rand_bf16(rng, (n, d), 1.5)
    K, V = rand_bf16(rng, (n, m_max, d), 1.5), rand_bf16(rng, (n, m_max, d))
    m = np.array([9, 1, 4, 0, 7, 9], np.int32)
    O, LSE = oracle.attn_keys(q, K, V, m, scale=0.4)
    for i in range(n):
        if m[i] == 0:
            assert LSE[i] == -np.inf and np.all(O[i] == 0)
            continue
        row = 0.4 * values_of(K[i, : m[i]]) @ values_of(q[i])
        assert abs(LSE[i] - logsumexp(row)) < 1e-12
        assert np.allclose(O[i], softmax(row) @ values_of(V[i, : m[i]]), atol=1e-12)


def pin_keyed_attention_uniform():
    rng = np.random.default_rng(52)
    K, V = rand_bf16(rng, (2, 5, 4)), rand_bf16(rng, (2, 5, 4))
    O, LSE = oracle.attn_keys(np.zeros((2, 4), np.uint16), K, V, np.array([5, 3], np.int32))
    assert np.allclose(LSE, np.log([5, 3]), atol=1e-15)
    assert np.allclose(O[1], values_of(V[1, :3]).mean(axis=0), atol=1e-15)


def pin_streaming_normaliser_is_lse_plus_log_ratio():
    """Over the key set K_i of row i, log sum exp(s_ij) = LSE_i + log r_i: the
    streaming attention's normaliser is the full one times the lazy ratio."""
    cu, Q, K = _ratio_problem(53, lengths=(37, 12), hq=2, hkv=1, d=8)
    V = rand_bf16(np.random.default_rng(54), K.shape)
    S, W = 3, 5
    _, LSE = oracle.attn(cu, Q, K, V)
    for b in range(len(cu) - 1):
        t = int(cu[b + 1] - 1)
        i = int(t - cu[b])
        keys = sorted(key_set(i, S, W))
        for h in range(Q.shape[1]):
            r = oracle.lazy_ratio_rows(cu, Q, K, S, W, np.array([t]), np.array([h]))[0]
            Ks = np.ascontiguousarray(K[[cu[b] + j for j in keys], 0][None])
            Vs = np.ascontiguousarray(V[[cu[b] + j for j in keys], 0][None])
            _, lse_s = oracle.attn_keys(np.ascontiguousarray(Q[t, h][None]), Ks, Vs, np.array([len(keys)], np.int32))
            assert abs(lse_s[0] - (LSE[h, t] + np.log(r))) < 1e-12


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]

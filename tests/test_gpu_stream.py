"""Decode attention: on a demoted layer's streaming cache against the fp64
oracle, against the prefill through the identity
    log sum_{j in K_i} exp(s_ij) = LSE_i + log r_i,
the ring-buffer append against a Python model of it; and on a kept layer's
full cache against the oracle and against the prefill's last row."""
import numpy as np
import pytest
import torch

import kv_cache_compression_tcgen05_b200 as lt
import oracle
import synth
from tests.gpu_common import LSE_ABS, O_REL_L2, cu_tensor, gpu_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lt.library()
    yield
    assert lt.lt_device_status(True) == lt.LT_OK


def oracle_decode(q, Ks, Vs, ln, scale=None):
    """Oracle of lt_stream_decode: q [B, hq, d], caches [B, hkv, slots, d], ln [B]."""
    B, hq, d = q.shape
    hkv, slots = Ks.shape[1], Ks.shape[2]
    g = hq // hkv
    qb, kb, vb = synth.bf16_bits(q), synth.bf16_bits(Ks), synth.bf16_bits(Vs)
    items_q = qb.reshape(B * hq, d)
    items_k = np.ascontiguousarray(np.repeat(kb, g, axis=1).reshape(B * hq, slots, d))
    items_v = np.ascontiguousarray(np.repeat(vb, g, axis=1).reshape(B * hq, slots, d))
    m = np.repeat(np.asarray(ln, np.int32), hq)
    O, LSE = oracle.attn_keys(items_q, items_k, items_v, m, scale=scale)
    return O.reshape(B, hq, d), LSE.reshape(B, hq)


def compare(O, LSE, O_ref, L_ref):
    Of = O.float().cpu().numpy().astype(np.float64)
    Lg = LSE.cpu().numpy().astype(np.float64)
    finite = np.isfinite(L_ref)
    assert np.array_equal(np.isfinite(Lg), finite)
    assert np.abs(Lg[finite] - L_ref[finite]).max() <= LSE_ABS
    assert np.all(Of[~finite] == 0)
    num = np.linalg.norm(Of - O_ref)
    assert num / max(np.linalg.norm(O_ref), 1e-30) <= O_REL_L2


@pytest.mark.parametrize("B,hq,hkv,d,slots", [(5, 8, 2, 64, 40), (3, 10, 2, 128, 100), (4, 4, 4, 64, 1024),
                                              (2, 5, 1, 128, 2048)])
def test_stream_decode_matches_oracle(B, hq, hkv, d, slots):
    g = torch.Generator(device="cuda").manual_seed(B * 1000 + slots)
    q = torch.randn((B, hq, d), generator=g, device="cuda").bfloat16()
    Ks = (torch.randn((B, hkv, slots, d), generator=g, device="cuda") * 1.5).bfloat16()
    Vs = torch.randn((B, hkv, slots, d), generator=g, device="cuda").bfloat16()
    ln = torch.tensor([slots, 1, 0, slots // 2, 7][:B], dtype=torch.int32, device="cuda")
    O, LSE = lt.lt_stream_decode(q, Ks, Vs, ln)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_decode(q, Ks, Vs, ln.cpu().numpy())
    compare(O, LSE, O_ref, L_ref)


@pytest.mark.parametrize("name_or_spec", ["tiny", dict(seqlens=(300, 37, 1500), hq=8, hkv=2, d=128, S=4, W=100,
                                                        n_obs=16)], ids=["tiny", "ragged-d128"])
def test_stream_decode_normaliser_is_lse_plus_log_ratio(name_or_spec):
    """Decoding the last prefill row over its layer's compacted cache gives
    LSE_last + log r_last: the streaming normaliser is the full one times the
    row's lazy ratio."""
    if isinstance(name_or_spec, str):
        cfg = synth.CONFIGS[name_or_spec]
    else:
        s = name_or_spec
        cfg = synth.custom(seqlens=s["seqlens"], hq=s["hq"], hkv=s["hkv"], d=s["d"], S=s["S"], W=s["W"],
                           n_obs=s["n_obs"], seed=81)
    Q, K, V = synth.layer_inputs(cfg, 1, "cuda")
    _, LSE = gpu_attention(cfg, Q, K, V)
    cu = cu_tensor(cfg)
    mask = torch.ones(cfg.batch, dtype=torch.uint8, device="cuda")
    Ks, Vs, ln = lt.lt_compact_kv(K, V, mask, cfg.S, cfg.W, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    last = torch.tensor(cfg.cu_seqlens()[1:], device="cuda") - 1
    q = Q[last].contiguous()                                     # [B, hq, d]
    O, L_dec = lt.lt_stream_decode(q, Ks, Vs, ln)
    torch.cuda.synchronize()
    cu_h = np.array(cfg.cu_seqlens(), np.int32)
    toks = np.repeat(cu_h[1:] - 1, cfg.hq).astype(np.int32)
    heads = np.tile(np.arange(cfg.hq, dtype=np.int32), cfg.batch)
    r = oracle.lazy_ratio_rows(cu_h, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, toks, heads)
    _, lse_full = oracle.attn(cu_h, synth.bf16_bits(Q), synth.bf16_bits(K), synth.bf16_bits(V), tokens=toks,
                              heads=heads)
    want = (lse_full + np.log(r)).reshape(cfg.batch, cfg.hq)
    assert np.abs(L_dec.cpu().numpy() - want).max() <= LSE_ABS
    O_ref, L_ref = oracle_decode(q, Ks, Vs, ln.cpu().numpy())
    compare(O, L_dec, O_ref, L_ref)
    assert np.abs(L_ref - want).max() < 1e-9                      # the identity, in the oracle alone


def test_stream_append_ring_and_decode():
    """Appending tokens keeps exactly the sink and W most recent positions, in
    ring order, and decoding the newest token equals the oracle's attention
    over that key set."""
    S, W, hkv, hq, d = 3, 5, 2, 4, 64
    lengths = [2, 6, 20]                       # below S, below S+W, above S+W
    B, slots, steps = len(lengths), S + W, 9
    g = torch.Generator(device="cuda").manual_seed(91)
    total = max(lengths) + steps
    Kfull = torch.randn((B, total, hkv, d), generator=g, device="cuda").bfloat16()
    Vfull = torch.randn((B, total, hkv, d), generator=g, device="cuda").bfloat16()
    # Prefill part as a packed batch, compacted on the GPU.
    Kp = torch.cat([Kfull[b, :n] for b, n in enumerate(lengths)]).contiguous()
    Vp = torch.cat([Vfull[b, :n] for b, n in enumerate(lengths)]).contiguous()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    mask = torch.ones(B, dtype=torch.uint8, device="cuda")
    Ks, Vs, ln = lt.lt_compact_kv(Kp, Vp, mask, S, W, cu_seqlens=cu, max_seqlen=max(lengths))
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    lt.lt_stream_ring_init(ln, nxt, S, W)
    # Python model of the cache: slot -> position.
    model = []
    for n in lengths:
        keep = sorted(set(range(min(S, n))) | set(range(max(S, n - W), n)))
        model.append({"pos": keep + [None] * (slots - len(keep)), "len": len(keep),
                      "next": len(keep) if len(keep) < slots else S})
    for t in range(steps):
        pos = [n + t for n in lengths]
        k_new = torch.stack([Kfull[b, pos[b]] for b in range(B)]).contiguous()
        v_new = torch.stack([Vfull[b, pos[b]] for b in range(B)]).contiguous()
        lt.lt_stream_append(Ks, Vs, ln, nxt, k_new, v_new, S, W)
        for b in range(B):
            m = model[b]
            m["pos"][m["next"]] = pos[b]
            if m["len"] < slots:
                m["len"] += 1
                m["next"] = m["len"] if m["len"] < slots else S
            else:
                m["next"] = S + (m["next"] - S + 1) % W
        torch.cuda.synchronize()
        for b in range(B):
            m = model[b]
            assert int(ln[b]) == m["len"] and int(nxt[b]) == m["next"]
            want = set(range(min(S, pos[b] + 1))) | set(range(max(S, pos[b] - W + 1), pos[b] + 1))
            assert set(p for p in m["pos"][: m["len"]]) == want
            for slot, p_ in enumerate(m["pos"][: m["len"]]):
                assert torch.equal(Ks[b, :, slot], Kfull[b, p_]) and torch.equal(Vs[b, :, slot], Vfull[b, p_])
        q = torch.randn((B, hq, d), generator=g, device="cuda").bfloat16()
        O, L = lt.lt_stream_decode(q, Ks, Vs, ln)
        torch.cuda.synchronize()
        O_ref, L_ref = oracle_decode(q, Ks, Vs, ln.cpu().numpy())
        compare(O, L, O_ref, L_ref)


def test_stream_rejects_bad_args():
    q = torch.zeros((1, 4, 96), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 2, 8, 96), dtype=torch.bfloat16, device="cuda")
    ln = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(lt.LtError):
        lt.lt_stream_decode(q, K, K, ln)
    nxt = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(lt.LtError):
        lt.lt_stream_ring_init(ln, nxt, 4, 0)


def oracle_decode_full(q, K, V, starts, ln):
    """Oracle of lt_decode_attn on a token-major cache K/V [rows, hkv, d]."""
    B, hq, d = q.shape
    hkv = K.shape[1]
    g = hq // hkv
    m_max = max(1, int(max(ln)))
    kb, vb = synth.bf16_bits(K), synth.bf16_bits(V)
    items_k = np.zeros((B * hq, m_max, d), np.uint16)
    items_v = np.zeros((B * hq, m_max, d), np.uint16)
    for b in range(B):
        n = int(ln[b])
        for h in range(hq):
            items_k[b * hq + h, :n] = kb[starts[b]:starts[b] + n, h // g]
            items_v[b * hq + h, :n] = vb[starts[b]:starts[b] + n, h // g]
    m = np.repeat(np.asarray(ln, np.int32), hq)
    O, LSE = oracle.attn_keys(synth.bf16_bits(q).reshape(B * hq, d), items_k, items_v, m)
    return O.reshape(B, hq, d), LSE.reshape(B, hq)


@pytest.mark.parametrize("spec", [dict(seqlens=(300, 37, 1500), hq=8, hkv=2, d=64),
                                  dict(seqlens=(129, 2000), hq=10, hkv=2, d=128),
                                  dict(seqlens=(4096,), hq=32, hkv=8, d=64)], ids=["ragged-d64", "d128-g5", "4k"])
def test_full_decode_of_last_row_equals_prefill(spec):
    """Decoding each sequence's last prefill query over the packed prefill K/V
    gives the prefill's own last-row O and LSE (the last row sees every key)."""
    cfg = synth.custom(seqlens=spec["seqlens"], hq=spec["hq"], hkv=spec["hkv"], d=spec["d"], S=4, W=64, n_obs=8,
                       seed=17)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    O_pf, LSE_pf = gpu_attention(cfg, Q, K, V)
    cu_h = np.array(cfg.cu_seqlens(), np.int32)
    starts = torch.tensor(cu_h[:-1], dtype=torch.int32, device="cuda")
    ln = torch.tensor(np.diff(cu_h), dtype=torch.int32, device="cuda")
    last = torch.tensor(cu_h[1:] - 1, device="cuda", dtype=torch.long)
    q = Q[last].contiguous()
    O, L = lt.lt_decode_attn(q, K, V, ln, seq_start=starts, max_len=cfg.max_seqlen)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_decode_full(q, K, V, cu_h[:-1], np.diff(cu_h))
    compare(O, L, O_ref, L_ref)
    # Same numbers as the prefill kernel's last rows.
    assert (L - LSE_pf[:, last].T).abs().max().item() <= 2 * LSE_ABS
    diff = (O.float() - O_pf[last].float()).norm() / O_pf[last].float().norm()
    assert diff.item() <= 2 * O_REL_L2


@pytest.mark.parametrize("B,cap,hq,hkv,d", [(6, 300, 8, 2, 64), (3, 20000, 8, 8, 128), (2, 70, 6, 3, 128),
                                             (1, 9000, 16, 8, 64)])
def test_full_decode_padded_cache_matches_oracle(B, cap, hq, hkv, d):
    g = torch.Generator(device="cuda").manual_seed(cap + d)
    q = torch.randn((B, hq, d), generator=g, device="cuda").bfloat16()
    K = (torch.randn((B, cap, hkv, d), generator=g, device="cuda") * 1.2).bfloat16()
    V = torch.randn((B, cap, hkv, d), generator=g, device="cuda").bfloat16()
    lens = [cap, 0, 1, cap // 3, cap - 1, 129][:B]
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    O, L = lt.lt_decode_attn(q, K, V, ln)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_decode_full(q, K.reshape(B * cap, hkv, d), V.reshape(B * cap, hkv, d),
                                      [b * cap for b in range(B)], lens)
    compare(O, L, O_ref, L_ref)


def test_full_decode_rejects_bad_args():
    q = torch.zeros((2, 4, 64), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((2, 16, 2, 64), dtype=torch.bfloat16, device="cuda")
    ln = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(lt.LtError):            # capacity below max_len
        lt.lt_decode_attn(q, K, K, ln, max_len=17)
    with pytest.raises(ValueError):            # packed cache without seq_start
        lt.lt_decode_attn(q, K[0], K[0], ln)


# ------------------------------------------------------------ split-K decode

@pytest.mark.parametrize("B,cap,hq,hkv,d", [(6, 300, 8, 2, 64), (3, 20000, 8, 8, 128), (2, 70, 6, 3, 128),
                                             (1, 9000, 16, 8, 64), (1, 40000, 32, 8, 128)])
def test_splitk_decode_padded_cache_matches_oracle(B, cap, hq, hkv, d):
    """The split-K decode (many CTAs per (sequence, KV head), partial states in
    a workspace, merged in split order) against the oracle on ragged lengths
    (0, 1, the whole capacity, and ones that leave splits empty)."""
    g = torch.Generator(device="cuda").manual_seed(cap + d + 1)
    q = torch.randn((B, hq, d), generator=g, device="cuda").bfloat16()
    K = (torch.randn((B, cap, hkv, d), generator=g, device="cuda") * 1.2).bfloat16()
    V = torch.randn((B, cap, hkv, d), generator=g, device="cuda").bfloat16()
    lens = [cap, 0, 1, cap // 3, cap - 1, 129][:B]
    ln = torch.tensor(lens, dtype=torch.int32, device="cuda")
    O, L = lt.lt_decode_attn_splitk(q, K, V, ln)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_decode_full(q, K.reshape(B * cap, hkv, d), V.reshape(B * cap, hkv, d),
                                      [b * cap for b in range(B)], lens)
    compare(O, L, O_ref, L_ref)
    # Deterministic: the same bits on a second call with a dirty workspace.
    ws = torch.full((lt.lt_decode_splitk_workspace_bytes(B, hq, d, cap),), 0x7F, dtype=torch.uint8, device="cuda")
    O2, L2 = lt.lt_decode_attn_splitk(q, K, V, ln, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(O, O2) and torch.equal(L, L2)


def test_splitk_decode_of_last_row_equals_prefill():
    """Packed prefill K/V of a long and a short sequence: decoding each
    sequence's last prefill query gives the prefill's own last-row O and LSE."""
    cfg = synth.custom(seqlens=(33000, 700), hq=8, hkv=2, d=128, S=4, W=64, n_obs=8, seed=19)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    O_pf, LSE_pf = gpu_attention(cfg, Q, K, V)
    cu_h = np.array(cfg.cu_seqlens(), np.int32)
    starts = torch.tensor(cu_h[:-1], dtype=torch.int32, device="cuda")
    ln = torch.tensor(np.diff(cu_h), dtype=torch.int32, device="cuda")
    last = torch.tensor(cu_h[1:] - 1, device="cuda", dtype=torch.long)
    q = Q[last].contiguous()
    O, L = lt.lt_decode_attn_splitk(q, K, V, ln, seq_start=starts, max_len=cfg.max_seqlen)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_decode_full(q, K, V, cu_h[:-1], np.diff(cu_h))
    compare(O, L, O_ref, L_ref)
    assert (L - LSE_pf[:, last].T).abs().max().item() <= 2 * LSE_ABS
    diff = (O.float() - O_pf[last].float()).norm() / O_pf[last].float().norm()
    assert diff.item() <= 2 * O_REL_L2


def test_splitk_decode_rejects_a_small_workspace():
    q = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 5000, 2, 64), dtype=torch.bfloat16, device="cuda")
    ln = torch.full((1,), 5000, dtype=torch.int32, device="cuda")
    need = lt.lt_decode_splitk_workspace_bytes(1, 4, 64, 5000)
    assert need == 4 * 16 * (64 + 2) * 4         # 4 heads; splits of ceil(5000 / 16) = 313 rows: 16 splits
    with pytest.raises(lt.LtError):
        lt.lt_decode_attn_splitk(q, K, K, ln, workspace=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))

"""Guard bands around every output of the library's calls: each output tensor
is a view into a larger buffer whose guard regions (before and after) and
whose own elements are first filled with a sentinel bit pattern.  After the
call the guards must be intact (no write outside the output) and no output
element may still hold the sentinel (every element the call owns is written).
Ragged packed batches with lengths 1, 129 and 300 put tiles' tails at buffer
ends.  Also: the binding rejects outputs and per-sequence vectors of the wrong
size before anything is enqueued."""
import numpy as np
import pytest
import torch

import kv_cache_compression_tcgen05_b200 as lt
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lt.library()
    yield
    assert lt.lt_device_status(True) == lt.LT_OK

GUARD_BYTES = 8192
PATTERN = 0x5A


def guarded(shape, dtype):
    """(buffer of bytes, view of `shape` inside it) with sentinel everywhere."""
    itemsize = torch.empty((), dtype=dtype).element_size()
    n = int(np.prod(shape)) * itemsize
    buf = torch.full((GUARD_BYTES + n + GUARD_BYTES,), PATTERN, dtype=torch.uint8, device="cuda")
    view = buf[GUARD_BYTES:GUARD_BYTES + n].view(dtype).view(shape)
    return buf, view


def check(buf, view, name, fully_written=True):
    torch.cuda.synchronize()
    assert bool((buf[:GUARD_BYTES] == PATTERN).all()), f"{name}: write before the output"
    assert bool((buf[-GUARD_BYTES:] == PATTERN).all()), f"{name}: write after the output"
    if fully_written:
        item = view.element_size()
        words = view.reshape(-1).view(torch.uint8).view(-1, item)
        untouched = (words == PATTERN).all(dim=1)
        assert not bool(untouched.any()), f"{name}: {int(untouched.sum())} elements not written"


CASES = [((1, 129, 300), 6, 2, 64), ((129, 1, 300), 4, 4, 128), ((300,), 8, 2, 64)]


@pytest.mark.parametrize("seqlens,hq,hkv,d", CASES)
def test_prefill_outputs_stay_inside_their_buffers(seqlens, hq, hkv, d):
    cfg = synth.custom(seqlens=seqlens, hq=hq, hkv=hkv, d=d, S=4, W=16, n_obs=24, seed=3)
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    T = cfg.total_tokens
    cu = torch.tensor(cfg.cu_seqlens(), dtype=torch.int32, device="cuda") if cfg.batch > 1 else None
    kw = dict(cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    bo, O = guarded((T, hq, d), torch.bfloat16)
    bl, LSE = guarded((hq, T), torch.float32)
    lt.lt_prefill_attn(Q, K, V, out=O, lse=LSE, **kw)
    check(bo, O, "attn O")
    check(bl, LSE, "attn LSE")
    bo, O = guarded((T, hq, d), torch.bfloat16)
    bl, LSE = guarded((hq, T), torch.float32)
    br, R = guarded((cfg.batch, hq), torch.float32)
    lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, out=O, lse=LSE, ratio=R, **kw)
    check(bo, O, "fused O")
    check(bl, LSE, "fused LSE")
    check(br, R, "fused ratio")
    br, R = guarded((cfg.batch, hq), torch.float32)
    lt.lt_lazy_ratio(Q, K, LSE, cfg.S, cfg.W, cfg.n_obs, out=R, **kw)
    check(br, R, "separate ratio")
    slots = cfg.S + cfg.W
    bk, Ks = guarded((cfg.batch, hkv, slots, d), torch.bfloat16)
    bv, Vs = guarded((cfg.batch, hkv, slots, d), torch.bfloat16)
    bn, ln = guarded((cfg.batch,), torch.int32)
    mask = torch.ones(cfg.batch, dtype=torch.uint8, device="cuda")
    lt.lt_compact_kv(K, V, mask, cfg.S, cfg.W, k_stream=Ks, v_stream=Vs, stream_len=ln, **kw)
    check(bk, Ks, "compact K")
    check(bv, Vs, "compact V")
    check(bn, ln, "compact len")
    # decode over the compacted cache and over the full packed cache
    q = torch.randn((cfg.batch, hq, d), device="cuda").bfloat16()
    bo, Od = guarded((cfg.batch, hq, d), torch.bfloat16)
    bl, Ld = guarded((cfg.batch, hq), torch.float32)
    lt.lt_stream_decode(q, Ks, Vs, ln, out=Od, lse=Ld)
    check(bo, Od, "stream decode O")
    check(bl, Ld, "stream decode LSE")
    cu_h = cfg.cu_seqlens()
    starts = torch.tensor(cu_h[:-1], dtype=torch.int32, device="cuda")
    lens = torch.tensor(np.diff(cu_h), dtype=torch.int32, device="cuda")
    bo, Od = guarded((cfg.batch, hq, d), torch.bfloat16)
    bl, Ld = guarded((cfg.batch, hq), torch.float32)
    lt.lt_decode_attn(q, K, V, lens, seq_start=starts, max_len=cfg.max_seqlen, out=Od, lse=Ld)
    check(bo, Od, "full decode O")
    check(bl, Ld, "full decode LSE")


def test_queue_and_pool_outputs_stay_inside_their_buffers():
    cfg = synth.custom(layers=4, seqlens=(1, 129, 300), hq=4, hkv=2, d=64, S=4, W=16, n_obs=24, seed=5)
    L, B, budget = cfg.layers, cfg.batch, 2
    layers = [synth.layer_inputs(cfg, l, "cuda") for l in range(L)]
    Kp = lt.layer_pointer_table([lay[1] for lay in layers])
    Vp = lt.layer_pointer_table([lay[2] for lay in layers])
    slots = cfg.S + cfg.W
    bk, K_pool = guarded((budget, B, cfg.hkv, slots, cfg.d), torch.bfloat16)
    bv, V_pool = guarded((budget, B, cfg.hkv, slots, cfg.d), torch.bfloat16)
    bn, pool_len = guarded((budget, B), torch.int32)
    cu = torch.tensor(cfg.cu_seqlens(), dtype=torch.int32, device="cuda")
    dq = lt.DeviceQueue(L, budget, B)
    ratios = torch.rand((L, B, cfg.hq), device="cuda")
    for l in range(L):
        dq.push(l, ratios[l])
        lt.lt_compact_kv_pending(Kp, Vp, dq, cfg.S, cfg.W, K_pool, V_pool, pool_len, cfg.total_tokens, cfg.hkv,
                                 cfg.d, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    check(bk, K_pool, "pending K pool")
    check(bv, V_pool, "pending V pool")
    check(bn, pool_len, "pending pool len")
    bm, mask = guarded((B, L), torch.uint8)
    bo, order = guarded((B, budget), torch.int32)
    lt.lt_dqueue_result(dq.state, L, B, budget, lazy_mask=mask, order=order)
    check(bm, mask, "lazy mask", fully_written=False)   # uint8 0/1 never equals the sentinel byte anyway
    check(bo, order, "order")
    # several layers in one launch
    bk, K_pool = guarded((3, B, cfg.hkv, slots, cfg.d), torch.bfloat16)
    bv, V_pool = guarded((3, B, cfg.hkv, slots, cfg.d), torch.bfloat16)
    bn, pool_len = guarded((3, B), torch.int32)
    pick = torch.tensor([2, 0, 3], dtype=torch.int32, device="cuda")
    lt.lt_compact_kv_layers(Kp, Vp, pick, cfg.S, cfg.W, K_pool, V_pool, pool_len, cfg.total_tokens, cfg.hkv, cfg.d,
                            cu_seqlens=cu, max_seqlen=cfg.max_seqlen)
    check(bk, K_pool, "layers K pool")
    check(bv, V_pool, "layers V pool")
    check(bn, pool_len, "layers pool len")


def test_binding_rejects_wrong_sizes():
    B, hq, hkv, d, slots = 3, 4, 2, 64, 20
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device="cuda")
    Ks = torch.zeros((B, hkv, slots, d), dtype=torch.bfloat16, device="cuda")
    ln = torch.ones(B, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        lt.lt_stream_decode(q, Ks, Ks, ln[:2])
    with pytest.raises(ValueError):
        lt.lt_stream_decode(q, Ks, Ks, ln, out=torch.empty((B, hq, d - 8), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        lt.lt_stream_decode(q, Ks, Ks, ln, lse=torch.empty((B, hq), dtype=torch.float32))   # host tensor
    Kc = torch.zeros((B, 16, hkv, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        lt.lt_decode_attn(q, Kc, Kc, ln[:1])
    with pytest.raises(ValueError):
        lt.lt_decode_attn(q, Kc, Kc, ln, lse=torch.empty((B, hq + 1), dtype=torch.float32, device="cuda"))
    nxt = torch.zeros(B - 1, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        lt.lt_stream_ring_init(ln, nxt, 4, 16)
    dq = lt.DeviceQueue(4, 2, B)
    with pytest.raises(ValueError):
        lt.lt_dqueue_result(dq.state, 4, B, 2, order=torch.empty((B, 1), dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert lt.lt_device_status(True) == lt.LT_OK

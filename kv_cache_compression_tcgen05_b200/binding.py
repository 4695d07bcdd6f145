"""ctypes binding of ``liblt.so``: the C functions of ``include/lt.h`` under the
same names, with torch tensors in and out.  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

from .build import LIB

LT_OK = 0
LT_ERR_INVALID_ARG = 1
LT_ERR_UNSUPPORTED = 2
LT_ERR_CUDA = 3
LT_ERR_TIMEOUT = 4

_lock = threading.Lock()
_lib = None


class LtShape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("total_tokens", ctypes.c_int),
        ("max_seqlen", ctypes.c_int),
        ("hq", ctypes.c_int),
        ("hkv", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("cu_seqlens", ctypes.c_void_p),
    ]


class LtError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {lt_status_string(status)}")
        self.status = status


_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_shp = ctypes.POINTER(LtShape)

_SIGS = {
    "lt_prefill_attn": (_i, [_shp, _vp, _vp, _vp, _vp, _vp, _f, _vp]),
    "lt_prefill_attn_ratio": (_i, [_shp, _vp, _vp, _vp, _vp, _vp, _f, _i, _i, _i, _vp, _vp]),
    "lt_prefill_attn_ratio_acc": (_i, [_shp, _vp, _vp, _vp, _vp, _vp, _f, _i, _i, _i, _vp, _vp]),
    "lt_prefill_attn_ratio_push": (_i, [_shp, _vp, _vp, _vp, _vp, _vp, _f, _i, _i, _i, _vp, _vp, _i, _i, _vp]),
    "lt_lazy_ratio": (_i, [_shp, _vp, _vp, _vp, _f, _i, _i, _i, _vp, _vp]),
    "lt_layer_score": (_f, [_vp, _i]),
    "lt_select_layers": (_i, [_vp, _i, _i, _i, _i, _vp, _vp]),
    "lt_attn_schedule": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i]),
    "lt_queue_create": (_i, [_i, _i, ctypes.POINTER(_vp)]),
    "lt_queue_push": (_i, [_vp, _i, _f, ctypes.POINTER(_i)]),
    "lt_queue_size": (_i, [_vp]),
    "lt_queue_destroy": (None, [_vp]),
    "lt_compact_kv": (_i, [_shp, _vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp]),
    "lt_dqueue_state_bytes": (ctypes.c_size_t, [_i, _i]),
    "lt_dqueue_init": (_i, [_vp, _i, _i, _i, _vp]),
    "lt_dqueue_push": (_i, [_vp, _i, _i, _i, _vp, _i, _vp]),
    "lt_dqueue_push_gathered": (_i, [_vp, _i, _i, _i, _vp, _i, _i, _vp]),
    "lt_dqueue_result": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp]),
    "lt_dqueue_error": (_i, [_vp, ctypes.POINTER(_i)]),
    "lt_compact_kv_pending": (_i, [_shp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "lt_compact_kv_layers": (_i, [_shp, _vp, _vp, _i, _vp, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "lt_kv_pool_commit": (_i, [_shp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "lt_dqueue_slots": (_i, [_vp, _i, _i, _vp, _vp]),
    "lt_stream_ring_init": (_i, [_vp, _vp, _i, _i, _i, _vp]),
    "lt_stream_append": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "lt_stream_decode": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _f, _vp]),
    "lt_decode_attn": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _f, _vp]),
    "lt_decode_splitk_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i]),
    "lt_decode_splitk_noalloc_capacity_bytes": (ctypes.c_size_t, []),
    "lt_decode_attn_splitk_noalloc": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _f, _vp]),
    "lt_decode_attn_splitk": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _f, _vp,
                                   ctypes.c_size_t, _vp]),
    "lt_device_status": (_i, [_i]),
    "lt_selftest_wait_timeout": (_i, [ctypes.c_uint, _vp]),
    "lt_status_string": (ctypes.c_char_p, [_i]),
    "lt_version": (_i, []),
}


def library_path() -> str:
    return LIB


def library():
    """The loaded ``liblt.so``; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB):
                raise RuntimeError(f"{LIB} is missing: build it with "
                                   "`python -m kv_cache_compression_tcgen05_b200.build`")
            lib = ctypes.CDLL(LIB)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def lt_status_string(status: int) -> str:
    return library().lt_status_string(int(status)).decode()


def lt_version() -> int:
    return library().lt_version()


def _check(status: int, where: str):
    if status != LT_OK:
        raise LtError(status, where)


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dev_tensor(t, name, dtype, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device; another GPU's memory is not its to read
        raise ValueError(f"{name} is on {t.device}, the current device is cuda:{torch.cuda.current_device()}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _sized(t, name, dtype, shape):
    """A caller's device tensor that must have exactly `shape` (the library indexes it so)."""
    _dev_tensor(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _shape(T, hq, hkv, d, cu_seqlens, max_seqlen):
    s = LtShape()
    s.total_tokens = int(T)
    s.hq = int(hq)
    s.hkv = int(hkv)
    s.head_dim = int(d)
    if cu_seqlens is None:
        s.batch = 1
        s.max_seqlen = int(T)
        s.cu_seqlens = None
    else:
        _dev_tensor(cu_seqlens, "cu_seqlens", torch.int32, 1)
        s.batch = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        s.max_seqlen = int(max_seqlen)
        s.cu_seqlens = cu_seqlens.data_ptr()
    return s


def lt_prefill_attn(Q, K, V, cu_seqlens=None, max_seqlen=None, softmax_scale=None, out=None, lse=None,
                    stream=None):
    """Causal GQA prefill attention.  Q [T, hq, d], K/V [T, hkv, d] bf16 (CUDA).
    Returns (O [T, hq, d] bf16, LSE [hq, T] fp32)."""
    _dev_tensor(Q, "Q", torch.bfloat16, 3)
    _dev_tensor(K, "K", torch.bfloat16, 3)
    _dev_tensor(V, "V", torch.bfloat16, 3)
    T, hq, d = Q.shape
    hkv = K.shape[1]
    if K.shape != (T, hkv, d) or V.shape != K.shape:
        raise ValueError("K and V must be [T, hkv, d] with Q's T and d")
    if out is None:
        out = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=Q.device)
    _dev_tensor(out, "out", torch.bfloat16, 3)
    _dev_tensor(lse, "lse", torch.float32, 2)
    if out.shape != Q.shape or lse.shape != (hq, T):
        raise ValueError("out must be [T, hq, d] and lse [hq, T]")
    shape = _shape(T, hq, hkv, d, cu_seqlens, max_seqlen)
    _check(library().lt_prefill_attn(ctypes.byref(shape), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                     out.data_ptr(), lse.data_ptr(),
                                     0.0 if softmax_scale is None else float(softmax_scale),
                                     _stream_handle(stream)), "lt_prefill_attn")
    return out, lse


def lt_prefill_attn_ratio(Q, K, V, S, W, n_obs, cu_seqlens=None, max_seqlen=None, softmax_scale=None, out=None,
                          lse=None, ratio=None, stream=None, accumulate=False):
    """Attention fused with the lazy ratio.  Returns (O [T, hq, d] bf16,
    LSE [hq, T] fp32, ratio [batch, hq] fp32).  accumulate=True adds into a
    ratio buffer the caller has zeroed (no zeroing launch)."""
    if accumulate and ratio is None:
        raise ValueError("accumulate=True needs a zeroed ratio buffer")
    _dev_tensor(Q, "Q", torch.bfloat16, 3)
    _dev_tensor(K, "K", torch.bfloat16, 3)
    _dev_tensor(V, "V", torch.bfloat16, 3)
    T, hq, d = Q.shape
    hkv = K.shape[1]
    if K.shape != (T, hkv, d) or V.shape != K.shape:
        raise ValueError("K and V must be [T, hkv, d] with Q's T and d")
    shape = _shape(T, hq, hkv, d, cu_seqlens, max_seqlen)
    if out is None:
        out = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=Q.device)
    if ratio is None:
        ratio = torch.empty((shape.batch, hq), dtype=torch.float32, device=Q.device)
    _dev_tensor(out, "out", torch.bfloat16, 3)
    _dev_tensor(lse, "lse", torch.float32, 2)
    _dev_tensor(ratio, "ratio", torch.float32, 2)
    if out.shape != Q.shape or lse.shape != (hq, T) or ratio.shape != (shape.batch, hq):
        raise ValueError("out must be [T, hq, d], lse [hq, T] and ratio [batch, hq]")
    fn = library().lt_prefill_attn_ratio_acc if accumulate else library().lt_prefill_attn_ratio
    _check(fn(ctypes.byref(shape), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                           out.data_ptr(), lse.data_ptr(),
                                           0.0 if softmax_scale is None else float(softmax_scale), int(S), int(W),
                                           int(n_obs), ratio.data_ptr(), _stream_handle(stream)),
           "lt_prefill_attn_ratio_acc" if accumulate else "lt_prefill_attn_ratio")
    return out, lse, ratio


def lt_prefill_attn_ratio_push(Q, K, V, S, W, n_obs, queue, layer, ratio, cu_seqlens=None, max_seqlen=None,
                               softmax_scale=None, out=None, lse=None, stream=None):
    """Attention fused with the lazy ratio and the device-queue push of `layer`
    (see include/lt.h): ratio [batch, hq] must be zero on entry; queue is a
    DeviceQueue.  Returns (O, LSE, ratio)."""
    _dev_tensor(Q, "Q", torch.bfloat16, 3)
    _dev_tensor(K, "K", torch.bfloat16, 3)
    _dev_tensor(V, "V", torch.bfloat16, 3)
    T, hq, d = Q.shape
    hkv = K.shape[1]
    if K.shape != (T, hkv, d) or V.shape != K.shape:
        raise ValueError("K and V must be [T, hkv, d] with Q's T and d")
    shape = _shape(T, hq, hkv, d, cu_seqlens, max_seqlen)
    if shape.batch != queue.batch:
        raise ValueError("batch differs from the queue's")
    if out is None:
        out = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty((hq, T), dtype=torch.float32, device=Q.device)
    _sized(out, "out", torch.bfloat16, (T, hq, d))
    _sized(lse, "lse", torch.float32, (hq, T))
    _sized(ratio, "ratio", torch.float32, (shape.batch, hq))
    _dev_tensor(queue.state, "state", torch.uint8, 1)
    _check(library().lt_prefill_attn_ratio_push(ctypes.byref(shape), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                                out.data_ptr(), lse.data_ptr(),
                                                0.0 if softmax_scale is None else float(softmax_scale), int(S),
                                                int(W), int(n_obs), ratio.data_ptr(), queue.state.data_ptr(),
                                                queue.L, int(layer), _stream_handle(stream)),
           "lt_prefill_attn_ratio_push")
    return out, lse, ratio


def lt_lazy_ratio(Q, K, LSE, S, W, n_obs, cu_seqlens=None, max_seqlen=None, softmax_scale=None, out=None,
                  stream=None):
    """Lazy ratio [batch, hq] fp32 from Q, K and the attention's LSE [hq, T]."""
    _dev_tensor(Q, "Q", torch.bfloat16, 3)
    _dev_tensor(K, "K", torch.bfloat16, 3)
    _dev_tensor(LSE, "LSE", torch.float32, 2)
    T, hq, d = Q.shape
    hkv = K.shape[1]
    if K.shape != (T, hkv, d) or LSE.shape != (hq, T):
        raise ValueError("K must be [T, hkv, d] and LSE [hq, T]")
    shape = _shape(T, hq, hkv, d, cu_seqlens, max_seqlen)
    if out is None:
        out = torch.empty((shape.batch, hq), dtype=torch.float32, device=Q.device)
    _dev_tensor(out, "out", torch.float32, 2)
    if out.shape != (shape.batch, hq):
        raise ValueError("out must be [batch, hq]")
    _check(library().lt_lazy_ratio(ctypes.byref(shape), Q.data_ptr(), K.data_ptr(), LSE.data_ptr(),
                                   0.0 if softmax_scale is None else float(softmax_scale), int(S), int(W),
                                   int(n_obs), out.data_ptr(), _stream_handle(stream)), "lt_lazy_ratio")
    return out


def lt_compact_kv(K, V, mask, S, W, cu_seqlens=None, max_seqlen=None, k_stream=None, v_stream=None,
                  stream_len=None, stream=None):
    """Streaming KV of the sequences with mask[b] != 0.
    Returns (K_stream, V_stream [batch, hkv, S+W, d] bf16, stream_len [batch] int32)."""
    _dev_tensor(K, "K", torch.bfloat16, 3)
    _dev_tensor(V, "V", torch.bfloat16, 3)
    _dev_tensor(mask, "mask", torch.uint8, 1)
    T, hkv, d = K.shape
    if V.shape != K.shape:
        raise ValueError("V must match K")
    shape = _shape(T, hkv, hkv, d, cu_seqlens, max_seqlen)
    if mask.numel() != shape.batch:
        raise ValueError("mask must have one entry per sequence")
    slots = int(S) + int(W)
    if k_stream is None:
        k_stream = torch.empty((shape.batch, hkv, slots, d), dtype=torch.bfloat16, device=K.device)
    if v_stream is None:
        v_stream = torch.empty((shape.batch, hkv, slots, d), dtype=torch.bfloat16, device=K.device)
    if stream_len is None:
        stream_len = torch.empty((shape.batch,), dtype=torch.int32, device=K.device)
    for t, n in ((k_stream, "k_stream"), (v_stream, "v_stream")):
        _dev_tensor(t, n, torch.bfloat16, 4)
        if t.shape != (shape.batch, hkv, slots, d):
            raise ValueError(f"{n} must be [batch, hkv, S+W, d]")
    _sized(stream_len, "stream_len", torch.int32, (shape.batch,))
    _check(library().lt_compact_kv(ctypes.byref(shape), K.data_ptr(), V.data_ptr(), mask.data_ptr(), int(S),
                                   int(W), k_stream.data_ptr(), v_stream.data_ptr(), stream_len.data_ptr(),
                                   _stream_handle(stream)), "lt_compact_kv")
    return k_stream, v_stream, stream_len


def _host_f32(x):
    a = x.detach().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x)
    return np.ascontiguousarray(a, dtype=np.float32)


def lt_layer_score(ratio_of_heads) -> float:
    r = _host_f32(ratio_of_heads).ravel()
    return float(library().lt_layer_score(r.ctypes.data, r.size))


def lt_select_layers(ratios, budget):
    """Offline selection.  ratios [L, batch, hq] (host); returns
    (lazy_mask [batch, L] uint8, order [batch, budget] int32) as numpy arrays."""
    r = _host_f32(ratios)
    if r.ndim != 3:
        raise ValueError("ratios must be [L, batch, hq]")
    L, B, H = r.shape
    lazy = np.empty((B, L), np.uint8)
    order = np.empty((B, max(int(budget), 1)), np.int32)
    _check(library().lt_select_layers(r.ctypes.data, L, B, H, int(budget), lazy.ctypes.data, order.ctypes.data),
           "lt_select_layers")
    return lazy, order[:, : int(budget)]


def lt_attn_schedule(head_dim, len, hq, hkv, grid, S=0, W=0, n_obs=0, fused=False):
    """The attention launch's work assignment for one sequence of `len` tokens
    on `grid` SMs (host-only).  Returns (num_items, None) when the launch keeps
    its round-robin or banded order, else (num_items, [items of CTA 0, items of
    CTA 1, ...]) with the item indices of each CTA in run order."""
    used, n = ctypes.c_int(0), ctypes.c_int(0)
    st = library().lt_attn_schedule(int(head_dim), 1 if fused else 0, int(len), int(hq), int(hkv), int(S), int(W),
                                    int(n_obs), int(grid), ctypes.byref(used), ctypes.byref(n), None, None, 0)
    if st == LT_ERR_INVALID_ARG and used.value == 1:
        off = np.empty(int(grid) + 1, np.int32)
        item = np.empty(max(n.value, 1), np.int32)
        st = library().lt_attn_schedule(int(head_dim), 1 if fused else 0, int(len), int(hq), int(hkv), int(S),
                                        int(W), int(n_obs), int(grid), ctypes.byref(used), ctypes.byref(n),
                                        off.ctypes.data, item.ctypes.data, item.size)
        _check(st, "lt_attn_schedule")
        g = min(int(grid), n.value)
        return n.value, [item[off[c]:off[c + 1]].tolist() for c in range(g)]
    _check(st, "lt_attn_schedule")
    return n.value, None


def lt_queue_create(L, budget):
    q = ctypes.c_void_p()
    _check(library().lt_queue_create(int(L), int(budget), ctypes.byref(q)), "lt_queue_create")
    return q


def lt_queue_push(q, layer, score) -> int:
    demoted = ctypes.c_int(-1)
    _check(library().lt_queue_push(q, int(layer), float(score), ctypes.byref(demoted)), "lt_queue_push")
    return demoted.value


def lt_queue_size(q) -> int:
    return library().lt_queue_size(q)


def lt_queue_destroy(q):
    library().lt_queue_destroy(q)


class LayerQueue:
    """Owning wrapper of one lt_queue (one sequence)."""

    def __init__(self, L, budget):
        self._q = lt_queue_create(L, budget)

    def push(self, layer, score) -> int:
        return lt_queue_push(self._q, layer, score)

    def __len__(self):
        return lt_queue_size(self._q)

    def close(self):
        if self._q is not None:
            lt_queue_destroy(self._q)
            self._q = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lt_device_status(clear: bool = True) -> int:
    """LT_OK or LT_ERR_TIMEOUT (synchronises the current device)."""
    return library().lt_device_status(1 if clear else 0)


def lt_selftest_wait_timeout(limit_us, stream=None):
    """Run the bounded-wait self-test kernel (see include/lt.h)."""
    _check(library().lt_selftest_wait_timeout(int(limit_us), _stream_handle(stream)), "lt_selftest_wait_timeout")


def lt_dqueue_state_bytes(L, batch) -> int:
    return int(library().lt_dqueue_state_bytes(int(L), int(batch)))


def lt_dqueue_init(state, L, budget, batch, stream=None):
    _dev_tensor(state, "state", torch.uint8, 1)
    if state.numel() < lt_dqueue_state_bytes(L, batch):
        raise ValueError("state is smaller than lt_dqueue_state_bytes(L, batch)")
    _check(library().lt_dqueue_init(state.data_ptr(), int(L), int(budget), int(batch), _stream_handle(stream)),
           "lt_dqueue_init")


def lt_dqueue_push(state, L, batch, layer, ratio, stream=None):
    _dev_tensor(state, "state", torch.uint8, 1)
    _dev_tensor(ratio, "ratio", torch.float32, 2)
    if ratio.shape[0] != batch:
        raise ValueError("ratio must be [batch, hq]")
    _check(library().lt_dqueue_push(state.data_ptr(), int(L), int(batch), int(layer), ratio.data_ptr(),
                                    int(ratio.shape[1]), _stream_handle(stream)), "lt_dqueue_push")


def lt_dqueue_push_gathered(state, L, batch, layer, gathered, stream=None):
    """Push of ratios gathered from head-sharded ranks: gathered is device fp32
    [shards, batch, hq_shard], shard n holding heads [n hq_shard, (n+1) hq_shard)."""
    _dev_tensor(state, "state", torch.uint8, 1)
    _dev_tensor(gathered, "gathered", torch.float32, 3)
    if gathered.shape[1] != batch:
        raise ValueError("gathered must be [shards, batch, hq_shard]")
    _check(library().lt_dqueue_push_gathered(state.data_ptr(), int(L), int(batch), int(layer), gathered.data_ptr(),
                                             int(gathered.shape[0]), int(gathered.shape[2]), _stream_handle(stream)),
           "lt_dqueue_push_gathered")


def lt_dqueue_result(state, L, batch, budget, lazy_mask=None, order=None, stream=None):
    _dev_tensor(state, "state", torch.uint8, 1)
    if lazy_mask is None:
        lazy_mask = torch.empty((batch, L), dtype=torch.uint8, device=state.device)
    if order is None:
        order = torch.empty((batch, max(int(budget), 1)), dtype=torch.int32, device=state.device)
    _sized(lazy_mask, "lazy_mask", torch.uint8, (batch, L))
    _sized(order, "order", torch.int32, (batch, max(int(budget), 1)))
    _check(library().lt_dqueue_result(state.data_ptr(), int(L), int(batch), int(budget), lazy_mask.data_ptr(),
                                      order.data_ptr(), _stream_handle(stream)), "lt_dqueue_result")
    return lazy_mask, order[:, : int(budget)]


def lt_dqueue_error(state) -> int:
    bits = ctypes.c_int(0)
    _check(library().lt_dqueue_error(state.data_ptr(), ctypes.byref(bits)), "lt_dqueue_error")
    return bits.value


class DeviceQueue:
    """Owning wrapper of one device-resident queue state for `batch` sequences."""

    def __init__(self, L, budget, batch, device="cuda", stream=None):
        self.L, self.budget, self.batch = int(L), int(budget), int(batch)
        self.state = torch.empty(lt_dqueue_state_bytes(L, batch), dtype=torch.uint8, device=device)
        lt_dqueue_init(self.state, L, budget, batch, stream)

    def reset(self, stream=None):
        lt_dqueue_init(self.state, self.L, self.budget, self.batch, stream)

    def push(self, layer, ratio, stream=None):
        lt_dqueue_push(self.state, self.L, self.batch, layer, ratio, stream)

    def push_gathered(self, layer, gathered, stream=None):
        lt_dqueue_push_gathered(self.state, self.L, self.batch, layer, gathered, stream)

    def result(self, stream=None):
        return lt_dqueue_result(self.state, self.L, self.batch, self.budget, stream=stream)

    def error(self) -> int:
        return lt_dqueue_error(self.state)

    def slots(self, stream=None):
        return lt_dqueue_slots(self.state, self.L, self.batch, stream=stream)


def layer_pointer_table(tensors, device="cuda"):
    """Device int64 array of the tensors' data pointers (for lt_compact_kv_pending)."""
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def lt_compact_kv_pending(K_layers, V_layers, queue, S, W, K_pool, V_pool, pool_len, total_tokens, hkv, d,
                          cu_seqlens=None, max_seqlen=None, stream=None):
    """Compaction of the layers the latest device-queue push demoted (see include/lt.h).
    K_layers / V_layers: device int64 pointer tables from layer_pointer_table."""
    for t, n in ((K_layers, "K_layers"), (V_layers, "V_layers")):
        _dev_tensor(t, n, torch.int64, 1)
        if t.numel() != queue.L:
            raise ValueError(f"{n} must hold L pointers")
    slots = int(S) + int(W)
    for t, n in ((K_pool, "K_pool"), (V_pool, "V_pool")):
        _dev_tensor(t, n, torch.bfloat16, 5)
        if t.shape != (queue.budget, queue.batch, hkv, slots, d):
            raise ValueError(f"{n} must be [budget, batch, hkv, S+W, d]")
    _sized(pool_len, "pool_len", torch.int32, (queue.budget, queue.batch))
    shape = _shape(total_tokens, hkv, hkv, d, cu_seqlens, max_seqlen)
    if shape.batch != queue.batch:
        raise ValueError("batch differs from the queue's")
    _check(library().lt_compact_kv_pending(ctypes.byref(shape), K_layers.data_ptr(), V_layers.data_ptr(),
                                           queue.state.data_ptr(), queue.L, queue.budget, int(S), int(W),
                                           K_pool.data_ptr(), V_pool.data_ptr(), pool_len.data_ptr(),
                                           _stream_handle(stream)), "lt_compact_kv_pending")


def lt_compact_kv_layers(K_layers, V_layers, layers, S, W, K_pool, V_pool, pool_len, total_tokens, hkv, d,
                         cu_seqlens=None, max_seqlen=None, stream=None):
    """Compaction of the layers listed in `layers` (device int32 [n]) into
    pool slots 0..n-1 in one launch (see include/lt.h).  K_layers / V_layers:
    device int64 pointer tables from layer_pointer_table."""
    for t, n in ((K_layers, "K_layers"), (V_layers, "V_layers")):
        _dev_tensor(t, n, torch.int64, 1)
    _dev_tensor(layers, "layers", torch.int32, 1)
    L, n = K_layers.numel(), layers.numel()
    if V_layers.numel() != L:
        raise ValueError("K_layers and V_layers must hold the same number of layers")
    slots = int(S) + int(W)
    shape = _shape(total_tokens, hkv, hkv, d, cu_seqlens, max_seqlen)
    for t, nm in ((K_pool, "K_pool"), (V_pool, "V_pool")):
        _dev_tensor(t, nm, torch.bfloat16, 5)
        if t.shape != (n, shape.batch, hkv, slots, d):
            raise ValueError(f"{nm} must be [n, batch, hkv, S+W, d]")
    _sized(pool_len, "pool_len", torch.int32, (n, shape.batch))
    _check(library().lt_compact_kv_layers(ctypes.byref(shape), K_layers.data_ptr(), V_layers.data_ptr(), L,
                                          layers.data_ptr(), n, int(S), int(W), K_pool.data_ptr(), V_pool.data_ptr(),
                                          pool_len.data_ptr(), _stream_handle(stream)), "lt_compact_kv_layers")


def lt_kv_pool_commit(K_cur, V_cur, queue, layer, S, W, K_full, V_full, K_stream, V_stream, stream_len,
                      cu_seqlens=None, max_seqlen=None, stream=None):
    """One layer of the memory-capped prefill after its push (see include/lt.h):
    the demoted layer's streaming rows into its streaming slot, the current
    layer's K/V (K_cur, V_cur [T, hkv, d]) into its full-KV slot.
    K_full / V_full [L - budget, T, hkv, d]; K_stream / V_stream
    [budget, batch, hkv, S+W, d]; stream_len [budget, batch]."""
    _dev_tensor(K_cur, "K_cur", torch.bfloat16, 3)
    _dev_tensor(V_cur, "V_cur", torch.bfloat16, 3)
    T, hkv, d = K_cur.shape
    if V_cur.shape != K_cur.shape:
        raise ValueError("V_cur must match K_cur")
    shape = _shape(T, hkv, hkv, d, cu_seqlens, max_seqlen)
    if shape.batch != queue.batch:
        raise ValueError("batch differs from the queue's")
    L, budget, B, slots = queue.L, queue.budget, queue.batch, int(S) + int(W)
    _sized(K_full, "K_full", torch.bfloat16, (L - budget, T, hkv, d))
    _sized(V_full, "V_full", torch.bfloat16, (L - budget, T, hkv, d))
    _sized(K_stream, "K_stream", torch.bfloat16, (budget, B, hkv, slots, d))
    _sized(V_stream, "V_stream", torch.bfloat16, (budget, B, hkv, slots, d))
    _sized(stream_len, "stream_len", torch.int32, (budget, B))
    _dev_tensor(queue.state, "state", torch.uint8, 1)
    _check(library().lt_kv_pool_commit(ctypes.byref(shape), K_cur.data_ptr(), V_cur.data_ptr(),
                                       queue.state.data_ptr(), L, budget, int(layer), int(S), int(W),
                                       K_full.data_ptr(), V_full.data_ptr(), K_stream.data_ptr(), V_stream.data_ptr(),
                                       stream_len.data_ptr(), _stream_handle(stream)), "lt_kv_pool_commit")


def lt_dqueue_slots(state, L, batch, out=None, stream=None):
    """Full-KV slot of every layer of every sequence: device int32 [batch, L] (-1: none)."""
    _dev_tensor(state, "state", torch.uint8, 1)
    if out is None:
        out = torch.empty((batch, L), dtype=torch.int32, device=state.device)
    _sized(out, "out", torch.int32, (batch, L))
    _check(library().lt_dqueue_slots(state.data_ptr(), int(L), int(batch), out.data_ptr(), _stream_handle(stream)),
           "lt_dqueue_slots")
    return out


def lt_stream_ring_init(stream_len, next_slot, S, W, stream=None):
    _dev_tensor(stream_len, "stream_len", torch.int32, 1)
    _sized(next_slot, "next_slot", torch.int32, (stream_len.numel(),))
    _check(library().lt_stream_ring_init(stream_len.data_ptr(), next_slot.data_ptr(), stream_len.numel(), int(S),
                                         int(W), _stream_handle(stream)), "lt_stream_ring_init")


def lt_stream_append(K_stream, V_stream, stream_len, next_slot, k_new, v_new, S, W, stream=None):
    """Append one token per sequence (k_new, v_new [batch, hkv, d]) to the streaming cache."""
    for t, n in ((K_stream, "K_stream"), (V_stream, "V_stream")):
        _dev_tensor(t, n, torch.bfloat16, 4)
    B, hkv, slots, d = K_stream.shape
    if slots != S + W or V_stream.shape != K_stream.shape:
        raise ValueError("caches must be [batch, hkv, S+W, d]")
    for t, n in ((k_new, "k_new"), (v_new, "v_new")):
        _dev_tensor(t, n, torch.bfloat16, 3)
        if t.shape != (B, hkv, d):
            raise ValueError(f"{n} must be [batch, hkv, d]")
    _sized(stream_len, "stream_len", torch.int32, (B,))
    _sized(next_slot, "next_slot", torch.int32, (B,))
    _check(library().lt_stream_append(K_stream.data_ptr(), V_stream.data_ptr(), stream_len.data_ptr(),
                                      next_slot.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), B, hkv, d, int(S),
                                      int(W), _stream_handle(stream)), "lt_stream_append")


def lt_stream_decode(q, K_stream, V_stream, stream_len, softmax_scale=None, out=None, lse=None, stream=None):
    """Decode attention over the streaming cache: q [batch, hq, d] -> (O [batch, hq, d], LSE [batch, hq])."""
    _dev_tensor(q, "q", torch.bfloat16, 3)
    for t, n in ((K_stream, "K_stream"), (V_stream, "V_stream")):
        _dev_tensor(t, n, torch.bfloat16, 4)
    B, hq, d = q.shape
    _, hkv, slots, dk = K_stream.shape
    if K_stream.shape[0] != B or dk != d or V_stream.shape != K_stream.shape:
        raise ValueError("caches must be [batch, hkv, S+W, d] with q's batch and d")
    _sized(stream_len, "stream_len", torch.int32, (B,))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    _sized(out, "out", torch.bfloat16, (B, hq, d))
    _sized(lse, "lse", torch.float32, (B, hq))
    _check(library().lt_stream_decode(q.data_ptr(), K_stream.data_ptr(), V_stream.data_ptr(), stream_len.data_ptr(),
                                      B, hq, hkv, d, slots, out.data_ptr(), lse.data_ptr(),
                                      0.0 if softmax_scale is None else float(softmax_scale), _stream_handle(stream)),
           "lt_stream_decode")
    return out, lse


def _decode_full_args(q, K, V, seq_len, seq_start, max_len, out, lse):
    """Checked arguments of a decode over a full cache (shared by the cluster
    and split-K calls): (q, K, V, seq_start, capacity, len, B, hq, hkv, d,
    max_len, out, lse)."""
    _dev_tensor(q, "q", torch.bfloat16, 3)
    B, hq, d = q.shape
    if K.dim() == 4:
        for t, n in ((K, "K"), (V, "V")):
            _dev_tensor(t, n, torch.bfloat16, 4)
        if seq_start is not None:
            raise ValueError("a padded [batch, capacity, hkv, d] cache takes no seq_start")
        Bk, cap, hkv, dk = K.shape
        if Bk != B:
            raise ValueError("padded cache batch differs from q's")
        limit = cap if max_len is None else int(max_len)
    else:
        for t, n in ((K, "K"), (V, "V")):
            _dev_tensor(t, n, torch.bfloat16, 3)
        if seq_start is None:
            raise ValueError("a packed [rows, hkv, d] cache needs seq_start")
        _dev_tensor(seq_start, "seq_start", torch.int32, 1)
        rows, hkv, dk = K.shape
        cap = 0
        limit = rows if max_len is None else int(max_len)
    if dk != d or V.shape != K.shape:
        raise ValueError("K and V must have the same shape and q's head dim")
    _sized(seq_len, "seq_len", torch.int32, (B,))
    if seq_start is not None:
        _sized(seq_start, "seq_start", torch.int32, (B,))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    _sized(out, "out", torch.bfloat16, (B, hq, d))
    _sized(lse, "lse", torch.float32, (B, hq))
    return q, K, V, seq_start, cap, seq_len, B, hq, hkv, d, limit, out, lse


def lt_decode_attn(q, K, V, seq_len, seq_start=None, max_len=None, softmax_scale=None, out=None, lse=None,
                   stream=None):
    """Decode attention over a kept layer's full cache: q [batch, hq, d] ->
    (O [batch, hq, d], LSE [batch, hq]).  K/V either token-major packed
    [rows, hkv, d] with seq_start (device int32 [batch], first row of each
    sequence), or padded [batch, capacity, hkv, d] with seq_start None.
    seq_len: device int32 [batch] positions attended."""
    q, K, V, seq_start, cap, seq_len, B, hq, hkv, d, limit, out, lse = _decode_full_args(
        q, K, V, seq_len, seq_start, max_len, out, lse)
    _check(library().lt_decode_attn(q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                    None if seq_start is None else seq_start.data_ptr(), cap, seq_len.data_ptr(), B,
                                    hq, hkv, d, limit, out.data_ptr(), lse.data_ptr(),
                                    0.0 if softmax_scale is None else float(softmax_scale), _stream_handle(stream)),
           "lt_decode_attn")
    return out, lse


def lt_decode_splitk_workspace_bytes(batch, hq, head_dim, max_len) -> int:
    return int(library().lt_decode_splitk_workspace_bytes(int(batch), int(hq), int(head_dim), int(max_len)))


def lt_decode_attn_splitk(q, K, V, seq_len, seq_start=None, max_len=None, softmax_scale=None, out=None, lse=None,
                          workspace=None, stream=None):
    """lt_decode_attn for long caches, split over many CTAs with a workspace
    (device uint8 tensor of at least lt_decode_splitk_workspace_bytes bytes;
    allocated here when None).  Same arguments and results otherwise."""
    q, K, V, seq_start, cap, seq_len, B, hq, hkv, d, limit, out, lse = _decode_full_args(
        q, K, V, seq_len, seq_start, max_len, out, lse)
    need = lt_decode_splitk_workspace_bytes(B, hq, d, limit)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _dev_tensor(workspace, "workspace", torch.uint8, 1)
    _check(library().lt_decode_attn_splitk(q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                           None if seq_start is None else seq_start.data_ptr(), cap,
                                           seq_len.data_ptr(), B, hq, hkv, d, limit, out.data_ptr(), lse.data_ptr(),
                                           0.0 if softmax_scale is None else float(softmax_scale),
                                           workspace.data_ptr(), workspace.numel(), _stream_handle(stream)),
           "lt_decode_attn_splitk")
    return out, lse


def lt_decode_splitk_noalloc_capacity_bytes() -> int:
    return int(library().lt_decode_splitk_noalloc_capacity_bytes())


def lt_decode_attn_splitk_noalloc(q, K, V, seq_len, seq_start=None, max_len=None, softmax_scale=None, out=None,
                                  lse=None, stream=None):
    """lt_decode_attn_splitk with the library's fixed workspace instead of one
    the caller allocates (see include/lt.h): for callers that cannot allocate
    device memory at decode time.  Raises ValueError, before any launch, when
    the call's workspace would exceed the fixed capacity."""
    q, K, V, seq_start, cap, seq_len, B, hq, hkv, d, limit, out, lse = _decode_full_args(
        q, K, V, seq_len, seq_start, max_len, out, lse)
    need, have = lt_decode_splitk_workspace_bytes(B, hq, d, limit), lt_decode_splitk_noalloc_capacity_bytes()
    if need > have:
        raise ValueError(f"split-K decode of batch {B}, {hq} heads, head_dim {d}, {limit} rows needs {need} bytes "
                         f"of workspace; the allocation-free entry point holds {have}")
    _check(library().lt_decode_attn_splitk_noalloc(q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                                   None if seq_start is None else seq_start.data_ptr(), cap,
                                                   seq_len.data_ptr(), B, hq, hkv, d, limit, out.data_ptr(),
                                                   lse.data_ptr(), 0.0 if softmax_scale is None else
                                                   float(softmax_scale), _stream_handle(stream)),
           "lt_decode_attn_splitk_noalloc")
    return out, lse

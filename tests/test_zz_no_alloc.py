"""The allocation-free split-K decode, lt_decode_attn_splitk_noalloc.

Some callers cannot allocate device memory when they decode: a plugin whose
host framework owns all of the GPU's memory, or a serving loop in which
cudaMalloc's implicit synchronisation is not allowed.  For them the library
keeps the split-K decode's partial states in a fixed array of its own device
memory instead of a workspace the caller allocates.  Checked here through the
C ABI: two calls in a row (different sizes and inputs; the array keeps the
first call's contents) against lt_decode_attn_splitk with a caller workspace,
within the decode tolerances of the other tests, and a size beyond the array
rejected before anything is launched.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_compression_tcgen05_b200 as lt
from tests.gpu_common import LSE_ABS, O_REL_L2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lt.library()
    yield
    assert lt.lt_device_status(True) == lt.LT_OK


def _inputs(B, cap, hq, hkv, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, hq, d), generator=g, device="cuda").bfloat16()
    K = (torch.randn((B, cap, hkv, d), generator=g, device="cuda") * 1.2).bfloat16()
    V = torch.randn((B, cap, hkv, d), generator=g, device="cuda").bfloat16()
    lens = torch.tensor([cap, cap // 3, 1, 0][:B], dtype=torch.int32, device="cuda")
    return q, K, V, lens


def _noalloc_c(q, K, V, lens):
    """The new entry point called through the C ABI (padded cache, no seq_start)."""
    B, hq, d = q.shape
    _, cap, hkv, _ = K.shape
    O = torch.empty_like(q)
    LSE = torch.empty((B, hq), dtype=torch.float32, device="cuda")
    rc = lt.library().lt_decode_attn_splitk_noalloc(
        q.data_ptr(), K.data_ptr(), V.data_ptr(), None, cap, lens.data_ptr(), B, hq, hkv, d, cap, O.data_ptr(),
        LSE.data_ptr(), 0.0, torch.cuda.current_stream().cuda_stream)
    return rc, O, LSE


def _close(O, L, O_ref, L_ref):
    lr, l = L_ref.cpu().numpy().astype(np.float64), L.cpu().numpy().astype(np.float64)
    finite = np.isfinite(lr)
    assert np.array_equal(np.isfinite(l), finite)
    assert np.abs(l[finite] - lr[finite]).max() <= LSE_ABS
    o, orf = O.float().cpu(), O_ref.float().cpu()
    assert ((o - orf).norm() / max(orf.norm().item(), 1e-30)).item() <= O_REL_L2


def test_noalloc_decode_equals_workspace_decode_on_two_calls_in_a_row():
    cases = [(2, 40000, 32, 8, 128, 1), (3, 5000, 8, 2, 64, 2)]
    for B, cap, hq, hkv, d, seed in cases:
        q, K, V, lens = _inputs(B, cap, hq, hkv, d, seed)
        assert lt.lt_decode_splitk_workspace_bytes(B, hq, d, cap) <= lt.lt_decode_splitk_noalloc_capacity_bytes()
        O_ref, L_ref = lt.lt_decode_attn_splitk(q, K, V, lens)      # the entry point with a caller workspace
        rc, O, L = _noalloc_c(q, K, V, lens)
        torch.cuda.synchronize()
        assert rc == lt.LT_OK
        _close(O, L, O_ref, L_ref)


def test_noalloc_decode_rejects_sizes_beyond_its_array():
    cap_bytes = lt.lt_decode_splitk_noalloc_capacity_bytes()
    B, hq, d, rows = 8, 64, 128, 131072          # 8 * 64 * 128 splits * 130 floats: beyond 4 MiB
    assert lt.lt_decode_splitk_workspace_bytes(B, hq, d, rows) > cap_bytes
    fake = ctypes.c_void_p(256)                  # never dereferenced: the size check comes first
    rc = lt.library().lt_decode_attn_splitk_noalloc(fake, fake, fake, None, rows, fake, B, hq, 8, d, rows, fake, fake,
                                                    0.0, None)
    assert rc == lt.LT_ERR_INVALID_ARG
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((B, 16, 8, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        lt.lt_decode_attn_splitk_noalloc(q, K, K, torch.ones(B, dtype=torch.int32, device="cuda"), max_len=rows)

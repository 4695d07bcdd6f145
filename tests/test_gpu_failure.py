"""Failure detection on the GPU without a fault: a kernel's bounded wait on an
mbarrier that nothing arrives on gives up, the device status word reports it,
and the context keeps working."""
import numpy as np
import pytest
import torch

import kv_cache_compression_tcgen05_b200 as lt
import synth
from tests.gpu_common import LSE_ABS, O_REL_L2, check_attention, gpu_attention

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lt.library()
    assert lt.lt_device_status(True) == lt.LT_OK
    yield
    lt.lt_device_status(True)


def test_bounded_wait_reports_timeout_and_context_survives():
    lt.lt_selftest_wait_timeout(50_000)            # 50 ms limit
    assert lt.lt_device_status(True) == lt.LT_ERR_TIMEOUT
    assert lt.lt_device_status(True) == lt.LT_OK   # cleared
    cfg = synth.CONFIGS["tiny"]
    Q, K, V = synth.layer_inputs(cfg, 0, "cuda")
    O, LSE = gpu_attention(cfg, Q, K, V)
    torch.cuda.synchronize()
    rel, lse_err = check_attention(cfg, Q, K, V, O, LSE)
    assert rel <= O_REL_L2 and lse_err <= LSE_ABS
    assert lt.lt_device_status(True) == lt.LT_OK


def test_selftest_rejects_bad_limits():
    for bad in (0, 10_000_001):
        with pytest.raises(lt.LtError):
            lt.lt_selftest_wait_timeout(bad)

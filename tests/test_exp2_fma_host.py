"""Host check of the FMA-pipe exp2 used by the attention softmax: the cubic's
constants are read from the device header and the same float32 steps are
replayed with numpy against 2^x (no GPU needed)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "kv_cache_compression_tcgen05_b200", "csrc", "lt_device.cuh")


def constants():
    text = open(HDR).read()
    body = text[text.index("float exp2_fma("):]
    vals = dict(re.findall(r"(kC\d) = ([0-9.eE+-]+)f", body))
    return [np.float32(vals[f"kC{i}"]) for i in range(4)]


def exp2_fma_replay(x):
    c0, c1, c2, c3 = constants()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    n_bits = (t.view(np.uint32) << np.uint32(23)).astype(np.uint32)
    f = (x - (t - shift)).astype(np.float32)
    p = np.float32(c3)
    for c in (c2, c1, c0):
        p = (p * f + c).astype(np.float32)
    return (p.view(np.uint32) + n_bits).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-100.0, 8.0, 2_000_001).astype(np.float32)
    got = exp2_fma_replay(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()


def test_underflow_and_masked_inputs():
    x = np.array([-np.inf, -1e30, -200.0, -126.0], np.float32)
    y = exp2_fma_replay(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 1e-37)


def test_integers_are_near_exact():
    x = np.arange(-60, 9, dtype=np.float32)
    rel = np.abs(exp2_fma_replay(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1e-4

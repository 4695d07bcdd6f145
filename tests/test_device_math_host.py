"""The softmax's FMA-pipe exponential (`exp2_fma` in csrc/lt_device.cuh),
emulated step by step in IEEE float32 on the host with the coefficients read
from that source file: relative error below 8e-5 against 2^x over the
softmax's input range [-125, 0] (the bound the kernel's comment states, well
under the 2^-9 rounding of P to bf16), and a result that stands for 0 below it.
A fused multiply-add is emulated as an exact product and sum in float64
rounded once to float32."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "kv_cache_compression_tcgen05_b200", "csrc", "lt_device.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("float exp2_fma(float x)"):]
    body = body[: body.index("\n}")]
    vals = [float(v) for v in re.findall(r"(-?\d+\.\d*)f", body)]
    # clamp, 1.5 * 2^23 twice, then the cubic's four coefficients, highest degree first
    assert vals[0] == -126.0 and vals[1] == vals[2] == 12582912.0 and len(vals) == 7
    return [np.float32(v) for v in vals[3:]]


def exp2_fma(x):
    c3, c2, c1, c0 = _coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    p = (np.float64(c3) * f.astype(np.float64) + np.float64(c2)).astype(np.float32)
    p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c1)).astype(np.float32)
    p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c0)).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_on_the_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 0.0, 2_000_001, dtype=np.float64),
                        np.arange(-125, 1, dtype=np.float64) + 0.5,      # the reduction's seams
                        np.arange(-125, 1, dtype=np.float64)]).astype(np.float32)
    got = exp2_fma(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 8e-5, float(rel.max())


def test_reduction_keeps_f_within_half_and_integer_inputs_near_exact():
    x = np.arange(-125, 1, dtype=np.float32)
    got = exp2_fma(x).astype(np.float64)
    # at integer x the cubic is evaluated at f = 0: 2^x times the constant term
    assert np.allclose(got / np.exp2(x.astype(np.float64)), float(_coefficients()[3]), rtol=0, atol=1e-7)


def test_inputs_below_the_clamp_give_a_negligible_result():
    x = np.array([-126.0, -130.0, -1e4, -np.inf], dtype=np.float32)
    got = exp2_fma(x).astype(np.float64)
    assert np.all(np.isfinite(got)) and np.all(np.abs(got) < 2.0 ** -124)

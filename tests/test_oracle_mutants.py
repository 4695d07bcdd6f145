"""Plants plausible mistakes in a copy of the oracle and checks that the pins
catch each one (the mistakes live only in a temporary copy, on the CPU)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import oracle_pins

# (name, text in oracle.c, replacement): a dropped term, a wrong sign or index,
# a transposed operand, an off-by-one in a window, a wrong comparison.
MUTANTS = [
    ("scale dropped", "return p->scale * acc;", "return acc;"),
    ("gqa modulo mapping", "const int kh = h / (p->hq / p->hkv);\n  const uint16_t* q", "const int kh = h % p->hkv;\n  const uint16_t* q"),
    ("query/key token swapped", "p->Q + ((size_t)tq * p->hq + h)", "p->Q + ((size_t)tk * p->hq + h)"),
    ("diagonal key dropped", "for (int64_t j = 0; j <= i; ++j) {\n    s[j] = score", "for (int64_t j = 0; j < i; ++j) {\n    s[j] = score"),
    ("max dropped from LSE", "return m + log(sum);", "return log(sum);"),
    ("output weight sign", "const double w = exp(s[j] - lse);", "const double w = exp(lse - s[j]);"),
    ("value of wrong head", "p->V + ((size_t)(start + j) * p->hkv + kh) * p->d;\n    for (int ch", "p->V + ((size_t)(start + j) * p->hkv + h % p->hkv) * p->d;\n    for (int ch"),
    ("value ignores sequence start", "p->V + ((size_t)(start + j) * p->hkv", "p->V + ((size_t)(j) * p->hkv"),
    ("window one short", "return j >= i - (int64_t)W + 1;", "return j >= i - (int64_t)W + 2;"),
    ("window one long", "return j >= i - (int64_t)W + 1;", "return j >= i - (int64_t)W;"),
    ("sink one long", "if (j < S) return 1;", "if (j <= S) return 1;"),
    ("ratio ignores LSE", "r += exp(score(p, t, h, start + j) - lse);", "r += exp(score(p, t, h, start + j));"),
    ("ratio mean over n_obs", "ratio[(size_t)b * hq + h] = nb > 0 ? sum / (double)nb : 0.0;", "ratio[(size_t)b * hq + h] = nb > 0 ? sum / (double)n_obs : 0.0;"),
    ("observed rows from the front", "tokens[k] = (int32_t)(cu_seqlens[b + 1] - nb + x);", "tokens[k] = (int32_t)(cu_seqlens[b] + x);"),
    ("layer score sums heads", "scores[(size_t)b * L + l] = sum / (double)hq;", "scores[(size_t)b * L + l] = sum;"),
    ("queue pops the minimum", "if (sa != sb) return sa > sb;", "if (sa != sb) return sa < sb;"),
    ("queue tie-break reversed", "return a < b;\n}", "return a > b;\n}"),
    ("queue capacity off by one", "while (size > cap) {", "while (size > cap + 1) {"),
    ("compaction window one short", "const int recent = pos >= N - W && pos >= S;", "const int recent = pos > N - W && pos >= S;"),
    ("compaction keeps no sinks", "const int sink = pos < S;", "const int sink = 0;"),
    ("compaction tail not zeroed", "memset(Ks + dst, 0, sizeof(uint16_t) * (size_t)d);", ";"),
    ("keyed attention drops scale", "s[j] = scale * acc;", "s[j] = acc;"),
    ("keyed attention skips last key", "for (int j = 0; j < mk; ++j) sum += exp(s[j] - mx);", "for (int j = 0; j + 1 < mk; ++j) sum += exp(s[j] - mx);"),
    ("keyed attention wrong value row", "const uint16_t* vr = V + ((size_t)it * m_max + j) * d;", "const uint16_t* vr = V + ((size_t)it * m_max) * d;"),
]


def _build_mutant(tmp_path, find, repl):
    src = open(oracle._SRC).read()
    assert src.count(find) >= 1, f"mutation anchor not found: {find!r}"
    mutated = src.replace(find, repl, 1)
    c = tmp_path / "mutant.c"
    so = tmp_path / "libmutant.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", str(c), "-o", str(so), "-lm", "-lpthread"])
    return str(so)


@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, find, repl):
    so = _build_mutant(tmp_path, find, repl)
    real = oracle._load()
    oracle._lib = oracle._configure(ctypes.CDLL(so))
    caught = []
    try:
        # a mutant may produce inf/NaN (e.g. a row left with no keys); the pins
        # still fail on it, and numpy's warnings about that arithmetic are noise
        with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
            for pin in oracle_pins.ALL_PINS + [_tiny_selection_pin]:
                try:
                    pin()
                except (AssertionError, ValueError, IndexError, FloatingPointError):
                    caught.append(pin.__name__)
    finally:
        oracle._lib = real
    assert caught, f"no pin catches the mutant '{name}'"


def _tiny_selection_pin():
    from tests.test_oracle_pins import test_tiny_designed_selection
    test_tiny_designed_selection()

"""The fp64 oracle against closed forms, invariants, scipy and brute force."""
import pytest

from tests import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_tiny_designed_selection():
    """The tiny workload gives layers 1 and 3 a strong sink bias; with a budget
    of 2 of 4 layers both the offline sort and the online queue demote exactly
    those two."""
    import numpy as np
    import oracle
    import synth

    cfg = synth.CONFIGS["tiny"]
    cu = np.array(cfg.cu_seqlens(), np.int32)
    ratios = []
    for layer in range(cfg.layers):
        Q, K, _ = synth.layer_inputs(cfg, layer)
        ratios.append(oracle.lazy_ratio(cu, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, cfg.n_obs))
    scores = oracle.layer_scores(np.stack(ratios))[0]
    lazy, order = oracle.select_layers(scores, cfg.budget)
    assert sorted(order.tolist()) == [1, 3]
    assert sorted(oracle.queue_online(scores, cfg.budget).tolist()) == [1, 3]


def test_golden_fixture_is_current():
    """The stored tiny fixture still equals what the oracle computes."""
    import json
    import os

    import numpy as np
    import oracle
    import synth

    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")
    gold = json.load(open(path))
    cfg = synth.CONFIGS["tiny"]
    cu = np.array(cfg.cu_seqlens(), np.int32)
    Q, K, _ = synth.layer_inputs(cfg, 1)
    r = oracle.lazy_ratio(cu, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, cfg.n_obs)
    assert np.allclose(r, gold["ratio"][1], atol=1e-12)
    assert gold["lazy_layers"] == gold["designed_lazy_layers"] == [1, 3]

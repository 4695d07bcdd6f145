"""Writes tests/golden/tiny_oracle.json from the fp64 oracle alone.

The pages print no worked example (no LSE, ratio or selection values survive in
them), so the stored values here come from the oracle on the tiny synthetic
workload: 4 layers, one 256-token sequence, 2 query heads / 1 KV head, d = 64,
S = 4, W = 32, n_obs = 16, budget 2; layers 1 and 3 carry a sink bias of 4u.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    cfg = synth.CONFIGS["tiny"]
    cu = np.array(cfg.cu_seqlens(), np.int32)
    ratios, lse_rows = [], []
    for layer in range(cfg.layers):
        Q, K, V = synth.layer_inputs(cfg, layer)
        q, k, v = synth.bf16_bits(Q), synth.bf16_bits(K), synth.bf16_bits(V)
        ratios.append(oracle.lazy_ratio(cu, q, k, cfg.S, cfg.W, cfg.n_obs))
        _, lse = oracle.attn(cu, q, k, v)
        lse_rows.append(lse[:, [0, 1, 127, 128, 255]].tolist())
    ratios = np.stack(ratios)
    scores = oracle.layer_scores(ratios)[0]
    lazy, order = oracle.select_layers(scores, cfg.budget)
    out = {
        "workload": "tiny: 4 layers, 1 x 256 tokens, hq=2, hkv=1, d=64, S=4, W=32, n_obs=16, budget=2",
        "source": "fp64 oracle (oracle/oracle.c) on synth.CONFIGS['tiny']",
        "ratio": ratios.tolist(),
        "layer_scores": scores.tolist(),
        "lse_rows_0_1_127_128_255": lse_rows,
        "lazy_layers": sorted(order.tolist()),
        "designed_lazy_layers": list(cfg.lazy_layers),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()

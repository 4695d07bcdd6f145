"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
binding and compare with the fp64 oracle on the same bf16 inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import kv_cache_compression_tcgen05_b200 as lt
import oracle
import synth

# Tolerances of the parity bar.
O_REL_L2 = 1e-2      # output: relative L2 error over all checked rows of a layer
LSE_ABS = 2e-3       # LSE: absolute error
RATIO_ABS = 2e-3     # lazy ratio: absolute error


def cu_tensor(cfg, device="cuda"):
    return torch.tensor(cfg.cu_seqlens(), dtype=torch.int32, device=device)


def gpu_attention(cfg, Q, K, V):
    cu = cu_tensor(cfg) if cfg.batch > 1 else None
    return lt.lt_prefill_attn(Q, K, V, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)


def gpu_fused(cfg, Q, K, V):
    cu = cu_tensor(cfg) if cfg.batch > 1 else None
    return lt.lt_prefill_attn_ratio(Q, K, V, cfg.S, cfg.W, cfg.n_obs, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)


def gpu_ratio(cfg, Q, K, LSE):
    cu = cu_tensor(cfg) if cfg.batch > 1 else None
    return lt.lt_lazy_ratio(Q, K, LSE, cfg.S, cfg.W, cfg.n_obs, cu_seqlens=cu, max_seqlen=cfg.max_seqlen)


def check_attention(cfg, Q, K, V, O, LSE, tokens=None, heads=None, nthreads=None):
    """Compare the listed rows (all rows when tokens is None) with the oracle.
    Returns (relative L2 error of O, max abs error of LSE)."""
    cu = np.array(cfg.cu_seqlens(), np.int32)
    q, k, v = synth.bf16_bits(Q), synth.bf16_bits(K), synth.bf16_bits(V)
    o_gpu = O.float().cpu().numpy().astype(np.float64)
    lse_gpu = LSE.cpu().numpy().astype(np.float64)
    if tokens is None:
        o_ref, lse_ref = oracle.attn(cu, q, k, v, nthreads=nthreads)
        o_got, lse_got = o_gpu, lse_gpu
    else:
        o_ref, lse_ref = oracle.attn(cu, q, k, v, tokens=tokens, heads=heads, nthreads=nthreads)
        o_got = o_gpu[tokens, heads]
        lse_got = lse_gpu[heads, tokens]
    rel = float(np.linalg.norm(o_got - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    lse_err = float(np.abs(lse_got - lse_ref).max()) if lse_ref.size else 0.0
    return rel, lse_err


def sample_rows(cfg, n_random, seed, last_rows=128, heads_for_last=4):
    """Rows to check at full size: the last `last_rows` rows of every sequence
    (the observed rows and a ragged q-tile) for a few heads, the first rows,
    and `n_random` random (token, head) pairs."""
    rng = np.random.default_rng(seed)
    cu = cfg.cu_seqlens()
    toks, hds = [], []
    for b in range(cfg.batch):
        lo = max(cu[b], cu[b + 1] - last_rows)
        for h in rng.choice(cfg.hq, size=min(heads_for_last, cfg.hq), replace=False):
            toks += list(range(lo, cu[b + 1]))
            hds += [int(h)] * (cu[b + 1] - lo)
        toks += [cu[b], min(cu[b] + 1, cu[b + 1] - 1)]
        hds += [0, cfg.hq - 1]
    T = cfg.total_tokens
    toks += rng.integers(0, T, n_random).tolist()
    hds += rng.integers(0, cfg.hq, n_random).tolist()
    return np.array(toks, np.int32), np.array(hds, np.int32)


def oracle_ratio(cfg, Q, K, lse=None, nthreads=None):
    cu = np.array(cfg.cu_seqlens(), np.int32)
    return oracle.lazy_ratio(cu, synth.bf16_bits(Q), synth.bf16_bits(K), cfg.S, cfg.W, cfg.n_obs, lse=lse,
                             nthreads=nthreads)


def expected_uniform_ratio(cfg):
    """Closed form of the ratio when every query is zero: the mean over the last
    min(n_obs, N) rows of min(S+W, i+1) / (i+1)."""
    out = []
    for n in cfg.seqlens:
        nb = min(cfg.n_obs, n)
        rows = np.arange(n - nb, n, dtype=np.float64)
        out.append(float(np.mean(np.minimum(cfg.S + cfg.W, rows + 1) / (rows + 1))) if nb else 0.0)
    return np.array(out)


def scale_of(cfg):
    return 1.0 / math.sqrt(cfg.d)

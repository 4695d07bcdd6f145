"""Host logic of the attention launch's static work schedule (no GPU needed).

lt_attn_schedule returns the assignment of work items to CTAs that
lt_prefill_attn / lt_prefill_attn_ratio compute on the host for a single
sequence.  The checks: the assignment is a partition of the items, each CTA runs
its items heaviest first, it is used only where it lowers the slowest CTA's work
below the round-robin (snake) order's, and long or tiny launches keep their own
orders.  The item costs are restated here from the kernels' item numbering: an
item is two 128-row query tiles on one K/V stream (two heads of a KV group on
the same q-tile when the group is even, else q-tiles 2p+1 and 2p of one head,
heaviest first), costing its key tiles (the two tiles run side by side) plus one
tile of fixed work, and with the fused ratio two more tiles per key tile that
holds a sink or an observed row's first window key.
"""
import ctypes

import numpy as np
import pytest

import kv_cache_compression_tcgen05_b200 as lt
from kv_cache_compression_tcgen05_b200.binding import LT_ERR_INVALID_ARG, library


def masked_tiles(qt, n, S, W, n_obs):
    obs_lo = n - min(n_obs, n)
    r0, r1 = max(qt * 128, obs_lo), min(n, qt * 128 + 128) - 1
    if r0 > r1:
        return 0
    tiles = set(range(min((S + 127) // 128, qt + 1)))
    for i in range(r0, r1 + 1):
        w = i - W + 1
        if w > 0 and w % 128 != 0 and (w // 128) * 128 >= S:
            tiles.add(w // 128)
    return len(tiles)


def item_costs(n, hq, hkv, fused, S, W, n_obs):
    """Cost of every item in quarter key-tile units, in the kernels' numbering."""
    nq = (n + 127) // 128
    g = hq // hkv
    mw = 8 if fused else 0
    costs = []
    if g % 2 == 0:
        for t in range(nq * (hq // 2)):
            qt = nq - 1 - t // (hq // 2)
            costs.append(4 * (qt + 1) + 4 + mw * masked_tiles(qt, n, S, W, n_obs))
    else:
        npairs = (nq + 1) // 2
        for t in range(npairs * hq):
            qp = npairs - 1 - t // hq
            t1, t0 = 2 * qp + 1, 2 * qp
            if t1 * 128 < n:
                c = 4 + 2 * (t1 + 1 + t0 + 1) + mw * (masked_tiles(t0, n, S, W, n_obs) + masked_tiles(t1, n, S, W, n_obs))
            else:
                c = 4 + 4 * (t0 + 1) + mw * masked_tiles(t0, n, S, W, n_obs)
            costs.append(c)
    return costs


def snake_max(costs, grid):
    n = len(costs)
    loads = [0] * grid
    for r in range((n + grid - 1) // grid):
        for c in range(grid):
            t = r * grid + ((grid - 1 - c) if r & 1 else c)
            if t < n:
                loads[c] += costs[t]
    return max(loads)


CASES = [
    dict(d=64, n=4096, hq=32, hkv=8, fused=True, S=4, W=1020, n_obs=64),      # the gqa1p2b layer
    dict(d=128, n=4096, hq=32, hkv=8, fused=True, S=4, W=1020, n_obs=64),
    dict(d=64, n=8000, hq=12, hkv=4, fused=True, S=4, W=700, n_obs=100),      # odd group, ragged tail
    dict(d=128, n=5000, hq=16, hkv=4, fused=True, S=4, W=1500, n_obs=128),
    dict(d=64, n=3000, hq=24, hkv=8, fused=True, S=0, W=1, n_obs=128),        # g = 3
    dict(d=128, n=2500, hq=16, hkv=2, fused=False, S=0, W=0, n_obs=0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"d{c['d']}-n{c['n']}-{c['hq']}x{c['hkv']}-{'fused' if c['fused'] else 'plain'}")
def test_static_schedule_partitions_and_balances(case):
    grid = 148
    n_items, sched = lt.lt_attn_schedule(case["d"], case["n"], case["hq"], case["hkv"], grid, S=case["S"],
                                         W=case["W"], n_obs=case["n_obs"], fused=case["fused"])
    costs = item_costs(case["n"], case["hq"], case["hkv"], case["fused"], case["S"], case["W"], case["n_obs"])
    assert n_items == len(costs)
    if sched is None:
        return     # the launch keeps the snake order (its slowest CTA was no heavier)
    g = min(grid, n_items)
    assert len(sched) == g
    flat = [t for cta in sched for t in cta]
    assert sorted(flat) == list(range(n_items))                      # every item exactly once
    for cta in sched:
        cs = [costs[t] for t in cta]
        assert cs == sorted(cs, reverse=True)                         # heaviest first
    loads = [sum(costs[t] for t in cta) for cta in sched]
    assert max(loads) < snake_max(costs, g)                           # used only where it helps
    # A longest-first greedy stays within the heaviest item of the mean load.
    assert max(loads) <= sum(costs) / g + max(costs)


def test_gqa1p2b_fused_schedule_is_used_and_beats_snake():
    n_items, sched = lt.lt_attn_schedule(64, 4096, 32, 8, 148, S=4, W=1020, n_obs=64, fused=True)
    assert n_items == 512 and sched is not None


def test_long_and_tiny_launches_keep_their_orders():
    # 131 072 tokens: banded item order (no static schedule).
    n, sched = lt.lt_attn_schedule(128, 131072, 32, 8, 148, S=4, W=4092, n_obs=128, fused=True)
    assert sched is None and n == 16576     # 1024 q-tiles in 14 bands of 74, 8 KV heads, 2 head pairs each
    # Fewer items than CTAs: one item per CTA already.
    n, sched = lt.lt_attn_schedule(64, 256, 2, 1, 148)
    assert sched is None and n == 2
    # More items than the schedule holds (1536): the snake order (an odd group over
    # 32 768 tokens, and an even group too short for bands).
    n, sched = lt.lt_attn_schedule(128, 32768, 40, 8, 148, S=4, W=2044, n_obs=128, fused=True)
    assert sched is None and n == 128 * 40
    n, sched = lt.lt_attn_schedule(64, 16384, 32, 16, 148, S=4, W=1020, n_obs=64, fused=True)
    assert sched is None and n == 128 * 16


def test_schedule_argument_errors():
    f = library().lt_attn_schedule
    used, n = ctypes.c_int(0), ctypes.c_int(0)
    for args in [(96, 0, 4096, 32, 8, 0, 0, 0, 148),      # head_dim
                 (64, 0, 4096, 30, 8, 0, 0, 0, 148),      # hq not a multiple of hkv
                 (64, 0, 0, 32, 8, 0, 0, 0, 148),         # empty sequence
                 (64, 0, 4096, 32, 8, 0, 0, 0, 0),        # no SMs
                 (64, 1, 4096, 32, 8, 0, 0, 64, 148),     # fused with S + W = 0
                 (64, 1, 4096, 32, 8, 4, 1020, 0, 148)]:  # fused with n_obs = 0
        assert f(*args, ctypes.byref(used), ctypes.byref(n), None, None, 0) == LT_ERR_INVALID_ARG
    # Too small an item buffer for a used schedule: rejected after reporting the sizes.
    off = np.zeros(149, np.int32)
    item = np.zeros(10, np.int32)
    st = f(64, 1, 4096, 32, 8, 4, 1020, 64, 148, ctypes.byref(used), ctypes.byref(n), off.ctypes.data,
           item.ctypes.data, item.size)
    assert st == LT_ERR_INVALID_ARG and used.value == 1 and n.value == 512

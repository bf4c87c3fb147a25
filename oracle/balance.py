"""Reference of the expert-bias update that balances load under noaux_tc
routing (the training side of the router's selection bias).

TEST INFRASTRUCTURE ONLY, like ``oracle.py``: imported by the test suite,
never by the product library (whose moe_bias_update it checks).

What it follows.  "dots3-note 架构深度解析" (mlqm.cn), 稀疏激活, names the
routing method noaux_tc: top-k over sigmoid scores plus a per-expert bias
that steers the choice and is kept out of the routing weights, with no
auxiliary balancing loss.  The pages print no rule for updating that bias.
The reading taken here (the plainest one the name supports): after a batch
has been routed, every expert whose load is above the batch's mean load
gets its bias lowered by a fixed step gamma, every expert below the mean
gets it raised by gamma, and an expert exactly at the mean keeps its bias:

    load_e = #{(t, j) : idx[t, j] = e}            (slots routed to e)
    mean   = T * k / E
    b_e   <- b_e + gamma * sign(mean - load_e)

The comparison is exact (load_e * E against T * k in integers); the bias is
fp32 and the update is one fp32 addition, so the result is a plain
definition with no rounding choices beyond that addition.
"""
from __future__ import annotations

import numpy as np


def expert_loads(topk_idx: np.ndarray, E: int) -> np.ndarray:
    """Slots routed to each expert; indices outside [0, E) are not counted."""
    idx = np.asarray(topk_idx, dtype=np.int64).ravel()
    idx = idx[(idx >= 0) & (idx < E)]
    return np.bincount(idx, minlength=E).astype(np.int64)


def bias_update(topk_idx: np.ndarray, bias: np.ndarray, gamma: float) -> np.ndarray:
    """The updated fp32 bias (a new array; the input is not changed).

    ``topk_idx`` is [T, k] (any shape with T * k entries counts as T * k
    slots), ``bias`` fp32 [E], ``gamma`` the step (rounded to fp32)."""
    b = np.asarray(bias, dtype=np.float32)
    E = b.shape[0]
    n = int(np.asarray(topk_idx).size)
    loads = expert_loads(topk_idx, E)
    # sign(mean - load) with mean = n / E, compared exactly as n against load * E
    s = np.sign(n - loads * E).astype(np.float32)
    g = np.float32(gamma)
    out = b.copy()
    for e in range(E):  # one fp32 addition per expert
        if s[e] > 0:
            out[e] = np.float32(b[e] + g)
        elif s[e] < 0:
            out[e] = np.float32(b[e] - g)
    return out

"""Calibrate the expert-bias tables of the skewed workloads (run offline).

Writes ``sigmoid_top_routing_warp_b200/workload_bias/<name>_<kind>_T<T>_E<E>.txt``
for the prefill (capped Zipf(1.1) load) and grouped (4 hot experts at 5x the
mean load) workloads.  The router it steers is the oracle's (fp32 sigmoid +
bias, group-limited top-k); the logits are iid N(0, (0.02^2) H) draws, the
distribution of x W_g^T for x ~ N(0,1) and W_g ~ N(0, 0.02).  Nothing here
touches the CUDA library.

Update rule (multiplicative load matching, per expert e):
    b_e <- b_e + eta * (log(target_e + 1) - log(load_e + 1))
repeated until the total-variation distance between load and target is below
the tolerance, or the iteration budget runs out.

Usage:  python -m oracle.calibrate_bias [prefill|grouped ...]
"""
from __future__ import annotations

import math
import os
import sys

import numpy as np

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, _ROOT)

from oracle import oracle as O  # noqa: E402
from sigmoid_top_routing_warp_b200 import workloads as W  # noqa: E402


def calibrate(wl: W.Workload, iters: int = 400, eta: float = 0.02, tol: float = 0.02,
              seed: int = 12345, verbose: bool = True) -> tuple[np.ndarray, float]:
    if wl.bias == "zipf":
        target = np.array(W.zipf_targets(wl.T, wl.k, wl.E, seed=wl.seed))
    elif wl.bias == "hot":
        target = np.array(W.hot_targets(wl.T, wl.k, wl.E, seed=wl.seed))
    else:
        raise ValueError(wl.bias)
    cfg = O.Config(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                   n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                   norm_topk_prob=wl.norm_topk_prob)
    rng = np.random.default_rng(seed)
    sd = wl.w_std * wl.x_std * math.sqrt(wl.H)
    logits = (rng.standard_normal((wl.T, wl.E)) * sd).astype(np.float32)
    b = np.zeros(wl.E, dtype=np.float32)
    best = (b.copy(), 1.0)
    total = float(wl.T * wl.k)
    for it in range(iters):
        idx, _, _ = O.route(cfg, logits, b)
        load = np.bincount(idx.ravel(), minlength=wl.E).astype(np.float64)
        tv = 0.5 * np.abs(load - target).sum() / total
        if tv < best[1]:
            best = (b.copy(), tv)
        if verbose and it % 25 == 0:
            print("%s it %d  TV %.4f  max load %d (target %.0f)" %
                  (wl.name, it, tv, load.max(), target.max()))
        if tv < tol:
            break
        b = (b + eta * (np.log(target + 1.0) - np.log(load + 1.0))).astype(np.float32)
    return best


def write_table(wl: W.Workload, b: np.ndarray, tv: float) -> str:
    path = W.bias_table_path(wl)
    os.makedirs(os.path.dirname(path), exist_ok=True)
    with open(path, "w") as f:
        f.write("# expert bias for workload %s (%s load), T=%d E=%d k=%d H=%d\n" %
                (wl.name, wl.bias, wl.T, wl.E, wl.k, wl.H))
        f.write("# written by oracle/calibrate_bias.py; total-variation distance to the\n")
        f.write("# target load on the calibration draw: %.4f\n" % tv)
        for v in b:
            f.write(float(v).hex() + "\n")
    return path


def main(argv):
    names = argv or ["prefill", "grouped"]
    O.set_threads(os.cpu_count() or 1)
    for n in names:
        wl = W.WORKLOADS[n]
        b, tv = calibrate(wl)
        print("%s: TV %.4f -> %s" % (n, tv, write_table(wl, b, tv)))


if __name__ == "__main__":
    main(sys.argv[1:])

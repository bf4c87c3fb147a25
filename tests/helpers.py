"""Shared helpers of the GPU parity tests: moving inputs to the oracle and the
tolerances of the comparison."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O

# Layer-output bar for bf16: relative L2 error <= 1e-2 and max-abs error
# <= 3e-2 * rms(out), against the fp64 oracle on the same bf16 inputs and the
# same routing.
REL_L2_BF16 = 1e-2
MAX_ABS_RMS_BF16 = 3e-2
NEAR_TIE = 1e-4


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_cfg(wl_or_cfg, T=None) -> O.Config:
    c = wl_or_cfg
    return O.Config(T=c.T if T is None else T, H=c.H, E=c.E, k=c.k, I=c.I, n_shared=c.n_shared,
                    n_group=c.n_group, topk_group=c.topk_group, group_topn=c.group_topn,
                    norm_topk_prob=c.norm_topk_prob,
                    routed_scaling_factor=c.routed_scaling_factor)


def oracle_layer_on_tokens(cfg, inp, idx: np.ndarray, w: np.ndarray, tokens) -> np.ndarray:
    """fp64 oracle output for the given tokens, moving only the experts those
    tokens use to the host."""
    tokens = np.asarray(tokens)
    sub_idx = idx[tokens]
    used = np.unique(sub_idx)
    remap = np.full(cfg.E, -1, np.int64)
    remap[used] = np.arange(used.size)
    sel = torch.as_tensor(used, device=inp["w13"].device)
    oc = oracle_cfg(cfg, T=tokens.size)
    oc.E = int(used.size)
    oc.k = cfg.k
    x = u16(inp["x"][torch.as_tensor(tokens, device=inp["x"].device)])
    return O.layer(oc, x, remap[sub_idx].astype(np.int32), w[tokens],
                   u16(inp["w13"][sel]), u16(inp["w2"][sel]), u16(inp["w13s"]),
                   u16(inp["w2s"]))


def assert_close_bf16(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = got - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    rms = np.sqrt(np.mean(ref ** 2))
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= REL_L2_BF16, "%s: rel-L2 %.3e > %.0e" % (what, rel, REL_L2_BF16)
    assert mx <= MAX_ABS_RMS_BF16 * rms, "%s: max-abs %.3e > %.0e * rms %.3e" % (
        what, mx, MAX_ABS_RMS_BF16, rms)
    return rel, mx / max(rms, 1e-30)

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


REL_L2_FP8 = 3e-2


def is_fp8(c) -> bool:
    return getattr(c, "dtype", 0) in (1, "fp8")


def oracle_cfg(wl_or_cfg, T=None) -> O.Config:
    c = wl_or_cfg
    return O.Config(T=c.T if T is None else T, H=c.H, E=c.E, k=c.k, I=c.I, n_shared=c.n_shared,
                    n_group=c.n_group, topk_group=c.topk_group, group_topn=c.group_topn,
                    norm_topk_prob=c.norm_topk_prob,
                    routed_scaling_factor=c.routed_scaling_factor, fp8=is_fp8(c))


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().astype(np.uint8)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().float().numpy()


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
    if oc.fp8:
        return O.layer(oc, x, remap[sub_idx].astype(np.int32), w[tokens],
                       u8(inp["w13"][sel]), u8(inp["w2"][sel]), u8(inp["w13s"]), u8(inp["w2s"]),
                       w13_scale=f32(inp["w13_scale"][sel]), w2_scale=f32(inp["w2_scale"][sel]),
                       w13s_scale=f32(inp["w13s_scale"]), w2s_scale=f32(inp["w2s_scale"]))
    return O.layer(oc, x, remap[sub_idx].astype(np.int32), w[tokens],
                   u16(inp["w13"][sel]), u16(inp["w2"][sel]), u16(inp["w13s"]),
                   u16(inp["w2s"]))


def assert_close_fp8(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel <= REL_L2_FP8, "%s: rel-L2 %.3e > %.0e" % (what, rel, REL_L2_FP8)
    return rel


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


def check_routing_fn(B, cfg, ws, inp):
    """Routing of a forward pass against the oracle fed the GPU's fp32 logits:
    indices and weights must match bit for bit.  Returns (logits, idx, w,
    near-tie count)."""
    L = B.ws_view(ws, cfg, "logits").cpu().numpy()
    idx = B.ws_view(ws, cfg, "topk_idx").cpu().numpy()
    w = B.ws_view(ws, cfg, "topk_w").cpu().numpy()
    oidx, ow, gap = O.route(oracle_cfg(cfg), L, inp["bias"].cpu().numpy())
    assert (idx == oidx).all(), "routing indices differ on %d tokens" % (idx != oidx).any(1).sum()
    assert (w.view(np.uint32) == ow.view(np.uint32)).all(), "routing weights differ"
    return L, idx, w, int((gap < NEAR_TIE).sum())


def cover_tokens(offs, rows, tile):
    """Tokens whose rows reach every expert segment and every token tile of
    the expert GEMMs: for each touched expert its first and last sorted rows,
    and the last row of each `tile`-row token tile (the ragged tail of every
    tile the GEMM launches)."""
    toks = set()
    for e in range(offs.size - 1):
        a, b = int(offs[e]), int(offs[e + 1])
        if b <= a:
            continue
        toks.add(int(rows[a]))
        for t0 in range(a, b, tile):
            toks.add(int(rows[min(t0 + tile, b) - 1]))
    return np.array(sorted(toks), dtype=np.int64)

"""Seeded synthetic workloads of the MoE FFN layer.

This module only draws inputs: activations, router/expert weights and expert
biases of the shapes and distributions the benchmarks use.  It holds none of
the layer's arithmetic and is shared by the tests and the benchmark.

Workloads (layer shapes from the dots3-note pages: hidden 5120, 256 routed +
1 shared expert, top-8, moe_intermediate_size 1536; the grouped variant uses
the Dots1 routing fields with 128 experts, top-6, 2 shared, 1408):

  tiny      T=128,   H=512,  E=32,  k=4, I=128,  1 shared
  decode    T=64,    H=5120, E=256, k=8, I=1536, 1 shared, bias U(-0.1,0.1)
  decode_nobias  the decode shape with a zero bias (near-uniform choice)
  prefill   T=8192,  same shape, bias giving a capped Zipf(1.1) expert load
  fp8_256 / fp8_4096   same shape, e4m3 weights with 128x128 block scales
  grouped   T=16384, H=4096, E=128, k=6, I=1408, 2 shared, n_group=8,
            topk_group=4, bias giving 4 hot experts at 5x the mean load

x ~ N(0,1), every weight ~ N(0, 0.02), all rounded to bf16 (round to nearest
even).  The skewed biases are stored tables (``workload_bias/*.txt``, binary32
hex) calibrated offline against iid N(0, 0.02^2 H) logits, the distribution of
x W_g^T for these draws.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, replace

import torch

_BIAS_DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "workload_bias")


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    n_shared: int = 1
    n_group: int = 1
    topk_group: int = 1
    group_topn: int = 2
    norm_topk_prob: bool = True
    routed_scaling_factor: float = 1.0
    dtype: str = "bf16"          # "bf16" | "fp8"
    bias: str = "uniform"        # "uniform" | "zero" | "zipf" | "hot"
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=T)

    @property
    def Is(self) -> int:
        return self.n_shared * self.I


WORKLOADS = {
    "tiny": Workload("tiny", T=128, H=512, E=32, k=4, I=128),
    "decode": Workload("decode", T=64, H=5120, E=256, k=8, I=1536),
    # The top-8 sigmoid scores of a decode token lie within ~0.05 of each other
    # near 1, so a U(-0.1, 0.1) bias largely decides the choice and T=64 tokens
    # touch ~135-139 experts.  With no bias the choice follows the logits alone
    # and ~229 of 256 experts are touched: the largest weight stream of a
    # 64-token batch.
    "decode_nobias": Workload("decode_nobias", T=64, H=5120, E=256, k=8, I=1536, bias="zero"),
    "prefill": Workload("prefill", T=8192, H=5120, E=256, k=8, I=1536, bias="zipf"),
    "fp8_256": Workload("fp8_256", T=256, H=5120, E=256, k=8, I=1536, dtype="fp8"),
    "fp8_4096": Workload("fp8_4096", T=4096, H=5120, E=256, k=8, I=1536, dtype="fp8"),
    "grouped": Workload("grouped", T=16384, H=4096, E=128, k=6, I=1408, n_shared=2,
                        n_group=8, topk_group=4, bias="hot"),
}


# --------------------------------------------------------------------------
# Target expert loads of the skewed workloads (what the stored biases aim at)
# --------------------------------------------------------------------------

def expert_permutation(E: int, seed: int) -> list[int]:
    g = torch.Generator().manual_seed(1000 + seed)
    return torch.randperm(E, generator=g).tolist()


def zipf_targets(T: int, k: int, E: int, s: float = 1.1, seed: int = 0) -> list[float]:
    """Capped Zipf(s) loads over a seeded permutation of the experts.

    Rank r (1-based) wants T*k * r^-s / sum_q q^-s assignments, but one expert
    can take at most T (a token picks an expert once): loads above T are
    capped and the excess is spread over the lower ranks in proportion to
    their Zipf weight (water filling).
    """
    wts = [r ** -s for r in range(1, E + 1)]
    total = float(T * k)
    load = [0.0] * E
    capped = [False] * E
    while True:
        free = [i for i in range(E) if not capped[i]]
        rest = total - sum(load[i] for i in range(E) if capped[i])
        wsum = sum(wts[i] for i in free)
        changed = False
        for i in free:
            load[i] = rest * wts[i] / wsum
            if load[i] > T:
                load[i] = float(T)
                capped[i] = True
                changed = True
        if not changed:
            break
    perm = expert_permutation(E, seed)
    out = [0.0] * E
    for r, e in enumerate(perm):
        out[e] = load[r]
    return out


def hot_targets(T: int, k: int, E: int, n_hot: int = 4, factor: float = 5.0,
                seed: int = 0) -> list[float]:
    """n_hot seeded experts at factor x the mean load, the rest equal."""
    mean = T * k / E
    hot = set(expert_permutation(E, seed)[:n_hot])
    rest = (T * k - n_hot * factor * mean) / (E - n_hot)
    return [factor * mean if e in hot else rest for e in range(E)]


def bias_table_path(wl: Workload) -> str:
    return os.path.join(_BIAS_DIR, "%s_%s_T%d_E%d.txt" % (wl.name, wl.bias, wl.T, wl.E))


def load_bias_table(path: str) -> torch.Tensor:
    vals = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.append(float.fromhex(line))
    return torch.tensor(vals, dtype=torch.float32)


# --------------------------------------------------------------------------
# Draws
# --------------------------------------------------------------------------

def _gen(device, seed: int) -> torch.Generator:
    return torch.Generator(device=device).manual_seed(seed)


def _normal_bf16(shape, std, g, device) -> torch.Tensor:
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(
        torch.bfloat16)


def quantize_weight_e4m3(w: torch.Tensor, block: int = 128):
    """fp32 [R, C] -> (e4m3 codes [R, C] as uint8, fp32 scales [R/128, C/128]).

    Storage recipe of the FP8 checkpoint workload: scale = amax / 448 per
    128x128 block, codes = round-to-nearest-even e4m3 of w / scale.
    """
    R, C = w.shape
    rb, cb = math.ceil(R / block), math.ceil(C / block)
    wp = torch.zeros(rb * block, cb * block, dtype=torch.float32, device=w.device)
    wp[:R, :C] = w
    blocks = wp.view(rb, block, cb, block)
    amax = blocks.abs().amax(dim=(1, 3))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (blocks / scale[:, None, :, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    q = q.view(rb * block, cb * block)[:R, :C].contiguous()
    return q.view(torch.uint8), scale.contiguous()


def make_inputs(wl: Workload, device="cpu", T: int | None = None, seed: int | None = None,
                weight_copies: int = 1):
    """Draw one layer's inputs.

    Returns a dict of tensors on ``device``:
      x [T,H] bf16, w_router [E,H] bf16, bias [E] fp32,
      w13 [E,2I,H], w2 [E,H,I], w13s [2Is,H], w2s [H,Is]  (bf16, or uint8 e4m3
      codes with fp32 block scales w13_scale [E,2I/128,H/128], w2_scale
      [E,H/128,I/128], w13s_scale, w2s_scale when wl.dtype == "fp8").
    ``weight_copies`` > 1 returns lists of independent expert-weight draws
    (used to rotate weights between timed steps of small workloads).
    """
    T = wl.T if T is None else T
    seed = wl.seed if seed is None else seed
    device = torch.device(device)
    g = _gen(device, seed)
    H, E, I, Is = wl.H, wl.E, wl.I, wl.Is
    out = {"x": _normal_bf16((T, H), wl.x_std, g, device),
           "w_router": _normal_bf16((E, H), wl.w_std, g, device)}
    if wl.bias == "uniform":
        out["bias"] = (torch.rand((E,), generator=g, device=device) * 0.2 - 0.1).float()
    elif wl.bias == "zero":
        out["bias"] = torch.zeros((E,), dtype=torch.float32, device=device)
    else:
        out["bias"] = load_bias_table(bias_table_path(wl)).to(device)

    def experts():
        if wl.dtype == "bf16":
            w13 = torch.empty((E, 2 * I, H), dtype=torch.bfloat16, device=device)
            w2 = torch.empty((E, H, I), dtype=torch.bfloat16, device=device)
            for e in range(E):
                w13[e] = _normal_bf16((2 * I, H), wl.w_std, g, device)
                w2[e] = _normal_bf16((H, I), wl.w_std, g, device)
            w13s = _normal_bf16((2 * Is, H), wl.w_std, g, device)
            w2s = _normal_bf16((H, Is), wl.w_std, g, device)
            return {"w13": w13, "w2": w2, "w13s": w13s, "w2s": w2s}
        w13 = torch.empty((E, 2 * I, H), dtype=torch.uint8, device=device)
        w2 = torch.empty((E, H, I), dtype=torch.uint8, device=device)
        s13 = torch.empty((E, math.ceil(2 * I / 128), math.ceil(H / 128)), device=device)
        s2 = torch.empty((E, math.ceil(H / 128), math.ceil(I / 128)), device=device)
        for e in range(E):
            q, s = quantize_weight_e4m3(
                torch.randn((2 * I, H), generator=g, device=device) * wl.w_std)
            w13[e], s13[e] = q, s
            q, s = quantize_weight_e4m3(
                torch.randn((H, I), generator=g, device=device) * wl.w_std)
            w2[e], s2[e] = q, s
        w13s, s13s = quantize_weight_e4m3(
            torch.randn((2 * Is, H), generator=g, device=device) * wl.w_std)
        w2s, s2s = quantize_weight_e4m3(
            torch.randn((H, Is), generator=g, device=device) * wl.w_std)
        return {"w13": w13, "w2": w2, "w13s": w13s, "w2s": w2s, "w13_scale": s13,
                "w2_scale": s2, "w13s_scale": s13s, "w2s_scale": s2s}

    if weight_copies == 1:
        out.update(experts())
    else:
        copies = [experts() for _ in range(weight_copies)]
        for key in copies[0]:
            out[key] = [c[key] for c in copies]
    return out


# Pre-norm block around the layer: the norm epsilon of the Dots1 config table
# (rms_norm_eps) and a synthetic norm weight.
RMS_NORM_EPS = 1e-6


def make_norm_weight(wl: Workload, device="cpu", seed: int | None = None) -> torch.Tensor:
    """RMSNorm weight gamma [H] bf16: 1 + 0.1 N(0, 1), a trained-looking spread
    around one (seeded separately from the layer's inputs)."""
    g = _gen(torch.device(device), (wl.seed if seed is None else seed) + 7919)
    return (1.0 + 0.1 * torch.randn((wl.H,), generator=g, device=device,
                                    dtype=torch.float32)).to(torch.bfloat16)


# ---------------------------------------------------------------- DSA indexer inputs
@dataclass(frozen=True)
class DsaWorkload:
    """Indexer scoring + top-k: Sq queries against Sk keys, n_heads index heads
    of dim 128 (the pages: 64 heads, top-2048)."""
    name: str
    Sq: int
    Sk: int
    n_heads: int = 64
    topk: int = 2048
    causal: bool = True
    q_offset: int = 0
    seed: int = 0


DSA_WORKLOADS = {
    "dsa_tiny": DsaWorkload("dsa_tiny", Sq=200, Sk=600, n_heads=8, topk=64, causal=False),
    # one 8K prefill chunk attending to itself
    "dsa_prefill": DsaWorkload("dsa_prefill", Sq=8192, Sk=8192),
    # the last 256 queries of a 64K context
    "dsa_long": DsaWorkload("dsa_long", Sq=256, Sk=65536, q_offset=65536 - 256),
}


def make_dsa_inputs(wl: DsaWorkload, device="cpu", seed: int | None = None):
    """q [Sq, nh, 128], k [Sk, nh, 128] ~ N(0, 1) and head weights w [Sq, nh] ~
    N(0, 1/nh), all bf16 (the projections' outputs; the key norm keeps k at
    unit scale)."""
    device = torch.device(device)
    g = _gen(device, (wl.seed if seed is None else seed) + 4242)
    D = 128
    return {"q": _normal_bf16((wl.Sq, wl.n_heads, D), 1.0, g, device),
            "k": _normal_bf16((wl.Sk, wl.n_heads, D), 1.0, g, device),
            "w": _normal_bf16((wl.Sq, wl.n_heads), wl.n_heads ** -0.5, g, device)}


def make_grad_output(wl: Workload, device="cpu", seed: int | None = None) -> torch.Tensor:
    """The upstream gradient of a backward step: dout [T, H] ~ N(0, 1) in bf16
    (its own seed stream, so it never aliases the forward's draws)."""
    seed = (wl.seed if seed is None else seed) + 7919
    return _normal_bf16((wl.T, wl.H), 1.0, _gen(torch.device(device), seed), torch.device(device))

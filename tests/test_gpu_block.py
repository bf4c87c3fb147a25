"""Pre-norm block on the GPU against the oracle: RMSNorm (u = gamma * h /
sqrt(mean(h^2) + eps)) and out = h + MoE(RMSNorm(h)) through the C ABI
(moe_rmsnorm, moe_forward_block).  Parity: u within one bf16 step of the
oracle's once-rounded fp64 value (both sides round a real number to bf16; the
GPU's fp32 pre-rounding value can land on the other side of a rounding
boundary), the block output within the bf16 layer tolerance, routing indices
and weights bit-exact for the GPU's logits."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from tests.helpers import (assert_close_bf16, assert_close_fp8, check_routing_fn, oracle_cfg,
                           u16, u8, f32)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sigmoid_top_routing_warp_b200 import binding
    return binding


@pytest.fixture(scope="module")
def W():
    from sigmoid_top_routing_warp_b200 import workloads
    return workloads


def bf16_steps(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 steps between two arrays of bf16 bit patterns (finite,
    same sign or zero)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(key(a_bits) - key(b_bits))


@pytest.mark.parametrize("T,H", [(64, 5120), (37, 1024), (1, 512), (300, 4096)])
def test_rmsnorm_against_oracle(B, W, T, H):
    wl = W.Workload("norm", T=T, H=H, E=32, k=4, I=128, seed=T + H)
    h = W.make_inputs(wl, device="cuda")["x"]
    if T > 1:
        h[T // 2] *= 0   # an all-zero row: u = 0 (eps keeps the scale finite)
    gamma = W.make_norm_weight(wl, device="cuda")
    u = torch.empty_like(h)
    cfg = B.MoeConfig(T=T, H=H, E=32, k=4, I=128)
    B.moe_rmsnorm(cfg, h, gamma, W.RMS_NORM_EPS, u)
    torch.cuda.synchronize()
    ou, _ = O.rmsnorm(u16(h), u16(gamma), W.RMS_NORM_EPS)
    d = bf16_steps(u16(u), ou)
    assert d.max() <= 1, "RMSNorm differs by %d bf16 steps" % d.max()
    assert (d == 0).mean() >= 0.999, "only %.4f of u bit-exact" % (d == 0).mean()
    if T > 1:
        assert (u[T // 2] == 0).all()


def block_inputs(W, wl):
    inp = W.make_inputs(wl, device="cuda")
    inp["h"] = inp.pop("x")
    inp["gamma"] = W.make_norm_weight(wl, device="cuda")
    return inp


def mk_cfg(B, wl):
    return B.MoeConfig(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                       n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                       norm_topk_prob=wl.norm_topk_prob,
                       routed_scaling_factor=wl.routed_scaling_factor,
                       dtype=B.MOE_DTYPE_FP8_E4M3_BLOCK128 if wl.dtype == "fp8" else B.MOE_DTYPE_BF16)


def run_block(B, W, cfg, inp, out=None):
    ws = B.alloc_workspace(cfg)
    if out is None:
        out = torch.empty_like(inp["h"])
    B.moe_forward_block(cfg, inp["h"], inp["gamma"], W.RMS_NORM_EPS, inp["w_router"],
                        inp["bias"], inp["w13"], inp["w2"], inp.get("w13s"), inp.get("w2s"), out,
                        ws, w13_scale=inp.get("w13_scale"), w2_scale=inp.get("w2_scale"),
                        w13s_scale=inp.get("w13s_scale"), w2s_scale=inp.get("w2s_scale"))
    B.moe_check_device_status(ws)
    return out, ws


def oracle_block_on_tokens(cfg, inp, idx, w, tokens, W):
    """fp64 oracle h + layer(RMSNorm(h)) for the given tokens, moving only the
    experts those tokens use to the host."""
    tokens = np.asarray(tokens)
    sub_idx = idx[tokens]
    used = np.unique(sub_idx)
    remap = np.full(cfg.E, -1, np.int64)
    remap[used] = np.arange(used.size)
    sel = torch.as_tensor(used, device=inp["w13"].device)
    oc = oracle_cfg(cfg, T=tokens.size)
    oc.E = int(used.size)
    h = u16(inp["h"][torch.as_tensor(tokens, device="cuda")])
    g = u16(inp["gamma"])
    cast = u8 if oc.fp8 else u16
    sc = {}
    if oc.fp8:
        sc = dict(w13_scale=f32(inp["w13_scale"][sel]), w2_scale=f32(inp["w2_scale"][sel]),
                  w13s_scale=f32(inp["w13s_scale"]), w2s_scale=f32(inp["w2s_scale"]))
    return O.block(oc, h, g, W.RMS_NORM_EPS, remap[sub_idx].astype(np.int32), w[tokens],
                   cast(inp["w13"][sel]), cast(inp["w2"][sel]), cast(inp["w13s"]),
                   cast(inp["w2s"]), **sc)


SMALL = [
    # name, T, H, E, k, I, n_shared, dtype
    ("block_tiny", 128, 512, 32, 4, 128, 1, "bf16"),
    ("block_ragged_s2", 77, 1024, 64, 6, 256, 2, "bf16"),
    ("block_pairs", 700, 1024, 32, 8, 256, 1, "bf16"),
    ("block_fp8", 96, 512, 32, 4, 256, 1, "fp8"),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_block_small(B, W, case):
    name, T, H, E, k, I, S, dt = case
    wl = W.Workload(name, T=T, H=H, E=E, k=k, I=I, n_shared=S, dtype=dt,
                    seed=sum(name.encode()) % 1000)
    inp = block_inputs(W, wl)
    cfg = mk_cfg(B, wl)
    out, ws = run_block(B, W, cfg, inp)
    # the normalised input the layer ran on
    ou, _ = O.rmsnorm(u16(inp["h"]), u16(inp["gamma"]), W.RMS_NORM_EPS)
    assert bf16_steps(u16(B.ws_view(ws, cfg, "u")), ou).max() <= 1
    _, idx, w, ties = check_routing_fn(B, cfg, ws, inp)
    ref = oracle_block_on_tokens(cfg, inp, idx, w, np.arange(T), W)
    got = out.float().cpu().numpy()
    if dt == "fp8":
        assert_close_fp8(got, ref, name)
    else:
        assert_close_bf16(got, ref, name)
    # element-wise: the single bf16 rounding of out (half a step, at most
    # 2^-8 |out|) plus the layer's max-abs tolerance on the MoE part's rms, so
    # that a MoE part much smaller than the residual is still checked
    hv = inp["h"].float().cpu().numpy()
    moe_rms = np.sqrt(np.mean((ref - hv) ** 2))
    tol = 2.0 ** -8 * np.abs(ref) + (1e-1 if dt == "fp8" else 3e-2) * moe_rms
    bad = np.abs(got - ref) > tol
    assert not bad.any(), "%s: %d elements outside rounding + layer tolerance" % (name, bad.sum())


def test_block_in_place_matches_out_of_place(B, W):
    wl = W.Workload("inplace", T=96, H=512, E=32, k=4, I=128, seed=5)
    inp = block_inputs(W, wl)
    cfg = mk_cfg(B, wl)
    ref, _ = run_block(B, W, cfg, inp)
    h2 = inp["h"].clone()
    inp2 = dict(inp, h=h2)
    run_block(B, W, cfg, inp2, out=h2)
    assert torch.equal(h2, ref)


def test_block_zero_experts_returns_h(B, W):
    wl = W.Workload("zero", T=64, H=512, E=32, k=4, I=128, seed=9)
    inp = block_inputs(W, wl)
    for key in ("w13", "w2", "w13s", "w2s"):
        inp[key] = torch.zeros_like(inp[key])
    out, _ = run_block(B, W, mk_cfg(B, wl), inp)
    assert torch.equal(out, inp["h"])


@pytest.mark.parametrize("name,sample", [("decode", 8), ("fp8_256", 6)])
def test_block_full_size(B, W, name, sample):
    wl = W.WORKLOADS[name]
    inp = block_inputs(W, wl)
    cfg = mk_cfg(B, wl)
    out, ws = run_block(B, W, cfg, inp)
    _, idx, w, ties = check_routing_fn(B, cfg, ws, inp)
    toks = np.unique(np.concatenate([np.random.default_rng(1).choice(cfg.T, sample, replace=False),
                                     [cfg.T - 1]]))
    ref = oracle_block_on_tokens(cfg, inp, idx, w, toks, W)
    got = out[torch.as_tensor(toks, device="cuda")].float().cpu().numpy()
    if wl.dtype == "fp8":
        assert_close_fp8(got, ref, name)
    else:
        assert_close_bf16(got, ref, name)

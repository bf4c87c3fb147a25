"""GPU parity of the layer's backward pass (moe_backward, through the C ABI)
against the fp64 reference oracle/backward.py, on every element of every
gradient: dx, the router weight, the routed experts' gate/up and down
weights, the shared expert's, and the router logits.

The forward's choice comes from the library's own router (moe_route) and is
held fixed on both sides.  The GEMMs accumulate in fp32 over bf16 operands;
the intermediates the GPU rounds to bf16 are the gradients of the gate/up
pre-activations, w * SiLU(g) * u, the per-slot input gradients and the
router's dlogits (each rounding relative error <= u = 2^-8), and dx is
rounded once to bf16.  Bars:
  - dx and dlogits (sums over many terms of either sign, like the forward
    output): relative L2 <= 1e-2 and max-abs <= 3e-2 * rms;
  - weight gradients: relative L2 <= 1e-2 and, element by element,
    |err| <= 2u |ref| + 3e-2 rms.  An element is a sum over an expert's
    token rows of products with one bf16-rounded factor; when its terms
    share a sign (an expert with one or two rows: the gradient is nearly an
    outer product, with elements tens of times the rms) the error is up to
    u relative to the element itself; the 3e-2 rms floor covers elements
    whose terms cancel.
"""
import numpy as np
import pytest
import torch

from helpers import assert_close_bf16
from oracle import backward as BW

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from sigmoid_top_routing_warp_b200 import binding
    assert torch.cuda.is_available()
    return binding


@pytest.fixture(scope="module")
def W():
    from sigmoid_top_routing_warp_b200 import workloads
    return workloads


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def mk_cfg(B, wl):
    return B.MoeConfig(T=wl.T, H=wl.H, E=wl.E, k=wl.k, I=wl.I, n_shared=wl.n_shared,
                       n_group=wl.n_group, topk_group=wl.topk_group, group_topn=wl.group_topn,
                       norm_topk_prob=wl.norm_topk_prob,
                       routed_scaling_factor=wl.routed_scaling_factor)


def backward_on_gpu(B, cfg, inp, dout):
    """Route with the library, then run moe_backward; returns the routing and
    every gradient as host arrays."""
    T, H, E, k, I, Is = cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is
    dev = "cuda"
    ws = B.alloc_workspace(cfg)
    logits = torch.empty((T, E), device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), device=dev)
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], logits, idx, w, ws)
    g = {"dx": torch.full((T, H), 7.0, dtype=torch.bfloat16, device=dev),
         "dwg": torch.full((E, H), 7.0, device=dev),
         "dw13": torch.full((E, 2 * I, H), 7.0, device=dev),
         "dw2": torch.full((E, H, I), 7.0, device=dev),
         "dw13s": torch.full((2 * Is, H), 7.0, device=dev) if Is else None,
         "dw2s": torch.full((H, Is), 7.0, device=dev) if Is else None,
         "dlogits": torch.full((T, E), 7.0, device=dev)}
    bws = B.alloc_backward_workspace(cfg)
    B.moe_backward(cfg, inp["x"], inp["w_router"], logits, idx, w, inp["w13"], inp["w2"],
                   inp["w13s"] if Is else None, inp["w2s"] if Is else None, dout, g["dx"],
                   g["dwg"], g["dw13"], g["dw2"], g["dw13s"], g["dw2s"], bws,
                   dlogits=g["dlogits"])
    B.moe_check_device_status(bws)
    B.moe_check_device_status(ws)
    host = {key: (None if v is None else f64(v)) for key, v in g.items()}
    return idx.cpu().numpy().astype(np.int64), host, g, bws


def oracle_backward(cfg, inp, idx, dout):
    Is = cfg.Is
    return BW.backward(f64(inp["x"]), f64(inp["w_router"]), f64(inp["w13"]), f64(inp["w2"]),
                       f64(inp["w13s"]) if Is else None, f64(inp["w2s"]) if Is else None, idx,
                       f64(dout), norm_topk_prob=cfg.norm_topk_prob,
                       rsf=cfg.routed_scaling_factor)


U_BF16 = 2.0 ** -8


def assert_close_grad(g, r, what):
    """Weight-gradient bar (see the module docstring); returns (rel-L2, worst
    |err| / (2u |ref| + 3e-2 rms))."""
    err = np.abs(g - r)
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    rms = np.sqrt(np.mean(r ** 2))
    bound = 2 * U_BF16 * np.abs(r) + 3e-2 * rms
    ratio = err / bound
    i = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert rel <= 1e-2, "%s: rel-L2 %.3e > 1e-2" % (what, rel)
    assert ratio[i] <= 1.0, "%s: at %s got %.6e ref %.6e, |err| %.3e > bound %.3e" % (
        what, tuple(int(v) for v in i), g[i], r[i], err[i], bound[i])
    return rel, float(ratio[i])


def compare(got, ref, name, Is, skip=()):
    dense = [("dx", "dx"), ("dlogits", "dlogits")]
    weights = [("dwg", "dwg"), ("dw13", "dw13"), ("dw2", "dw2")]
    if Is:
        weights += [("dw13s", "dw13s"), ("dw2s", "dw2s")]
    worst = {}
    for g_key, r_key in dense:
        if g_key in skip:
            continue
        worst[g_key] = assert_close_bf16(got[g_key], ref[r_key], "%s %s" % (name, g_key))
    for g_key, r_key in weights:
        if g_key in skip:
            continue
        worst[g_key] = assert_close_grad(got[g_key], ref[r_key], "%s %s" % (name, g_key))
    return worst


CASES = [
    # name, T, H, E, k, I, n_shared, n_group, topk_group, norm, rsf, bias
    ("tiny", 128, 512, 32, 4, 128, 1, 1, 1, True, 1.0, "uniform"),
    ("ragged_no_norm_rsf", 300, 640, 64, 6, 256, 2, 1, 1, False, 2.5, "uniform"),
    ("grouped_no_shared", 200, 512, 64, 6, 128, 0, 4, 2, True, 1.0, "uniform"),
    ("k1", 150, 512, 32, 1, 128, 1, 1, 1, True, 1.0, "uniform"),
    ("one_token", 1, 512, 32, 8, 256, 1, 1, 1, True, 1.0, "uniform"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_against_fp64_oracle(B, W, case):
    name, T, H, E, k, I, S, G, tg, norm, rsf, bias = case
    wl = W.Workload(name, T=T, H=H, E=E, k=k, I=I, n_shared=S, n_group=G, topk_group=tg,
                    norm_topk_prob=norm, routed_scaling_factor=rsf, bias=bias,
                    seed=sum(name.encode()) % 1000)
    inp = W.make_inputs(wl, device="cuda")
    dout = W.make_grad_output(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    idx, got, _, _ = backward_on_gpu(B, cfg, inp, dout)
    ref = oracle_backward(cfg, inp, idx, dout)
    no_router = k == 1 and norm  # w = rsf exactly: no gradient reaches the router
    worst = compare(got, ref, name, cfg.Is, skip=("dlogits", "dwg") if no_router else ())
    if no_router:
        assert (got["dlogits"] == 0).all() and (got["dwg"] == 0).all()
        assert np.abs(ref["dlogits"]).max() < 1e-12
    # experts no token chose get exactly zero weight gradients
    unused = np.setdiff1d(np.arange(E), np.unique(idx))
    assert (got["dw13"][unused] == 0).all() and (got["dw2"][unused] == 0).all()
    print("%s: %s" % (name, ", ".join("%s %.1e/%.1e" % (kk, a, b) for kk, (a, b) in worst.items())))


def test_backward_hot_expert_spans_many_tiles(B, W):
    """A bias that makes one expert every token's first choice: its segment
    holds all T = 1000 rows (eight 128-row tiles; the weight gradients
    contract over 1000 rows, 16 K steps) beside sparse experts."""
    wl = W.Workload("bwd_hot", T=1000, H=512, E=32, k=2, I=256, n_shared=1, seed=31)
    inp = W.make_inputs(wl, device="cuda")
    inp["bias"] = torch.zeros(32, device="cuda")
    inp["bias"][5] = 10.0
    dout = W.make_grad_output(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    idx, got, _, _ = backward_on_gpu(B, cfg, inp, dout)
    assert (idx[:, 0] == 5).all()
    compare(got, oracle_backward(cfg, inp, idx, dout), "hot", cfg.Is)


def test_backward_is_deterministic_and_linear(B, W):
    """Two calls give bit-identical gradients (fixed tile schedule, fixed
    summation orders); dout = 0 gives all-zero gradients."""
    wl = W.Workload("bwd_det", T=257, H=512, E=32, k=4, I=128, n_shared=1, seed=8)
    inp = W.make_inputs(wl, device="cuda")
    dout = W.make_grad_output(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    _, a, ga, _ = backward_on_gpu(B, cfg, inp, dout)
    _, b, gb, _ = backward_on_gpu(B, cfg, inp, dout)
    for key in ga:
        if ga[key] is not None:
            assert torch.equal(ga[key], gb[key]), key
    _, z, _, _ = backward_on_gpu(B, cfg, inp, torch.zeros_like(dout))
    for key, v in z.items():
        if v is not None:
            assert (v == 0).all(), key

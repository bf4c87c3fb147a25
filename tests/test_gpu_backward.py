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
    # M = I = 384 and H = 768 end half-way into a 256-row pair tile; group routing
    ("half_pair_tiles", 333, 768, 64, 6, 384, 2, 8, 4, True, 1.0, "uniform"),
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


def test_backward_full_size_prefill(B, W):
    """The Zipf prefill workload (T = 8192, H = 5120, E = 256, k = 8, I = 1536,
    one shared expert), sampled where the fp64 oracle can follow it:
      - dx and dlogits of sampled tokens: the oracle's backward on those
        tokens with only their experts (a token's dx and dlogits depend on no
        other token);
      - dW13_e and dW2_e of the least-loaded, a median and the most-loaded
        expert (7000+ rows): the oracle's per-expert gradients from the rows
        that chose the expert, with their routing weights;
      - dW13s and dW2s over all 8192 tokens (the shared expert, weight 1);
      - dW_g against dlogits^T x in fp64 from the kernel's own dlogits (a
        property of that GEMM at full size), within the dot-product error
        bound of dlogits' bf16 rounding."""
    wl = W.WORKLOADS["prefill"]
    inp = W.make_inputs(wl, device="cuda")
    dout = W.make_grad_output(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    T, H, E, k, I, Is = cfg.T, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is
    dev = "cuda"
    ws = B.alloc_workspace(cfg)
    logits = torch.empty((T, E), device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), device=dev)
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], logits, idx, w, ws)
    dx = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    dwg = torch.empty((E, H), device=dev)
    dw13 = torch.empty((E, 2 * I, H), device=dev)
    dw2 = torch.empty((E, H, I), device=dev)
    dw13s = torch.empty((2 * Is, H), device=dev)
    dw2s = torch.empty((H, Is), device=dev)
    dlg = torch.empty((T, E), device=dev)
    bws = B.alloc_backward_workspace(cfg)
    B.moe_backward(cfg, inp["x"], inp["w_router"], logits, idx, w, inp["w13"], inp["w2"],
                   inp["w13s"], inp["w2s"], dout, dx, dwg, dw13, dw2, dw13s, dw2s, bws,
                   dlogits=dlg)
    B.moe_check_device_status(bws)
    idx_h = idx.cpu().numpy().astype(np.int64)
    w_h = w.cpu().numpy().astype(np.float64)

    # sampled tokens, with only their experts
    toks = np.array([0, 4321, T - 1])
    used = np.unique(idx_h[toks])
    remap = np.full(E, -1, np.int64)
    remap[used] = np.arange(used.size)
    sel = torch.as_tensor(used, device=dev)
    ref = BW.backward(f64(inp["x"][toks]), f64(inp["w_router"][sel]), f64(inp["w13"][sel]),
                      f64(inp["w2"][sel]), f64(inp["w13s"]), f64(inp["w2s"]),
                      remap[idx_h[toks]], f64(dout[toks]))
    assert_close_bf16(f64(dx[toks]), ref["dx"], "prefill dx")
    assert_close_bf16(f64(dlg[toks][:, sel]), ref["dlogits"], "prefill dlogits")
    assert (dlg[toks].cpu().numpy()[:, np.setdiff1d(np.arange(E), used)] == 0).all()

    # three experts' weight gradients from the rows that chose them
    loads = np.bincount(idx_h.ravel(), minlength=E)
    order = np.argsort(loads, kind="stable")
    touched = order[loads[order] > 0]
    for e in (touched[0], touched[touched.size // 2], touched[-1]):
        t, j = np.nonzero(idx_h == e)
        ti = torch.as_tensor(t, device=dev)
        r13, r2 = BW.expert_grads(f64(inp["x"][ti]), f64(dout[ti]), w_h[t, j],
                                  f64(inp["w13"][int(e)]), f64(inp["w2"][int(e)]))
        assert_close_grad(f64(dw13[int(e)]), r13, "prefill dw13[%d] (%d rows)" % (e, t.size))
        assert_close_grad(f64(dw2[int(e)]), r2, "prefill dw2[%d] (%d rows)" % (e, t.size))

    # the shared expert over every token
    r13s, r2s = BW.expert_grads(f64(inp["x"]), f64(dout), np.ones(T), f64(inp["w13s"]),
                                f64(inp["w2s"]))
    assert_close_grad(f64(dw13s), r13s, "prefill dw13s")
    assert_close_grad(f64(dw2s), r2s, "prefill dw2s")

    # dW_g is dlogits^T x.  Its only rounding is that of dlogits to bf16 (x
    # is exact, the fp32 accumulation adds ~1e-5 rms), so every element obeys
    # the dot-product bound |err| <= 2u sum_t |dlogits[t, e] x[t, h]|; an
    # rms-relative bar does not fit here, where tokens with a small sum of
    # chosen scores give large terms that cancel
    x64 = f64(inp["x"])
    d64 = f64(dlg)
    ref_g = d64.T @ x64
    bound = 2 * U_BF16 * (np.abs(d64).T @ np.abs(x64)) + 1e-6 * np.sqrt(np.mean(ref_g ** 2))
    err = np.abs(f64(dwg) - ref_g)
    i = np.unravel_index(np.argmax(err / bound), err.shape)
    assert (err <= bound).all(), "prefill dwg at %s: |err| %.3e > bound %.3e" % (
        tuple(int(v) for v in i), err[i], bound[i])
    assert np.linalg.norm(f64(dwg) - ref_g) <= 1e-2 * np.linalg.norm(ref_g)

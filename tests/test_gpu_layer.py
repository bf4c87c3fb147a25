"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Routing indices and weights, and the dispatch permutation, must match the
oracle bit for bit when the oracle is fed the GPU's fp32 logits; logits and
the layer output must meet the stated tolerances.  Sizes span several tiles
with ragged tails; the full-size workloads are checked on every token for
routing and permutation and on sampled tokens for the layer output.
"""
import numpy as np
import pytest
import torch

from helpers import (NEAR_TIE, assert_close_bf16, oracle_cfg, oracle_layer_on_tokens, u16)
from oracle import oracle as O

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


def mk_cfg(B, wl, T=None):
    return B.MoeConfig(T=wl.T if T is None else T, H=wl.H, E=wl.E, k=wl.k, I=wl.I,
                       n_shared=wl.n_shared, n_group=wl.n_group, topk_group=wl.topk_group,
                       group_topn=wl.group_topn, norm_topk_prob=wl.norm_topk_prob,
                       routed_scaling_factor=wl.routed_scaling_factor)


def run_forward(B, cfg, inp):
    ws = B.alloc_workspace(cfg)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                  inp.get("w13s"), inp.get("w2s"), out, ws)
    B.moe_check_device_status(ws)
    return out, ws


def check_routing(B, cfg, ws, inp, exact_logits_tol=True):
    L = B.ws_view(ws, cfg, "logits").cpu().numpy()
    idx = B.ws_view(ws, cfg, "topk_idx").cpu().numpy()
    w = B.ws_view(ws, cfg, "topk_w").cpu().numpy()
    oc = oracle_cfg(cfg)
    oidx, ow, gap = O.route(oc, L, inp["bias"].cpu().numpy())
    assert (idx == oidx).all(), "routing indices differ on %d tokens" % (idx != oidx).any(1).sum()
    assert (w.view(np.uint32) == ow.view(np.uint32)).all(), "routing weights differ"
    return L, idx, w, int((gap < NEAR_TIE).sum())


def check_logits(cfg, L, inp, tokens=None):
    oc = oracle_cfg(cfg)
    x = inp["x"] if tokens is None else inp["x"][torch.as_tensor(tokens, device="cuda")]
    oc.T = x.shape[0]
    ref = O.router_logits(oc, u16(x), u16(inp["w_router"]))
    got = L if tokens is None else L[tokens]
    scale = max(1.0, float(np.std(ref)))
    assert np.abs(got - ref).max() <= 1e-4 * scale


def check_permutation(B, cfg, ws, idx):
    oc = oracle_cfg(cfg)
    offs, rows, pos = O.permute(oc, idx)
    assert (B.ws_view(ws, cfg, "offsets").cpu().numpy() == offs).all()
    assert (B.ws_view(ws, cfg, "rows").cpu().numpy() == rows).all()
    assert (B.ws_view(ws, cfg, "pos").cpu().numpy() == pos).all()
    return offs


# ------------------------------------------------------------------ small shapes

SMALL = [
    # name, T, H, E, k, I, n_shared, n_group, topk_group
    ("tiny", 128, 512, 32, 4, 128, 1, 1, 1),
    ("one_token", 1, 512, 64, 6, 256, 2, 1, 1),
    ("ragged7", 7, 1024, 64, 6, 256, 1, 1, 1),
    ("ragged300", 300, 1024, 64, 6, 256, 2, 1, 1),
    ("grouped", 257, 768, 128, 6, 128, 2, 8, 3),
    ("no_shared", 96, 512, 96, 8, 256, 0, 1, 1),
    ("k_equals_E", 40, 512, 32, 32, 128, 1, 1, 1),
    ("many_tokens", 1500, 512, 32, 4, 128, 1, 1, 1),
    # prefill-sized: CTA-pair GEMMs with ragged tiles and H, I not multiples of 256
    ("pair_ragged", 2000, 640, 32, 4, 384, 1, 1, 1),
    ("pair_grouped", 4096, 1024, 64, 6, 256, 2, 4, 2),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_layer_small_shapes_against_oracle(B, W, case):
    name, T, H, E, k, I, S, G, tg = case
    wl = W.Workload(name, T=T, H=H, E=E, k=k, I=I, n_shared=S, n_group=G, topk_group=tg,
                    seed=sum(name.encode()) % 1000)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    L, idx, w, ties = check_routing(B, cfg, ws, inp)
    check_logits(cfg, L, inp)
    check_permutation(B, cfg, ws, idx)
    ref = oracle_layer_on_tokens(cfg, inp, idx, w, np.arange(T))
    rel, mx = assert_close_bf16(out.float().cpu().numpy(), ref, name)
    print("%s: rel-L2 %.2e, max-abs/rms %.2e, near-ties %d" % (name, rel, mx, ties))


# routing options and the largest configurations the router accepts
ROUTING_EDGE = [
    # name, T, H, E, k, I, n_shared, n_group, topk_group, norm_topk_prob, routed_scaling_factor
    ("no_norm_rsf2.5", 200, 512, 64, 3, 128, 1, 1, 1, False, 2.5),
    ("norm_rsf0.5", 200, 512, 64, 6, 128, 1, 1, 1, True, 0.5),
    ("k1_norm", 150, 512, 32, 1, 128, 1, 1, 1, True, 1.0),
    ("max_E_k", 96, 128, 1024, 32, 128, 1, 1, 1, True, 1.0),
    ("max_groups", 96, 128, 1024, 16, 128, 0, 32, 4, True, 1.0),
    ("E768_groups", 130, 256, 768, 8, 128, 1, 8, 3, True, 1.0),
]


@pytest.mark.parametrize("case", ROUTING_EDGE, ids=[c[0] for c in ROUTING_EDGE])
def test_routing_options_and_max_sizes_against_oracle(B, W, case):
    name, T, H, E, k, I, S, G, tg, norm, rsf = case
    wl = W.Workload(name, T=T, H=H, E=E, k=k, I=I, n_shared=S, n_group=G, topk_group=tg,
                    norm_topk_prob=norm, routed_scaling_factor=rsf,
                    seed=sum(name.encode()) % 1000)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    L, idx, w, ties = check_routing(B, cfg, ws, inp)
    check_permutation(B, cfg, ws, idx)
    if k == 1 and norm:
        assert (w == np.float32(rsf)).all()
    ref = oracle_layer_on_tokens(cfg, inp, idx, w, np.arange(T))
    rel, mx = assert_close_bf16(out.float().cpu().numpy(), ref, name)
    print("%s: rel-L2 %.2e, max-abs/rms %.2e, near-ties %d" % (name, rel, mx, ties))


def test_one_expert_takes_every_token(B, W):
    """A bias that makes one expert every token's first choice: its segment
    holds all T rows, a dozen CTA-pair token tiles of one expert."""
    wl = W.Workload("hot", T=3000, H=640, E=32, k=2, I=384, n_shared=1, seed=11)
    inp = W.make_inputs(wl, device="cuda")
    inp["bias"] = torch.zeros(32, device="cuda")
    inp["bias"][5] = 10.0
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    L, idx, w, _ = check_routing(B, cfg, ws, inp)
    offs = check_permutation(B, cfg, ws, idx)
    assert (idx[:, 0] == 5).all() and offs[6] - offs[5] == wl.T
    toks = np.unique(np.concatenate([np.random.default_rng(1).choice(wl.T, 48, replace=False),
                                     [0, wl.T - 1]]))
    ref = oracle_layer_on_tokens(cfg, inp, idx, w, toks)
    assert_close_bf16(out[torch.as_tensor(toks, device="cuda")].float().cpu().numpy(), ref, "hot")


def test_empty_batch_is_a_no_op(B, W):
    """T = 0: every call validates its arguments and returns without a launch."""
    wl = W.Workload("empty", T=4, H=512, E=32, k=4, I=128, seed=2)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl, T=0)
    ws = B.alloc_workspace(cfg)
    out = torch.full((4, wl.H), 7.0, dtype=torch.bfloat16, device="cuda")
    B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                  inp["w13s"], inp["w2s"], out, ws)
    torch.cuda.synchronize()
    B.moe_check_device_status(ws)
    assert (out.float() == 7.0).all()


@pytest.mark.parametrize("k", [6, 1])
def test_stage_entry_points_match_forward(B, W, k):
    """The step calls reproduce moe_forward bit for bit (with k = 1 the routed
    outputs y are fp32)."""
    wl = W.Workload("stages", T=200, H=1024, E=64, k=k, I=256, n_shared=1, seed=5)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    T, E, k, H = cfg.T, cfg.E, cfg.k, cfg.H
    dev = "cuda"
    ws2 = B.alloc_workspace(cfg)
    logits = torch.empty((T, E), device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), device=dev)
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], logits, idx, w, ws2)
    idx2 = torch.empty_like(idx)
    w2 = torch.empty_like(w)
    B.moe_route_from_logits(cfg, logits, inp["bias"], idx2, w2)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    rows = torch.empty((T * k,), dtype=torch.int32, device=dev)
    pos = torch.empty((T * k,), dtype=torch.int32, device=dev)
    B.moe_permute(cfg, idx, offsets, rows, pos, ws2)
    y = torch.empty((T * k, H), dtype=torch.float32 if k == 1 else torch.bfloat16, device=dev)
    ysh = torch.empty((T, H), dtype=torch.float32, device=dev)
    B.moe_expert_ffn(cfg, inp["x"], offsets, rows, pos, w, inp["w13"], inp["w2"], inp["w13s"],
                     inp["w2s"], y, ysh, ws2)
    out2 = torch.empty_like(out)
    B.moe_combine(cfg, y, pos, ysh, out2)
    B.moe_check_device_status(ws2)
    assert torch.equal(logits, B.ws_view(ws, cfg, "logits"))
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    assert torch.equal(idx, B.ws_view(ws, cfg, "topk_idx"))
    assert torch.equal(pos, B.ws_view(ws, cfg, "pos"))
    assert torch.equal(y, B.ws_view(ws, cfg, "y"))
    assert torch.equal(out, out2)


def test_forward_is_deterministic(B, W):
    wl = W.Workload("det", T=513, H=1024, E=64, k=8, I=256, n_shared=1, seed=9)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    a, _ = run_forward(B, cfg, inp)
    b, _ = run_forward(B, cfg, inp)
    assert torch.equal(a, b)


def test_bias_only_steers_choice(B, W):
    """Forcing the choice with a large bias: the weights are the renormalised
    unbiased scores of the forced experts."""
    wl = W.Workload("forced", T=64, H=512, E=32, k=4, I=128, seed=3)
    inp = W.make_inputs(wl, device="cuda")
    forced = [2, 9, 17, 30]
    inp["bias"] = torch.zeros(32, device="cuda")
    inp["bias"][forced] = 10.0
    cfg = mk_cfg(B, wl)
    _, ws = run_forward(B, cfg, inp)
    L, idx, w, _ = check_routing(B, cfg, ws, inp)
    assert (np.sort(idx, 1) == np.array(forced)).all()
    s = O.sigmoid_f32(L).astype(np.float64)
    sel = np.take_along_axis(s, idx, 1)
    assert np.allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-6)


def test_zero_input_gives_zero_output(B, W):
    wl = W.Workload("zero", T=48, H=512, E=32, k=4, I=128, seed=4)
    inp = W.make_inputs(wl, device="cuda")
    inp["x"].zero_()
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    assert (out.float() == 0).all()
    w = B.ws_view(ws, cfg, "topk_w")
    assert torch.allclose(w, torch.full_like(w, 0.25))


# ------------------------------------------------------------------ full sizes

def full_size_check(B, W, name, sample):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    L, idx, w, ties = check_routing(B, cfg, ws, inp)
    offs = check_permutation(B, cfg, ws, idx)
    rng = np.random.default_rng(0)
    toks = rng.choice(cfg.T, size=min(sample, cfg.T), replace=False)
    # include a token of the most loaded expert and the last token
    big = int(np.argmax(np.diff(offs)))
    toks = np.unique(np.concatenate([toks, [np.where((idx == big).any(1))[0][0], cfg.T - 1]]))
    check_logits(cfg, L, inp, toks)
    ref = oracle_layer_on_tokens(cfg, inp, idx, w, toks)
    rel, mx = assert_close_bf16(out[torch.as_tensor(toks, device="cuda")].float().cpu().numpy(),
                                ref, name)
    loads = np.diff(offs)
    print("%s: rel-L2 %.2e, max-abs/rms %.2e, near-ties %d/%d, experts touched %d, max load %d"
          % (name, rel, mx, ties, cfg.T, (loads > 0).sum(), loads.max()))


def test_full_size_decode(B, W):
    full_size_check(B, W, "decode", sample=6)


def test_full_size_decode_nobias(B, W):
    """The decode shape with a zero bias: ~229 experts touched, one or two rows
    each, the largest set of segments a 64-token batch has."""
    full_size_check(B, W, "decode_nobias", sample=6)


def test_full_size_prefill_zipf(B, W):
    full_size_check(B, W, "prefill", sample=4)


def test_full_size_grouped(B, W):
    full_size_check(B, W, "grouped", sample=4)


def test_bounded_wait_timeout_is_reported_and_context_survives(B, W):
    """Failure detection without a GPU fault: with MOE_FLAG_TEST_STALL the
    router GEMM's first CTA never fills one pipeline stage, its bounded wait
    runs out (~1 s), the kernel records a timeout and returns.  The host sees
    MOE_ERR_TIMEOUT, and the next normal call on the same context is exact."""
    wl = W.Workload("stall", T=64, H=1024, E=64, k=4, I=128, seed=6)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    cfg.flags = B.MOE_FLAG_TEST_STALL
    ws = B.alloc_workspace(cfg)
    logits = torch.empty((wl.T, wl.E), device="cuda")
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), device="cuda")
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], logits, idx, w, ws)
    with pytest.raises(B.MoeError) as ei:
        B.moe_check_device_status(ws)
    assert ei.value.status == B.MOE_ERR_TIMEOUT
    cfg.flags = 0
    B.moe_route(cfg, inp["x"], inp["w_router"], inp["bias"], logits, idx, w, ws)
    B.moe_check_device_status(ws)
    oidx, ow, _ = O.route(oracle_cfg(cfg), logits.cpu().numpy(), inp["bias"].cpu().numpy())
    assert (idx.cpu().numpy() == oidx).all()


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_tile_claim_counters_reset_and_repeat(B, W, name):
    """The weight-major GEMMs claim tiles from counters in the workspace status
    block (words 16..21); every call must leave them at zero, and a second call
    on the same workspace must produce the same output bit for bit (no tile
    skipped or done twice)."""
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out1, ws = run_forward(B, cfg, inp)
    words = ws[:256].view(torch.int32).cpu().numpy()
    assert (words[16:22] == 0).all(), words[16:22]
    out2 = torch.empty_like(out1)
    for _ in range(3):
        B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                      inp.get("w13s"), inp.get("w2s"), out2, ws)
    B.moe_check_device_status(ws)
    assert torch.equal(out1, out2)
    assert (ws[:256].view(torch.int32).cpu().numpy()[16:22] == 0).all()

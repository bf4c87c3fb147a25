"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle.

Routing indices and weights, and the dispatch permutation, must match the
oracle bit for bit when the oracle is fed the GPU's fp32 logits; logits and
the layer output must meet the stated tolerances.  Sizes span several tiles
with ragged tails; the full-size workloads are checked on every token for
routing, permutation and logits, and for the layer output on every token at
decode and on a token set that reaches every expert segment and every token
tile at prefill sizes.
"""
import numpy as np
import pytest
import torch

from helpers import (NEAR_TIE, assert_close_bf16, cover_tokens, oracle_cfg,
                     oracle_layer_on_tokens, u16)
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

def group_gap(cfg, L, bias):
    """Per token, the gap between the topk_group-th and the next group score
    (sum of a group's top group_topn biased scores, larger first), +inf
    without group routing: a near-tie there can flip which groups are kept."""
    if cfg.n_group <= 1:
        return np.full(L.shape[0], np.inf, np.float32)
    c = (O.sigmoid_f32(L) + bias.astype(np.float32)).astype(np.float32)
    c = np.sort(c.reshape(L.shape[0], cfg.n_group, -1), axis=2)[:, :, ::-1]
    gs = np.zeros(c.shape[:2], np.float32)
    for j in range(cfg.group_topn):
        gs = (gs + c[:, :, j]).astype(np.float32)
    gs = np.sort(gs, axis=1)[:, ::-1]
    return gs[:, cfg.topk_group - 1] - gs[:, cfg.topk_group]


def near_tie_consistency(cfg, inp, idx, gap_gpu):
    """The oracle routes its own fp64 logits (rounded to fp32): every token
    whose chosen set differs from the GPU's must be a near-tie (gap between the
    k-th and (k+1)-th biased score, or with group routing between the kept
    and the next group score, below NEAR_TIE), since only the last bits of
    the logits differ.  Returns (near-ties, tokens routed differently)."""
    oc = oracle_cfg(cfg)
    ref_L = O.router_logits(oc, u16(inp["x"]), u16(inp["w_router"])).astype(np.float32)
    bias = inp["bias"].cpu().numpy()
    oidx, _, ogap = O.route(oc, ref_L, bias)
    # the same chosen set in another slot order is two chosen keys in a near
    # tie, not a different choice
    differ = (np.sort(oidx, 1) != np.sort(idx, 1)).any(1)
    near = (np.minimum(gap_gpu, ogap) < NEAR_TIE)
    if cfg.n_group > 1:
        near |= group_gap(cfg, ref_L, bias) < NEAR_TIE
    assert not (differ & ~near).any(), \
        "%d tokens routed differently that are not near-ties" % (differ & ~near).sum()
    return int((gap_gpu < NEAR_TIE).sum()), int(differ.sum())


def full_size_check(B, W, name, every_token=False, tile=256):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    out, ws = run_forward(B, cfg, inp)
    L = B.ws_view(ws, cfg, "logits").cpu().numpy()
    idx = B.ws_view(ws, cfg, "topk_idx").cpu().numpy()
    w = B.ws_view(ws, cfg, "topk_w").cpu().numpy()
    oidx, ow, gap = O.route(oracle_cfg(cfg), L, inp["bias"].cpu().numpy())
    assert (idx == oidx).all(), "routing indices differ on %d tokens" % (idx != oidx).any(1).sum()
    assert (w.view(np.uint32) == ow.view(np.uint32)).all(), "routing weights differ"
    offs = check_permutation(B, cfg, ws, idx)
    check_logits(cfg, L, inp)
    ties, differ = near_tie_consistency(cfg, inp, idx, gap)
    # near-ties (counted, and compared bit for bit like every other token) stay
    # a small share of the batch: ~1.3 % at prefill, ~2 % at T = 256
    assert ties <= cfg.T // 20 + 2, "near-ties %d of %d tokens" % (ties, cfg.T)
    if every_token:
        toks = np.arange(cfg.T)
    else:
        rows = B.ws_view(ws, cfg, "rows").cpu().numpy()
        toks = cover_tokens(offs, rows, tile)
        assert np.isin(np.arange(cfg.E)[np.diff(offs) > 0],
                       np.unique(idx[toks])).all(), "an expert is not covered"
    ref = oracle_layer_on_tokens(cfg, inp, idx, w, toks)
    rel, mx = assert_close_bf16(out[torch.as_tensor(toks, device="cuda")].float().cpu().numpy(),
                                ref, name)
    loads = np.diff(offs)
    print("%s: %d tokens compared, rel-L2 %.2e, max-abs/rms %.2e, near-ties %d/%d (routed "
          "differently from the oracle's own logits: %d), experts touched %d, max load %d"
          % (name, toks.size, rel, mx, ties, cfg.T, differ, (loads > 0).sum(), loads.max()))


def test_full_size_decode(B, W):
    """Every token of the 64-token decode batch against the oracle."""
    full_size_check(B, W, "decode", every_token=True)


def test_full_size_decode_nobias(B, W):
    """The decode shape with a zero bias: ~229 experts touched, one or two rows
    each, the largest set of segments a 64-token batch has; every token."""
    full_size_check(B, W, "decode_nobias", every_token=True)


def test_full_size_prefill_zipf(B, W):
    """Zipf-skewed prefill: a token of every expert and the last row of every
    256-row token tile (the CTA-pair GEMMs' tiles)."""
    full_size_check(B, W, "prefill", tile=256)


def test_full_size_grouped(B, W):
    full_size_check(B, W, "grouped", tile=256)


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


@pytest.mark.parametrize("shape", ["tiny", "pair"])
def test_dirty_claim_counters_are_reset_and_reported(B, W, shape):
    """A workspace whose tile-claim words hold garbage (a caller that did not
    zero it) still gives the clean run's output bit for bit: every call zeroes
    those words on its stream before the first claiming launch.  Counters that
    are non-zero once the stream has drained (what a launch that stopped
    part-way leaves; planted here by writing one after a call) make
    moe_check_device_status return MOE_ERR_WORKSPACE and clear the block."""
    if shape == "tiny":
        wl = W.WORKLOADS["tiny"]
    else:  # CTA-pair GEMMs (about 250 rows per expert)
        wl = W.Workload("pair_dirty", T=2000, H=640, E=32, k=4, I=384, n_shared=1, seed=21)
    inp = W.make_inputs(wl, device="cuda")
    cfg = mk_cfg(B, wl)
    ref, _ = run_forward(B, cfg, inp)
    ws = B.alloc_workspace(cfg)
    ws[64:256] = 0x5A  # words 16..63 hold garbage; the status word is zero
    out = torch.empty_like(ref)
    B.moe_forward(cfg, inp["x"], inp["w_router"], inp["bias"], inp["w13"], inp["w2"],
                  inp.get("w13s"), inp.get("w2s"), out, ws)
    B.moe_check_device_status(ws)
    assert torch.equal(out, ref)
    ws[64:68].view(torch.int32)[0] = 3  # a claim counter left behind
    with pytest.raises(B.MoeError) as ei:
        B.moe_check_device_status(ws)
    assert ei.value.status == B.MOE_ERR_WORKSPACE
    assert (ws[:256] == 0).all()
    B.moe_check_device_status(ws)
